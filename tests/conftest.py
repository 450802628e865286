import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.get()


def pytest_terminal_summary(terminalreporter):
    """Print how many routed rows each GPU parity workload matched exactly and
    how many differed from the oracle under each excuse."""
    try:
        from tests import fvtest
    except ImportError:
        return
    if not fvtest.RECORDED:
        return
    terminalreporter.write_sep("-", "routing lists vs the oracle")
    for name, res in fvtest.RECORDED.items():
        terminalreporter.write_line(f"{name}: {res.summary()}")
