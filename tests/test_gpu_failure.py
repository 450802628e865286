"""The failure path of the attention kernel (needs a B200).

Kernel failures must surface, not be masked (zskr.cn FastVideo VSA guide,
section 6): every wait inside the kernels is bounded, and one that runs out
raises FVATTN_FLAG_TIMEOUT, after which the kernel lets its copies and
products in flight finish, frees its tensor memory and returns. Here a
host-written test word makes the unit claimer withhold one unit, so the
roles of that CTA wait for a unit that never comes, with a 5 ms limit set for
the call. The call must return, report the timeout, leave every other unit's
output intact, and, after fvattn_workspace_init, the same engine must give
the reference output again. No GPU fault, trap or hang is involved: the
wait that runs out is bounded by design.
"""
import time

import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu

CASES = [
    gen.custom("fail_256tok", 1, 3, 128, (9, 20, 28), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=91),
    # near-dense 64-token heads: split units among the units in flight
    gen.custom("fail_64tok_split", 1, 3, 128, (16, 16, 16), (4, 4, 4), 0.95, 4, sigma=2.0,
               a_fixed=(0.25, 0.25, 6.0), seed=92),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("rank", [0, 5])
def test_withheld_unit_times_out_and_the_workspace_recovers(wl, rank):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    q, k, v = fvtest.make_on_gpu(wl)
    eng = fa.FVAttn(fvtest.geometry(wl), wl.p, wl.k_min, num_ctas=8)
    ref = eng(q, k, v).clone()
    torch.cuda.synchronize()
    assert eng.status() == 0

    fa.set_wait_limit(eng.ws, 5_000_000)        # 5 ms
    fa.test_withhold_unit(eng.ws, rank)
    out = torch.zeros_like(q)
    t0 = time.time()
    eng(q, k, v, out)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert elapsed < 10.0, elapsed                # the call returned
    flags = eng.status()
    assert flags & fa.FLAG_TIMEOUT, flags
    # only the withheld unit's rows (at most one unit: 256 query rows) are missing
    differ = (out.view(-1, wl.D) != ref.view(-1, wl.D)).any(dim=-1)
    assert 0 < int(differ.sum()) <= 256

    fa.workspace_init(eng.ws)                    # clears counters, the limit and the test word
    out2 = eng(q, k, v)
    torch.cuda.synchronize()
    assert eng.status() == 0
    assert torch.equal(out2, ref)
