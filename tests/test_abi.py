"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments synchronously (before anything is enqueued). CPU only: every call
here fails validation, so nothing reaches the GPU."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fvattn.h")


@pytest.fixture(scope="module")
def fa():
    from block_sparse_attention_fvattn_b200 import build
    build.build()
    from block_sparse_attention_fvattn_b200 import fvattn
    return fvattn


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fvattn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("fvattn_route", "fvattn_schedule", "fvattn_sparse_attn"):
        assert n in names


def test_every_declared_symbol_is_exported(fa):
    lib = ctypes.CDLL(fa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(fa.EXPORTED) | set(declared_functions())


def test_128_token_blocks_accepted(fa):
    # (2,8,8): one 128-row query tile per block
    g = fa.Geometry(1, 2, 128, (7, 20, 28), (2, 8, 8))
    assert fa.num_blocks(g) == 4 * 3 * 4
    assert fa.workspace_size(g) > 0


def test_num_blocks_worked_example(fa):
    # zskr.cn VSA guide, section 3: (31,22,40) with (4,8,8) -> 8*3*5 = 120 blocks
    g = fa.Geometry(1, 24, 128, (31, 22, 40), (4, 8, 8))
    assert fa.num_blocks(g) == 120
    assert fa.num_blocks(fa.Geometry(1, 12, 128, (96, 64, 64), (4, 8, 8))) == 1536
    assert fa.num_blocks(fa.Geometry(1, 16, 128, (16, 32, 32), (4, 4, 4))) == 1024 // 4 * 1
    assert fa.workspace_size(g) > 0


@pytest.mark.parametrize("geo_args,expect", [
    (dict(B=1, H=1, D=96, grid=(8, 16, 16), block=(4, 8, 8)), "UNSUPPORTED"),      # head dim
    (dict(B=1, H=1, D=128, grid=(8, 16, 16), block=(3, 8, 8)), "UNSUPPORTED"),     # 192-token blocks
    (dict(B=1, H=1, D=128, grid=(8, 16, 16), block=(2, 4, 4)), "UNSUPPORTED"),     # 32-token blocks
    (dict(B=1, H=1, D=128, grid=(8, 16, 16), block=(1, 16, 16)), "UNSUPPORTED"),   # odd blk_t, 256 tokens
    (dict(B=1, H=1, D=128, grid=(0, 16, 16), block=(4, 8, 8)), "INVALID_ARG"),     # empty grid axis
    (dict(B=1, H=1, D=128, grid=(8, 16, 16), block=(0, 8, 8)), "INVALID_ARG"),
    (dict(B=1, H=1, D=128, grid=(400, 64, 64), block=(4, 8, 8)), "UNSUPPORTED"),   # nb > 2048
])
def test_problem_validation(fa, geo_args, expect):
    g = fa.Geometry(**geo_args)
    p = g.problem()
    assert fa._lib.fvattn_num_blocks(ctypes.byref(p)) == -1
    st = fa._lib.fvattn_route(ctypes.byref(p), ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), 0.9, 1,
                              ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), None, ctypes.c_void_p(0x1000),
                              1 << 30, None)
    assert st == getattr(fa, expect)


def test_element_type(fa):
    # bf16 and fp16 are accepted; any other element type code is UNSUPPORTED
    for code, ok in ((fa.DTYPE_BF16, True), (fa.DTYPE_F16, True), (2, False), (-1, False)):
        p = fa.Geometry(1, 1, 128, (8, 16, 16), (4, 8, 8)).problem()
        p.dtype = code
        assert (fa._lib.fvattn_num_blocks(ctypes.byref(p)) == 8) == ok, code
    assert fa.Geometry(1, 1, 128, (8, 16, 16), (4, 8, 8), dtype=torch.float16).problem().dtype == fa.DTYPE_F16
    with pytest.raises(ValueError):
        fa.Geometry(1, 1, 128, (8, 16, 16), (4, 8, 8), dtype=torch.float32).problem()


def test_grid_product_must_equal_n(fa):
    g = fa.Geometry(1, 1, 128, (8, 16, 16), (4, 8, 8))
    p = g.problem()
    p.N = 2047
    assert fa._lib.fvattn_num_blocks(ctypes.byref(p)) == -1


def _route_status(fa, g, p=0.9, k_min=1, q=0x1000, k=0x1000, cnt=0x1000, idx=0x1000, ws=0x1000, ws_bytes=1 << 30):
    prob = g.problem()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return fa._lib.fvattn_route(ctypes.byref(prob), vp(q), vp(k), float(p), int(k_min), vp(cnt), vp(idx), None,
                                vp(ws), ws_bytes, None)


def test_route_argument_errors(fa):
    g = fa.Geometry(1, 2, 64, (8, 16, 16), (4, 8, 8))   # nb = 8
    assert _route_status(fa, g, k_min=9) == fa.INVALID_ARG        # floor above num_blocks
    assert _route_status(fa, g, k_min=0) == fa.INVALID_ARG
    assert _route_status(fa, g, p=0.0) == fa.INVALID_ARG
    assert _route_status(fa, g, p=1.5) == fa.INVALID_ARG
    assert _route_status(fa, g, p=float("nan")) == fa.INVALID_ARG
    assert _route_status(fa, g, q=None) == fa.INVALID_ARG
    assert _route_status(fa, g, q=0x1008) == fa.INVALID_ARG        # not 16-byte aligned
    assert _route_status(fa, g, cnt=None) == fa.INVALID_ARG
    assert _route_status(fa, g, ws=None) == fa.WORKSPACE
    assert _route_status(fa, g, ws_bytes=16) == fa.WORKSPACE


def test_schedule_and_attn_argument_errors(fa):
    g = fa.Geometry(1, 2, 64, (8, 16, 16), (4, 8, 8))
    prob = g.problem()
    vp = ctypes.c_void_p
    # sparse schedule needs lists; negative CTA count
    assert fa._lib.fvattn_schedule(ctypes.byref(prob), None, None, 0, 4, vp(0x1000), vp(0x1000), None,
                                   vp(0x1000), 1 << 30, None) == fa.INVALID_ARG
    assert fa._lib.fvattn_schedule(ctypes.byref(prob), vp(0x1000), vp(0x1000), 0, -1, vp(0x1000), vp(0x1000),
                                   None, vp(0x1000), 1 << 30, None) == fa.INVALID_ARG
    # attention: work without cta_range, missing output
    assert fa._lib.fvattn_sparse_attn(ctypes.byref(prob), vp(0x1000), vp(0x1000), vp(0x1000), vp(0x1000),
                                      vp(0x1000), vp(0x1000), None, 4, 0, vp(0x1000), None, vp(0x1000), 1 << 30,
                                      None) == fa.INVALID_ARG
    assert fa._lib.fvattn_sparse_attn(ctypes.byref(prob), vp(0x1000), vp(0x1000), vp(0x1000), None, None, None,
                                      None, 4, 0, vp(0x1000), None, vp(0x1000), 1 << 30, None) == fa.INVALID_ARG
    assert fa._lib.fvattn_sparse_attn(ctypes.byref(prob), vp(0x1000), vp(0x1000), vp(0x1000), None, None, None,
                                      None, 4, 1, None, None, vp(0x1000), 1 << 30, None) == fa.INVALID_ARG


def test_status_strings(fa):
    for s in range(7):
        assert fa.status_string(s) and fa.status_string(s) != "unknown status"
    assert fa.status_string(99) == "unknown status"
