"""fvattn_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they route (a runtime that hands a
plug-in only its input and output tensors, code under a fixed memory-pool
reservation, a process whose device footprint is fixed at start-up). The
no-allocation entry point keeps its scratch in a fixed array inside the
library instead of a caller workspace. These checks call it through the C ABI
and compare its lists and block probabilities with fvattn_route's on the same
inputs, on consecutive calls that reuse the array (with a different problem in
between), and check that a problem too large for the array is refused before
anything runs. This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu


def _reference(fa, wl, q, k):
    geo = fvtest.geometry(wl)
    nb = fa.num_blocks(geo)
    ws = torch.zeros(fa.workspace_size(geo), dtype=torch.uint8, device="cuda")
    fa.workspace_init(ws)
    cnt = torch.zeros((wl.B, wl.H, nb), dtype=torch.int32, device="cuda")
    idx = torch.zeros((wl.B, wl.H, nb, nb), dtype=torch.int32, device="cuda")
    probs = torch.zeros((wl.B, wl.H, nb, nb), dtype=torch.float32, device="cuda")
    fa.route(geo, q, k, wl.p, wl.k_min, cnt, idx, ws, probs)
    return cnt, idx, probs


def _noalloc(fa, wl, q, k):
    geo = fvtest.geometry(wl)
    nb = fa.num_blocks(geo)
    cnt = torch.full((wl.B, wl.H, nb), -1, dtype=torch.int32, device="cuda")
    idx = torch.full((wl.B, wl.H, nb, nb), -1, dtype=torch.int32, device="cuda")
    probs = torch.full((wl.B, wl.H, nb, nb), -1.0, dtype=torch.float32, device="cuda")
    fa.route_noalloc(geo, q, k, wl.p, wl.k_min, cnt, idx, probs)
    return cnt, idx, probs


def _same(ref, got):
    rc, ri, rp = (t.cpu().numpy() for t in ref)
    gc, gi, gp = (t.cpu().numpy() for t in got)
    assert np.array_equal(rc, gc)
    nb = rc.shape[-1]
    valid = np.arange(nb)[None, None, None, :] < rc[..., None]
    assert np.array_equal(np.where(valid, ri, 0), np.where(valid, gi, 0))
    np.testing.assert_allclose(gp, rp, rtol=2e-3, atol=1e-6)


def test_noalloc_matches_route_on_consecutive_calls():
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl_a = gen.WORKLOADS["wan5b"]
    wl_b = gen.custom("noalloc_b", 2, 3, 64, (9, 20, 28), (4, 8, 8), 0.8, 3, sigma=2.0, a_range=(0.5, 4.0), seed=41)
    qa, ka, _ = fvtest.make_on_gpu(wl_a)
    qb, kb, _ = fvtest.make_on_gpu(wl_b)
    ref_a = _reference(fa, wl_a, qa, ka)
    ref_b = _reference(fa, wl_b, qb, kb)
    got1 = _noalloc(fa, wl_a, qa, ka)
    got2 = _noalloc(fa, wl_a, qa, ka)
    got3 = _noalloc(fa, wl_b, qb, kb)
    got4 = _noalloc(fa, wl_a, qa, ka)
    torch.cuda.synchronize()
    _same(ref_a, got1)
    _same(ref_a, got2)
    _same(ref_b, got3)
    _same(ref_a, got4)


def test_noalloc_long_rows_match_the_oracle():
    # from 320 blocks on, fvattn_route scores on the tensor cores while the
    # no-allocation path keeps fp32 CUDA-core scores; its lists are held to
    # the parity rule against the oracle instead of bit-equality with
    # fvattn_route, on two calls in a row
    import math

    import oracle
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.WORKLOADS["wan14b_i2v_720p"]      # 40 heads x 360 blocks
    q, k, _ = fvtest.make_on_gpu(wl)
    got1 = _noalloc(fa, wl, q, k)
    got2 = _noalloc(fa, wl, q, k)
    torch.cuda.synchronize()
    _same(got1, got2)
    orc = oracle.get()
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    qh, kh = q.cpu(), k.cpu()
    qb, kb = orc.pool(g, qh), orc.pool(g, kh)
    scale = 1.0 / math.sqrt(wl.D)
    r = orc.route(g, qb, kb, scale, wl.p, wl.k_min)
    bound = fvtest.score_bound(orc, g, qh, kh, qb, kb, scale, tc=False)
    cmp = fvtest.compare_lists(got1[0].cpu().numpy(), got1[1].cpu().numpy(), r, bound, wl.p, wl.k_min)
    assert cmp.invalid == 0 and cmp.unexcused == 0, (cmp.summary(), cmp.first_invalid, cmp.first_unexcused)
    assert cmp.excused_topp + cmp.excused_tie <= max(2, fvtest.EXCUSED_MAX_SHARE * cmp.rows), cmp.summary()
    np.testing.assert_allclose(got1[2].cpu().numpy(), r["probs"], rtol=2e-3, atol=1e-6)


def test_noalloc_refuses_problems_beyond_its_array():
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.WORKLOADS["long_393k"]          # pooled means need ~18.9 MB > 16 MiB
    geo = fvtest.geometry(wl)
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ibuf = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(fa.FVAttnError) as e:
        fa.route_noalloc(geo, buf, buf, wl.p, wl.k_min, ibuf, ibuf)
    assert e.value.status == fa.WORKSPACE
