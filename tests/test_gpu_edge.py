"""Edge cases and special cases of the CUDA path (needs a B200)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu


def _engine(wl, **kw):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    return fa.FVAttn(fvtest.geometry(wl), wl.p, wl.k_min, **kw)


def test_floor_equal_to_num_blocks_is_dense():
    # VSA accepts topk == num_blocks (zskr.cn guide, section 3): every block is kept,
    # and the sparse kernel then reproduces dense mode exactly (same tiles, same order)
    wl0 = gen.custom("kmin_nb", 1, 2, 128, (9, 20, 28), (4, 8, 8), 0.5, 1, sigma=2.0, a_range=(0.5, 4.0), seed=31)
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    nb = fa.num_blocks(fvtest.geometry(wl0))
    wl = gen.custom("kmin_nb", 1, 2, 128, (9, 20, 28), (4, 8, 8), 0.5, nb, sigma=2.0, a_range=(0.5, 4.0), seed=31)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    out = eng(q, k, v)
    assert (eng.kv_cnt == nb).all()
    assert (eng.kv_idx == torch.arange(nb, device="cuda", dtype=torch.int32)).all()
    dense = torch.empty_like(q)
    eng.dense(q, k, v, dense)
    torch.cuda.synchronize()
    assert torch.equal(out, dense)


def test_p_one_keeps_every_block():
    wl = gen.custom("p1", 1, 2, 64, (8, 16, 24), (4, 8, 8), 1.0, 1, sigma=2.0, a_range=(2.0, 4.0), seed=32)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    eng.route(q, k)
    torch.cuda.synchronize()
    assert (eng.kv_cnt == eng.nb).all()


def test_tiny_p_is_top1_plus_diagonal():
    wl = gen.custom("p_tiny", 1, 2, 128, (12, 24, 24), (4, 8, 8), 1e-6, 1, sigma=2.0, a_range=(0.5, 4.0), seed=33)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    eng.route(q, k)
    torch.cuda.synchronize()
    cnt = eng.kv_cnt.cpu().numpy()
    assert ((cnt == 1) | (cnt == 2)).all()


def test_grid_smaller_than_one_block():
    # Sol-Attn's "seq_len < block_size" case (bjdmk.com.cn, section 6.1): one partial block
    import oracle
    wl = gen.custom("sub_block", 1, 3, 128, (2, 3, 5), (4, 8, 8), 0.9, 1, sigma=1.0, a_range=(0.5, 4.0), seed=34)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    out = eng(q, k, v)
    torch.cuda.synchronize()
    assert eng.nb == 1 and (eng.kv_cnt == 1).all()
    orc = oracle.get()
    g = orc.geom(1, 3, wl.grid, wl.block, 128)
    rows = np.arange(3 * wl.N)
    ref, _ = orc.attn_rows(g, q.cpu(), k.cpu(), v.cpu(), 1 / math.sqrt(128), rows)
    mx, mean = fvtest.attn_errors(out, rows, ref, 128)
    assert mx <= fvtest.ATTN_MAX_ABS and mean <= fvtest.ATTN_MEAN_ABS


def test_nonfinite_scores_are_repaired_and_flagged():
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.custom("nonfinite", 1, 2, 128, (8, 16, 16), (4, 8, 8), 0.5, 1, sigma=2.0, a_range=(1.0, 4.0), seed=35)
    q, k, v = fvtest.make_on_gpu(wl)
    q[0, 1, 5] = float("inf")          # token 5 lies in block 0 of head 1
    eng = _engine(wl)
    eng.route(q, k)
    flags = eng.status()
    assert flags & fa.FLAG_NONFINITE
    assert int(eng.kv_cnt[0, 1, 0]) == eng.nb
    assert eng.status() == 0           # reading clears the flag


def test_empty_batch_is_a_no_op():
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    geo = fa.Geometry(0, 4, 128, (8, 16, 16), (4, 8, 8))
    ws = torch.zeros(max(fa.workspace_size(geo), 256), dtype=torch.uint8, device="cuda")
    fa.workspace_init(ws)
    e = torch.empty((0, 4, 2048, 128), dtype=torch.bfloat16, device="cuda")
    cnt = torch.empty((0,), dtype=torch.int32, device="cuda")
    # zero-element tensors have no storage; pass any aligned allocation
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ibuf = torch.zeros(16, dtype=torch.int32, device="cuda")
    fa.route(geo, buf, buf, 0.9, 1, ibuf, ibuf, ws)
    work = torch.zeros(4, dtype=torch.int32, device="cuda")
    rng = torch.zeros(9, dtype=torch.int32, device="cuda")
    fa.schedule(geo, ibuf, ibuf, False, 8, work, rng, ws)
    fa.sparse_attn(geo, buf, buf, buf, ibuf, ibuf, work, rng, 8, False, buf, ws)
    torch.cuda.synchronize()
    assert (rng == 0).all()
    del e, cnt


@pytest.mark.parametrize("num_ctas", [1, 7, 148, 300])
def test_output_independent_of_cta_count(num_ctas):
    wl = gen.custom("ctas", 1, 3, 128, (9, 20, 28), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=36)
    q, k, v = fvtest.make_on_gpu(wl)
    ref = _engine(wl, num_ctas=148)(q, k, v)
    out = _engine(wl, num_ctas=num_ctas)(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("num_ctas", [1, 5, 148])
def test_paired_output_independent_of_cta_count_and_schedule(num_ctas):
    # 64-token blocks run as paired units; the result must not depend on the
    # CTA count, nor on whether work lists come from fvattn_schedule or the
    # call builds the pair unions itself (units in index order)
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.custom("paired_ctas", 1, 3, 128, (8, 12, 20), (4, 4, 4), 0.9, 3, sigma=2.0, a_range=(0.5, 4.0),
                    seed=38)
    q, k, v = fvtest.make_on_gpu(wl)
    ref = _engine(wl, num_ctas=148)(q, k, v).clone()
    eng = _engine(wl, num_ctas=num_ctas)
    out = eng(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # no work lists: a fresh workspace, so the pair unions must come from this call
    ws = torch.zeros_like(eng.ws)
    fa.workspace_init(ws)
    out2 = torch.zeros_like(q)
    fa.sparse_attn(eng.geo, q, k, v, eng.kv_cnt, eng.kv_idx, None, None, num_ctas, False, out2, ws)
    torch.cuda.synchronize()
    assert fa.read_device_status(ws) == 0
    assert torch.equal(out2, ref)


@pytest.mark.parametrize("num_ctas", [1, 5, 148])
def test_split_units_independent_of_cta_count(num_ctas):
    # near-dense 64-token heads run split units; the result must not depend on
    # which CTA runs which unit
    wl = gen.custom("split_ctas", 1, 3, 128, (16, 16, 16), (4, 4, 4), 0.95, 4, sigma=2.0,
                    a_fixed=(0.25, 0.25, 6.0), seed=45)
    q, k, v = fvtest.make_on_gpu(wl)
    ref = _engine(wl, num_ctas=148)
    o_ref = ref(q, k, v).clone()
    eng = _engine(wl, num_ctas=num_ctas)
    out = eng(q, k, v)
    torch.cuda.synchronize()
    assert eng.status() == 0
    U = int(eng.cta_range[num_ctas].item())
    assert U > 3 * 16, "no unit ran split"
    assert torch.equal(out, o_ref)


@pytest.mark.parametrize("groups", [1, 3, 4])
def test_host_pipeline_matches_device_path(groups):
    # host-resident tensors, copies overlapped with compute per group of heads:
    # every head is routed and attended alone, so the result is bit-identical
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.custom("host", 2, 3, 128, (9, 20, 28), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=39)
    q, k, v = fvtest.make_on_gpu(wl)
    ref = _engine(wl)(q, k, v).clone()
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.zeros(q.shape, dtype=q.dtype).pin_memory()
    pipe = fa.HostPipeline(fvtest.geometry(wl), wl.p, wl.k_min, groups=groups)
    for _ in range(2):  # a second call reuses the device buffers
        pipe(hq, hk, hv, hout)
    torch.cuda.synchronize()
    assert pipe.status() == 0
    assert torch.equal(hout, ref.cpu())


@pytest.mark.parametrize("groups", [2, 4])
def test_host_pipeline_overlapped_calls(groups):
    # overlap_calls: a call's copy of head group c waits only for the previous
    # call's compute of group c. Three different inputs in a row, no
    # synchronisation between the calls: each result is bit-identical to the
    # device path on its own inputs
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.custom("host_overlap", 1, 8, 128, (12, 24, 40), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0),
                    seed=41)
    eng = _engine(wl)
    ins, refs = [], []
    for seed in (41, 42, 43):
        q, k, v = fvtest.make_on_gpu(wl, seed=seed)
        refs.append(eng(q, k, v).clone().cpu())
        ins.append(tuple(t.cpu().pin_memory() for t in (q, k, v)))
    torch.cuda.synchronize()
    outs = [torch.zeros(ins[0][0].shape, dtype=ins[0][0].dtype).pin_memory() for _ in ins]
    pipe = fa.HostPipeline(fvtest.geometry(wl), wl.p, wl.k_min, groups=groups, overlap_calls=True)
    for (hq, hk, hv), hout in zip(ins, outs):
        pipe(hq, hk, hv, hout)
    torch.cuda.synchronize()
    assert pipe.status() == 0
    assert not torch.equal(refs[0], refs[1])
    for hout, ref in zip(outs, refs):
        assert torch.equal(hout, ref)


@pytest.mark.parametrize("block", [(4, 8, 8), (4, 4, 4)])
def test_cuda_graph_replay_matches_eager(block):
    wl = gen.custom("graph", 1, 3, 128, (9, 20, 28), block, 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=40)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    ref = eng(q, k, v).clone()
    out = torch.zeros_like(q)
    graph = eng.capture(q, k, v, out)
    out.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert eng.status() == 0
    assert torch.equal(out, ref)


def test_repeatable():
    wl = gen.WORKLOADS["wan5b"]
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    o1 = eng(q, k, v).clone()
    c1, i1 = eng.kv_cnt.clone(), eng.kv_idx.clone()
    o2 = eng(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(c1, eng.kv_cnt)
    assert torch.equal(o1, o2)
    mask = torch.arange(eng.nb, device="cuda")[None, None, None, :] < c1[..., None]
    assert torch.equal(torch.where(mask, i1, 0), torch.where(mask, eng.kv_idx, 0))


def _palette_inputs(grid, block, H, D, n_q, n_k, amp, seed):
    """Every token of a block is the same vector, drawn from a small palette
    per head, so block means -- and with them block scores -- tie exactly, in
    fp32 as in fp64 (the grid is a multiple of the block)."""
    T, Hg, W = grid
    bt, bh, bw = block
    nbh, nbw = Hg // bh, W // bw
    g = torch.Generator().manual_seed(seed)
    nb = (T // bt) * nbh * nbw
    pal_q = (torch.randn(H, n_q, D, generator=g) * amp).to(torch.bfloat16)
    pal_k = (torch.randn(H, n_k, D, generator=g) * amp).to(torch.bfloat16)
    c_q = torch.randint(n_q, (H, nb), generator=g)
    c_k = torch.randint(n_k, (H, nb), generator=g)
    t, y, x = torch.arange(T) // bt, torch.arange(Hg) // bh, torch.arange(W) // bw
    blk = ((t[:, None, None] * nbh + y[None, :, None]) * nbw + x[None, None, :]).reshape(-1)
    q = torch.stack([pal_q[h][c_q[h][blk]] for h in range(H)])[None]
    k = torch.stack([pal_k[h][c_k[h][blk]] for h in range(H)])[None]
    v = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("grid,n_k,k_min", [((16, 64, 64), 4, 5), ((16, 64, 64), 40, 24), ((24, 64, 64), 4, 5),
                                            ((24, 64, 64), 40, 24)])
def test_exact_score_ties_follow_block_order(grid, n_k, k_min):
    # Blocks whose scores tie exactly are ranked by block index (lower first),
    # at the Top-p boundary and at the Top-k floor alike; 256 blocks take the
    # warp-sort selection, 384 the key-space search
    import oracle
    block, H, D, p = (4, 8, 8), 2, 128, 0.6
    q, k, v = _palette_inputs(grid, block, H, D, 24, n_k, 1.5, seed=37 + n_k)
    wl = gen.custom("ties", 1, H, D, grid, block, p, k_min, seed=0)
    eng = _engine(wl)
    eng.route(q.cuda(), k.cuda())
    torch.cuda.synchronize()
    assert eng.status() == 0
    orc = oracle.get()
    g = orc.geom(1, H, grid, block, D)
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    scale = 1.0 / math.sqrt(D)
    r = orc.route(g, qb, kb, scale, p, k_min)
    bound = fvtest.score_bound(orc, g, q, k, qb, kb, scale, tc=eng.nb >= fvtest.TC_SCORES_MIN_BLOCKS)
    cmp = fvtest.compare_lists(eng.kv_cnt.cpu().numpy(), eng.kv_idx.cpu().numpy(), r, bound, p, k_min)
    assert cmp.invalid == 0, cmp.first_invalid
    assert cmp.unexcused == 0, cmp.first_unexcused
    assert cmp.excused_tie == 0, cmp.summary()
    # the case is meaningful: many rows have an exact tie across their boundary
    nb = eng.nb
    s = scale * np.einsum("bhid,bhjd->bhij", qb, kb)
    order, cnt = r["order"], r["kv_cnt"]
    tied = 0
    for h in range(H):
        for i in range(nb):
            m = int(cnt[0, h, i])
            o = order[0, h, i]
            if 0 < m < nb and s[0, h, i, o[m - 1]] == s[0, h, i, o[min(m, nb - 1)]]:
                tied += 1
    assert tied >= nb // 4, tied


def test_grouped_routing_equals_routing_the_groups_alone():
    # a layer this large routes in head groups (selection on a side stream
    # under the pooling of the next group); every head's lists must be the
    # ones it gets when its half of the heads is routed as a problem of its
    # own (small enough to route in one piece), and a CUDA-graph replay of
    # the grouped route must give the same lists again
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    wl = gen.custom("grouped", 1, 12, 128, (16, 64, 64), (4, 8, 8), 0.85, 8, sigma=2.0, a_range=(0.5, 4.0),
                    seed=42)
    q, k, v = fvtest.make_on_gpu(wl)
    eng = _engine(wl)
    eng.route(q, k)
    torch.cuda.synchronize()
    assert eng.status() == 0
    cnt, idx = eng.kv_cnt.clone(), eng.kv_idx.clone()
    nb = eng.nb
    for h0, h1 in ((0, 6), (6, 12)):
        geo = fa.Geometry(1, h1 - h0, wl.D, wl.grid, wl.block)
        e2 = fa.FVAttn(geo, wl.p, wl.k_min)
        e2.route(q[:, h0:h1].contiguous(), k[:, h0:h1].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(e2.kv_cnt[0], cnt[0, h0:h1])
        mask = torch.arange(nb, device="cuda")[None, None, :] < e2.kv_cnt[0][..., None]
        assert torch.equal(torch.where(mask, e2.kv_idx[0], 0), torch.where(mask, idx[0, h0:h1], 0))
    out = torch.zeros_like(q)
    graph = eng.capture(q, k, v, out)
    eng.kv_cnt.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(eng.kv_cnt, cnt)
    ref = _engine(wl)(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
