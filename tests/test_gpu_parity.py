"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Per workload: routing lists (bit-exact except the stated boundary excuses)
and block probabilities, the schedule (exact, recomputed on the host), and
attention on the GPU's own lists against the oracle -- every query row for
the small ragged cases, sampled rows (edges, heaviest and lightest units,
random) for the five full-size workloads, in the launch configuration the
benchmark uses (one persistent CTA per SM, scheduled work lists).
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu

SMALL = [
    gen.custom("ragged_256tok", 1, 3, 128, (9, 20, 28), (4, 8, 8), 0.9, 4, sigma=2.0, a_range=(0.5, 4.0), seed=21),
    gen.custom("last_frame_only", 1, 2, 128, (5, 11, 13), (4, 8, 8), 0.8, 2, sigma=1.5, a_range=(0.5, 4.0),
               seed=22),
    gen.custom("d64_b2", 2, 2, 64, (8, 16, 24), (4, 8, 8), 0.9, 2, sigma=2.0, a_range=(0.5, 3.0), seed=23),
    gen.custom("blk64", 1, 4, 128, (8, 12, 20), (4, 4, 4), 0.95, 4, sigma=2.0, a_range=(0.25, 6.0), seed=24),
    gen.custom("blk64_ragged_d64", 1, 2, 64, (6, 10, 9), (4, 4, 4), 0.9, 3, sigma=1.5, a_range=(0.5, 4.0),
               seed=25),
    gen.custom("iid_tiny", 1, 2, 64, (8, 16, 16), (4, 8, 8), 0.9, 2, seed=26),
    # 15 64-token blocks: the last pair holds one query block, the last unit one and a half pairs
    gen.custom("blk64_odd_pairs", 2, 2, 128, (4, 12, 20), (4, 4, 4), 0.8, 2, sigma=1.5, a_range=(0.5, 4.0),
               seed=27),
    # 128-token (2,8,8) blocks, ragged along every axis: one 128-row query tile per unit
    gen.custom("blk128_ragged", 1, 3, 128, (7, 20, 28), (2, 8, 8), 0.9, 3, sigma=2.0, a_range=(0.5, 4.0), seed=28),
    gen.custom("blk128_d64", 2, 2, 64, (8, 16, 24), (2, 8, 8), 0.85, 2, sigma=1.5, a_range=(0.5, 3.0), seed=29),
    # near-dense 64-token heads: units of >= 64 tiles run split (one pair on both
    # softmax warpgroups, combined at the end); the third head stays sparse
    gen.custom("blk64_split", 1, 3, 128, (16, 16, 16), (4, 4, 4), 0.95, 4, sigma=2.0, a_fixed=(0.25, 0.25, 6.0),
               seed=30),
    # split units with ragged edge blocks, D = 64, an even and an odd pair count per unit row
    gen.custom("blk64_split_ragged_d64", 1, 2, 64, (13, 16, 18), (4, 4, 4), 0.95, 3, sigma=2.0,
               a_fixed=(0.25, 0.3), seed=31),
]
FULL = [gen.WORKLOADS[n] for n in gen.WORKLOAD_ORDER]


def _oracle_route(orc, wl, q, k, scale):
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D, fp16=q.dtype == torch.float16)
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    r = orc.route(g, qb, kb, scale, wl.p, wl.k_min)
    return g, qb, kb, r


# A paired unit of at least this many key/value tiles runs as one split unit
# per pair (the scheduler's threshold).
SPLIT_MIN_TILES = 64


def _host_units(wl, nb, kv_cnt, kv_idx):
    """Every head's units as the scheduler defines them, recomputed on the
    host: (list per head of (unit id, cost), where the cost is the active
    128-row query tiles x kept key/value sub-tiles). With 64-token blocks a
    unit is query blocks 4q..4q+3: pairs (4q, 4q+1) and (4q+2, 4q+3), each one
    128-row tile over the union of its two lists, two blocks per step; a unit
    of at least SPLIT_MIN_TILES steps becomes one split unit per pair, with
    id B*H*upb + bh*npair + pair."""
    T, Hg, W = wl.grid
    bt, bh, bw = wl.block
    nbh, nbw = -(-Hg // bh), -(-W // bw)
    BH = wl.B * wl.H
    cnt = kv_cnt.reshape(BH, nb)
    idx = kv_idx.reshape(BH, nb, nb)
    heads = []
    if bt * bh * bw == 64:
        upb, npair = -(-nb // 4), -(-nb // 2)

        def tiles(h, pp):
            if pp >= npair:
                return 0
            kept = set(idx[h, 2 * pp, :cnt[h, 2 * pp]].tolist())
            if 2 * pp + 1 < nb:
                kept |= set(idx[h, 2 * pp + 1, :cnt[h, 2 * pp + 1]].tolist())
            return (len(kept) + 1) // 2
        for h in range(BH):
            units = []
            for q in range(upb):
                t0, t1 = tiles(h, 2 * q), tiles(h, 2 * q + 1)
                if t0 + t1 >= SPLIT_MIN_TILES:
                    for half, tc in ((0, t0), (1, t1)):
                        if 2 * q + half < npair:
                            units.append((BH * upb + h * npair + 2 * q + half, tc))
                else:
                    units.append((h * upb + q, t0 + t1))
            heads.append(units)
        return heads
    two = bt * bh * bw == 256
    subt = bt // 2 if two else bt

    def nsub(j):
        jt = j // (nbh * nbw)
        return 1 + (1 if two and jt * bt + subt < T else 0)

    ns = np.array([nsub(j) for j in range(nb)])
    nh = np.array([1 + (1 if two and (i // (nbh * nbw)) * bt + subt < T else 0) for i in range(nb)])
    for h in range(BH):
        heads.append([(h * nb + i, int(nh[i] * ns[idx[h, i, :cnt[h, i]]].sum())) for i in range(nb)])
    return heads


def _expected_work(heads, C):
    """Heads by total cost descending (ties: lower head), each head's units by
    cost descending (ties: lower id), ranks dealt to the CTAs in zigzag rounds."""
    order = sorted(range(len(heads)), key=lambda h: (-sum(c for _, c in heads[h]), h))
    ranked = []
    for h in order:
        ranked += [u for u, _ in sorted(heads[h], key=lambda x: (-x[1], x[0]))]
    lists = [[] for _ in range(C)]
    for r, u in enumerate(ranked):
        rd, pos = divmod(r, C)
        lists[C - 1 - pos if rd % 2 else pos].append(u)
    return lists


def _run(wl, full_rows, dtype=torch.bfloat16, softmax_scale=0.0, tag="", out_rel=0.0):
    import oracle
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    orc = oracle.get()
    q, k, v = fvtest.make_on_gpu(wl, dtype=dtype)
    geo = fvtest.geometry(wl, dtype, softmax_scale)
    assert geo.scale == (softmax_scale if softmax_scale > 0 else 1.0 / math.sqrt(wl.D))
    eng = fa.FVAttn(geo, wl.p, wl.k_min, with_probs=True)
    eng.route(q, k)
    eng.schedule()
    out = torch.zeros_like(q)
    eng.attend(q, k, v, out, timing=True)
    out_dense = torch.zeros_like(q)
    eng.dense(q, k, v, out_dense)
    torch.cuda.synchronize()
    assert eng.status() == 0
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    g, qb, kb, r = _oracle_route(orc, wl, qh, kh, geo.scale)
    nb = eng.nb
    cnt = eng.kv_cnt.cpu().numpy()
    idx = eng.kv_idx.cpu().numpy()

    # ---- routing: every GPU row valid, differences only under the excuses
    bound = fvtest.score_bound(orc, g, qh, kh, qb, kb, geo.scale, tc=nb >= fvtest.TC_SCORES_MIN_BLOCKS)
    cmp = fvtest.compare_lists(cnt, idx, r, bound, wl.p, wl.k_min)
    fvtest.record(f"{wl.name}" + ("" if dtype == torch.bfloat16 else " fp16") + tag, cmp)
    assert cmp.invalid == 0, (cmp.summary(), cmp.first_invalid)
    assert cmp.unexcused == 0, (cmp.summary(), cmp.first_unexcused)
    assert cmp.excused_topp + cmp.excused_tie <= max(2, fvtest.EXCUSED_MAX_SHARE * cmp.rows), cmp.summary()
    probs = eng.block_probs.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(probs, r["probs"], rtol=2e-3, atol=1e-6)

    # ---- schedule
    C = eng.num_ctas
    work = eng.work.cpu().numpy()
    rng = eng.cta_range.cpu().numpy()
    heads = _host_units(wl, nb, cnt, idx)
    cost = {u: c for units in heads for u, c in units}
    U = len(cost)
    assert rng[0] == 0 and rng[C] == U and (np.diff(rng) >= 0).all()
    assert sorted(work[:U].tolist()) == sorted(cost)
    expect = _expected_work(heads, C)
    for c in range(C):
        assert work[rng[c]:rng[c + 1]].tolist() == expect[c], c
    cta_cost = eng.cta_cost.cpu().numpy()
    assert all(cta_cost[c] == sum(cost[u] for u in work[rng[c]:rng[c + 1]]) for c in range(C))
    ns = eng.cta_ns.cpu().numpy()
    assert (ns[np.diff(rng) > 0] > 0).all()

    # ---- attention on the GPU's own lists, and dense mode
    rows = np.arange(wl.B * wl.H * wl.N) if full_rows else fvtest.sample_rows(wl, cnt)
    ref, wsum = orc.attn_rows(g, qh, kh, vh, geo.scale, rows, cnt, idx)
    assert np.abs(wsum - 1.0).max() < 1e-9
    mx, mean = fvtest.attn_errors(out, rows, ref, wl.D)
    lim = fvtest.attn_excess(out, rows, ref, wl.D, out_rel) if out_rel else mx
    assert lim <= fvtest.ATTN_MAX_ABS and mean <= fvtest.ATTN_MEAN_ABS, (mx, lim, mean)
    assert torch.isfinite(out).all()
    drows = rows if full_rows else rows[:: max(1, len(rows) // 48)]
    dref, _ = orc.attn_rows(g, qh, kh, vh, geo.scale, drows)
    dmx, dmean = fvtest.attn_errors(out_dense, drows, dref, wl.D)
    dlim = fvtest.attn_excess(out_dense, drows, dref, wl.D, out_rel) if out_rel else dmx
    assert dlim <= fvtest.ATTN_MAX_ABS and dmean <= fvtest.ATTN_MEAN_ABS, (dmx, dlim, dmean)
    return dict(cmp=cmp, max_abs=mx, mean_abs=mean, dense_max=dmx)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_every_row(wl):
    _run(wl, full_rows=True)


@pytest.mark.parametrize("name", ["ragged_256tok", "blk64", "blk64_ragged_d64", "blk128_ragged"])
def test_small_fp16_every_row(name):
    # fp16 Q, K, V: the same path with fp16 TMA tiles, fp16 MMAs and fp16 P and O
    _run([w for w in SMALL if w.name == name][0], full_rows=True, dtype=torch.float16)


@pytest.mark.parametrize("wl", FULL, ids=lambda w: w.name)
def test_full_size_sampled(wl):
    _run(wl, full_rows=False)


# A caller-chosen softmax scale (fvattn_problem.softmax_scale > 0) replaces
# 1/sqrt(D) in the block scores and in the attention alike: a sharper and a
# flatter scale on a 256-token, a paired 64-token and a 128-token layer, and
# on a layer of 320 blocks, whose routing scores run on the tensor cores.
# A sharp softmax makes an output row nearly one V row, whose entries reach
# |o| ~ 5 on these inputs; there bf16 values lie 2^-5 apart, so the rounding
# of the output alone is up to 2^-8 |o| (0.0156 at |o| = 4), beside the
# rounding of P to bf16 in the PV product. These cases allow each element its
# own output rounding, 2^-8 |o|, on top of the 2e-2 max-abs bound.
BF16_UNIT_ROUNDOFF = 2.0 ** -8
SCALED = [
    ("ragged_256tok", 0.3, True),
    ("blk64", 0.05, True),
    ("blk128_ragged", 0.2, True),
]


@pytest.mark.parametrize("name,scale,full", SCALED, ids=lambda x: str(x))
def test_custom_softmax_scale(name, scale, full):
    _run([w for w in SMALL if w.name == name][0], full_rows=full, softmax_scale=scale, tag=f" scale {scale}",
         out_rel=BF16_UNIT_ROUNDOFF)


def test_custom_softmax_scale_tensor_core_scores():
    wl = gen.custom("tc320_scaled", 1, 2, 64, (16, 64, 80), (4, 8, 8), 0.9, 8, sigma=2.0, a_range=(0.5, 4.0),
                    seed=32)
    assert math.prod(-(-g // b) for g, b in zip(wl.grid, wl.block)) >= fvtest.TC_SCORES_MIN_BLOCKS
    _run(wl, full_rows=False, softmax_scale=0.2, tag=" scale 0.2", out_rel=BF16_UNIT_ROUNDOFF)


# The largest block count the library accepts (nb = 2048): the longest routing
# rows (64 keys per lane, tensor-core scores) and the longest kept lists, on
# the 256-token route and on the paired 64-token route (a near-dense head,
# whose units run split, beside a floor-bound one).
MAX_NB = [
    gen.custom("max_blocks_256tok", 1, 1, 128, (64, 64, 128), (4, 8, 8), 0.9, 16, sigma=2.0, a_range=(0.5, 4.0),
               seed=33),
    gen.custom("max_blocks_64tok", 1, 2, 64, (32, 64, 64), (4, 4, 4), 0.95, 4, sigma=2.0, a_fixed=(0.25, 6.0),
               seed=34),
]


@pytest.mark.parametrize("wl", MAX_NB, ids=lambda w: w.name)
def test_max_block_count_sampled(wl):
    assert math.prod(-(-g // b) for g, b in zip(wl.grid, wl.block)) == 2048
    _run(wl, full_rows=False)


# fp16 and D = 64 at layer scale, sampled like the five configurations: the
# Wan-5B-like layer in fp16, the 64-token layer in fp16, and the Wan-5B-like
# geometry with 48 heads of D = 64.
LAYER_VARIANTS = [
    ("wan5b", torch.float16, None),
    ("head_skew_64tok", torch.float16, None),
    ("wan5b_d64", torch.bfloat16, gen.custom("wan5b_d64", 1, 48, 64, (31, 22, 40), (4, 8, 8), 0.9, 8, sigma=2.0,
                                             a_range=(0.5, 4.0), seed=1002)),
]


@pytest.mark.parametrize("name,dtype,wl", LAYER_VARIANTS, ids=["wan5b-fp16", "head_skew_64tok-fp16", "wan5b_d64"])
def test_layer_variants_sampled(name, dtype, wl):
    _run(wl if wl is not None else gen.WORKLOADS[name], full_rows=False, dtype=dtype)
