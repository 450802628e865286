"""The list checker of the GPU parity tests, on the CPU.

The GPU tests accept a kept list that differs from the oracle's only under
stated excuses, so the checker itself must reject every plausible wrong row.
Here the "GPU" rows are the oracle's own lists with one planted mistake each
(a dropped diagonal, a duplicate, a kept count one short, a block swapped for
a much weaker one, a list out of order); each must be flagged, while the
oracle's lists, and an exact tie resolved the other way, must pass.
"""
import math

import numpy as np
import pytest

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest


@pytest.fixture(scope="module")
def case(oracle_lib):
    orc = oracle_lib
    wl = gen.custom("chk", 1, 3, 64, (12, 24, 40), (4, 8, 8), 0.8, 3, sigma=2.0, a_range=(0.5, 3.0), seed=51)
    q, k, _ = gen.make_inputs(wl, "cpu")
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    scale = 1.0 / math.sqrt(wl.D)
    r = orc.route(g, qb, kb, scale, wl.p, wl.k_min)
    bound = fvtest.score_bound(orc, g, q, k, qb, kb, scale, tc=False)
    return wl, r, bound


def _check(wl, r, bound, cnt, idx):
    return fvtest.compare_lists(cnt, idx, r, bound, wl.p, wl.k_min)


def _rows(r, pred):
    cnt, order = r["kv_cnt"], r["order"]
    out = []
    B, H, nb = cnt.shape
    for h in range(H):
        for i in range(nb):
            if pred(h, i, cnt[0, h, i], order[0, h, i], r["cum"][0, h, i], r["probs"][0, h, i]):
                out.append((h, i))
    return out


def test_oracle_lists_pass(case):
    wl, r, bound = case
    res = _check(wl, r, bound, r["kv_cnt"], r["kv_idx"])
    assert res.identical == res.rows and res.invalid == 0 and res.unexcused == 0, res.summary()


@pytest.fixture(scope="module")
def iid_case(oracle_lib):
    # i.i.d. inputs: the diagonal block lands anywhere in the ranking
    orc = oracle_lib
    wl = gen.custom("chk_iid", 1, 3, 64, (12, 24, 40), (4, 8, 8), 0.6, 3, seed=52)
    q, k, _ = gen.make_inputs(wl, "cpu")
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    scale = 1.0 / math.sqrt(wl.D)
    r = orc.route(g, qb, kb, scale, wl.p, wl.k_min)
    return wl, r, fvtest.score_bound(orc, g, q, k, qb, kb, scale, tc=False)


@pytest.mark.parametrize("where", ["boundary_rank", "repair_only"])
def test_dropped_diagonal_is_invalid(iid_case, where):
    wl, r, bound = iid_case
    nb = r["kv_cnt"].shape[-1]
    if where == "boundary_rank":
        # the diagonal block is the last block Top-p / the floor kept
        rows = _rows(r, lambda h, i, c, o, cum, P: o[c - 1] == i)
    else:
        # the diagonal block entered only through the repair
        rows = _rows(r, lambda h, i, c, o, cum, P: i not in o[:c - 1].tolist())
    assert rows
    h, i = rows[0]
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    lst = [j for j in idx[0, h, i, :cnt[0, h, i]] if j != i]
    cnt[0, h, i] = len(lst)
    idx[0, h, i, :nb] = -1
    idx[0, h, i, :len(lst)] = lst
    res = _check(wl, r, bound, cnt, idx)
    assert res.invalid == 1 and res.first_invalid["i"] == i, res.summary()


def test_duplicate_entry_is_invalid(case):
    wl, r, bound = case
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    h, i = 1, 7
    assert cnt[0, h, i] >= 2
    idx[0, h, i, 1] = idx[0, h, i, 0]
    res = _check(wl, r, bound, cnt, idx)
    assert res.invalid >= 1, res.summary()


def test_unsorted_list_is_invalid(case):
    wl, r, bound = case
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    h, i = 0, 5
    assert cnt[0, h, i] >= 2
    idx[0, h, i, [0, 1]] = idx[0, h, i, [1, 0]]
    res = _check(wl, r, bound, cnt, idx)
    assert res.invalid >= 1, res.summary()


def test_short_count_is_invalid(case):
    wl, r, bound = case
    p, kmin = wl.p, wl.k_min
    nb = r["kv_cnt"].shape[-1]

    # rows whose Top-p count exceeds the floor and whose weakest ranked block
    # carries far more than the window of mass
    def pick(h, i, c, o, cum, P):
        m_p = int(np.argmax(cum >= p)) + 1
        return m_p > kmin + 1 and m_p < nb and cum[m_p - 2] < p - 1e-3 and o[m_p - 1] != i and i in o[:m_p].tolist()
    rows = _rows(r, pick)
    assert rows
    h, i = rows[0]
    m_p = int(np.argmax(r["cum"][0, h, i] >= p)) + 1
    weakest = int(r["order"][0, h, i, m_p - 1])
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    lst = [j for j in idx[0, h, i, :cnt[0, h, i]] if j != weakest]
    cnt[0, h, i] = len(lst)
    idx[0, h, i, :len(lst)] = lst
    res = _check(wl, r, bound, cnt, idx)
    assert res.invalid == 1 and res.unexcused == 1, res.summary()


def test_swap_for_a_weaker_block_is_unexcused(case):
    wl, r, bound = case
    nb = r["kv_cnt"].shape[-1]
    rows = _rows(r, lambda h, i, c, o, cum, P: c + 3 < nb and c >= 3)
    h, i = rows[0]
    o = r["order"][0, h, i]
    strongest = int(o[0]) if o[0] != i else int(o[1])
    weakest = int(o[nb - 1])
    assert weakest not in r["kv_idx"][0, h, i, :r["kv_cnt"][0, h, i]].tolist()
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    lst = sorted((set(idx[0, h, i, :cnt[0, h, i]].tolist()) - {strongest}) | {weakest})
    idx[0, h, i, :len(lst)] = lst
    res = _check(wl, r, bound, cnt, idx)
    assert res.unexcused == 1, res.summary()


def test_exact_tie_taken_the_other_way_is_excused(oracle_lib):
    # key blocks 1 and 3 have the same mean, so they tie exactly in every row;
    # in row 2 (scores 3, 1, 0.5, 1 times the scale) the floor k_min = 2 cuts
    # between them: the oracle keeps block 1, a kernel that kept block 3 must
    # be excused as a tie and nothing else
    orc = oracle_lib
    rng = np.random.default_rng(3)
    g = orc.geom(1, 1, (4, 16, 16), (4, 8, 8), 8)           # 4 blocks of 256 tokens
    qb = np.zeros((1, 1, 4, 8))
    qb[..., 0] = 1.0
    kb = rng.standard_normal((1, 1, 4, 8))
    kb[0, 0, :, 0] = [3.0, 1.0, 0.5, 1.0]
    kb[0, 0, 3] = kb[0, 0, 1]
    scale, i, kmin = 0.5, 2, 2
    r = orc.route(g, qb, kb, scale, 1e-12, kmin)
    assert r["order"][0, 0, i].tolist() == [0, 1, 3, 2]
    assert r["kv_idx"][0, 0, i, :r["kv_cnt"][0, 0, i]].tolist() == [0, 1, 2]
    bound = fvtest.ScoreBound(qb, kb, np.abs(qb), np.abs(kb), np.full(4, 256), scale, False)
    cnt, idx = r["kv_cnt"].copy(), r["kv_idx"].copy()
    idx[0, 0, i, :3] = [0, 2, 3]
    res = fvtest.compare_lists(cnt, idx, r, bound, 1e-12, kmin)
    assert res.invalid == 0 and res.unexcused == 0 and res.excused_tie == 1, res.summary()
    # the same swap against a block that does not tie is not excused
    idx[0, 0, i, :3] = [1, 2, 3]
    res = fvtest.compare_lists(cnt, idx, r, bound, 1e-12, kmin)
    assert res.unexcused == 1, res.summary()


def test_bound_covers_fp32_scores(case, oracle_lib):
    # the per-pair bound is an upper bound of the error of an fp32 evaluation
    # of the scores (pooled sums, reciprocal, dot product, scale) done here
    # in a different order than any kernel's
    import torch
    wl, r, bound = case
    orc = oracle_lib
    q, k, _ = gen.make_inputs(wl, "cpu")
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    sizes = orc.block_sizes(g)
    T, Hg, W = wl.grid
    bt, bh, bw = wl.block
    nbh, nbw = -(-Hg // bh), -(-W // bw)
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(W), indexing="ij")
    blk = torch.from_numpy((((t // bt) * nbh + (y // bh)) * nbw + (x // bw)).ravel())
    nb = sizes.size

    def pool32(a):
        out = torch.zeros((wl.H, nb, wl.D), dtype=torch.float32)
        out.index_add_(1, blk, a[0].float())
        return out * (1.0 / torch.from_numpy(sizes.astype(np.float32)))[None, :, None]
    qs, ks = pool32(q), pool32(k)
    s32 = (torch.einsum("hid,hjd->hij", qs, ks) * np.float32(bound.scale)).double().numpy()
    s64 = bound.scale * np.einsum("bhid,bhjd->bhij", bound.qbar, bound.kbar)[0]
    for h in range(wl.H):
        for i in range(0, nb, 5):
            e = bound.row(0, h, i)
            assert (np.abs(s32[h, i] - s64[h, i]) <= e).all()
