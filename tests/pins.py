"""Pins of the fp64 oracle to facts other than the oracle itself.

Each function takes an `oracle.Oracle` and raises AssertionError when the
oracle disagrees with:
  * numbers the pages print (worked VSA routing example; 96*64*64 tokens),
  * a library routine that computes the same thing by another road
    (numpy reshape-mean, numpy/torch top-k, torch scaled_dot_product_attention
    with or without a token mask),
  * brute force on tiny inputs (enumeration of all 2^nb block subsets), or
  * invariants the method fixes (kept mass >= p, floor, diagonal, ascending,
    weights summing to one, convex combination).
The same functions are re-run on deliberately broken copies of the oracle in
`test_oracle_mutants.py`; every broken copy must fail at least one of them.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _token_blocks(grid, block):
    """Independent token -> block map (numpy, raster order T slowest)."""
    T, Hg, W = grid
    bt, bh, bw = block
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(W), indexing="ij")
    nbh, nbw = -(-Hg // bh), -(-W // bw)
    return ((t // bt) * nbh + (y // bh)) * nbw + (x // bw)


def _softmax_rows(s):
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def _np_scores(qbar, kbar, scale):
    return scale * np.einsum("bhid,bhjd->bhij", qbar, kbar)


def _small(grid, block, H=2, D=32, sigma=1.5, seed=11, iid=False):
    if iid:
        wl = gen.custom("pin", 1, H, D, grid, block, 0.9, 2, seed=seed)
    else:
        wl = gen.custom("pin", 1, H, D, grid, block, 0.9, 2, sigma=sigma, a_range=(0.5, 3.0), seed=seed)
    q, k, v = gen.make_inputs(wl, "cpu")
    return wl, q, k, v


# ---------------------------------------------------------------- geometry
def pin_vsa_worked_example(orc):
    ex = _load("vsa_routing_example.json")
    g = orc.geom(1, 1, ex["dit_seq_shape"], ex["block_size"], 64)
    nb = orc.num_blocks(g)
    assert nb == ex["num_blocks"], nb
    assert int(np.prod(ex["dit_seq_shape"])) == ex["seq_len"]
    assert round(100.0 * ex["topk"] / nb, 1) == ex["keep_ratio_percent_1dp"]
    sizes = orc.block_sizes(g)
    tb = _token_blocks(ex["dit_seq_shape"], ex["block_size"]).ravel()
    brute = np.bincount(tb, minlength=nb)
    assert np.array_equal(sizes, brute), "valid token counts per block"
    assert sizes.sum() == ex["seq_len"]


def pin_long_video_tokens(orc):
    ex = _load("long_video_tokens.json")
    assert int(np.prod(ex["latent_grid"])) == ex["tokens"]
    g = orc.geom(1, 1, ex["latent_grid"], (4, 8, 8), 64)
    assert orc.num_blocks(g) == 24 * 8 * 8
    assert orc.block_sizes(g).sum() == ex["tokens"]
    # a token-level bool mask would take n^2 bytes (~155e9, "about 160 GB");
    # per-(head, query-block) lists take at most 4*nb^2 bytes per head
    assert abs(ex["tokens"] ** 2 / 1e9 - ex["bool_mask_gb_approx"]) < 0.05 * ex["bool_mask_gb_approx"]
    assert 4 * orc.num_blocks(g) ** 2 < ex["tokens"] ** 2 / 1000


# ---------------------------------------------------------------- pooling
def pin_pool_reshape_mean(orc):
    wl, q, k, v = _small((8, 16, 16), (4, 8, 8))
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    got = orc.pool(g, q)
    x = q.double().numpy().reshape(1, wl.H, 2, 4, 2, 8, 2, 8, wl.D)
    ref = x.mean(axis=(3, 5, 7)).reshape(1, wl.H, 8, wl.D)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_pool_ragged_bruteforce(orc):
    grid, block = (5, 11, 13), (4, 8, 8)
    wl, q, k, v = _small(grid, block, D=16)
    g = orc.geom(wl.B, wl.H, grid, block, wl.D)
    nb = orc.num_blocks(g)
    got = orc.pool(g, k)
    tb = _token_blocks(grid, block).ravel()
    x = k.double().numpy()[0]
    for h in range(wl.H):
        sums = np.zeros((nb, wl.D))
        np.add.at(sums, tb, x[h])
        cnt = np.bincount(tb, minlength=nb)[:, None]
        np.testing.assert_allclose(got[0, h], sums / cnt, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- routing
def _route_small(orc, grid, block, p, k_min, H=2, D=32, iid=True, seed=5, scale=None):
    wl, q, k, v = _small(grid, block, H=H, D=D, iid=iid, seed=seed)
    g = orc.geom(wl.B, wl.H, grid, block, D)
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    r = orc.route(g, qb, kb, scale, p, k_min)
    return wl, g, q, k, v, qb, kb, scale, r


def pin_topp_bruteforce(orc):
    """nb = 8: enumerate all 256 subsets of every row."""
    grid, block = (8, 16, 16), (4, 8, 8)
    for p, k_min in [(0.3, 1), (0.5, 1), (0.9, 2), (0.99, 1), (0.75, 5)]:
        wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, p, k_min, D=8, iid=True, seed=3)
        P = _softmax_rows(_np_scores(qb, kb, scale))
        nb = P.shape[-1]
        subsets = [np.array(c, dtype=int) for m in range(1, nb + 1) for c in itertools.combinations(range(nb), m)]
        for h in range(wl.H):
            for i in range(nb):
                row = P[0, h, i]
                best_m, best_set = None, None
                for sset in subsets:
                    mass = row[sset].sum()
                    if mass >= p and (best_m is None or len(sset) < best_m or
                                      (len(sset) == best_m and mass > row[best_set].sum())):
                        best_m, best_set = len(sset), sset
                m = min(nb, max(best_m, k_min))
                top_m = max((c for c in subsets if len(c) == m), key=lambda c: row[c].sum())
                expect = sorted(set(top_m.tolist()) | {i})
                cnt = r["kv_cnt"][0, h, i]
                got = r["kv_idx"][0, h, i, :cnt].tolist()
                assert got == expect, (p, k_min, h, i, got, expect)
                # the Top-p count read from the oracle's cumulative sums
                cum = r["cum"][0, h, i]
                m_p = int(np.argmax(cum >= p)) + 1
                assert m_p == best_m, (m_p, best_m)


def pin_topk_reduction(orc):
    """p -> 0+ with k_min = k is a fixed top-k (VSA's selection) plus the diagonal."""
    grid, block = (12, 24, 24), (4, 8, 8)
    for kk in (1, 3, 7, 18):
        wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, 1e-12, kk, D=32, iid=False)
        s = _np_scores(qb, kb, scale)
        nb = s.shape[-1]
        for h in range(wl.H):
            for i in range(nb):
                top = torch.topk(torch.from_numpy(s[0, h, i]), kk).indices.tolist()
                expect = sorted(set(top) | {i})
                cnt = r["kv_cnt"][0, h, i]
                assert r["kv_idx"][0, h, i, :cnt].tolist() == expect, (kk, h, i)


def pin_dense_reduction(orc):
    """p = 1 or k_min = nb keeps every block; attention is then plain softmax
    attention, checked against torch's scaled_dot_product_attention in fp64."""
    for grid in [(8, 16, 16), (5, 11, 13)]:
        block = (4, 8, 8)
        for p, k_min in [(1.0, 1), (0.5, None)]:
            wl, q, k, v = _small(grid, block, H=2, D=32)
            g = orc.geom(wl.B, wl.H, grid, block, wl.D)
            nb = orc.num_blocks(g)
            km = nb if k_min is None else k_min
            qb, kb = orc.pool(g, q), orc.pool(g, k)
            r = orc.route(g, qb, kb, 1.0 / math.sqrt(wl.D), p, km)
            assert (r["kv_cnt"] == nb).all()
            assert (r["kv_idx"] == np.arange(nb)).all()
            N = wl.N
            rows = np.arange(wl.H * N)
            out, ws = orc.attn_rows(g, q, k, v, 1.0 / math.sqrt(wl.D), rows, r["kv_cnt"], r["kv_idx"])
            ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
            np.testing.assert_allclose(out.reshape(1, wl.H, N, wl.D), ref.numpy(), rtol=0, atol=1e-12)
            np.testing.assert_allclose(ws, 1.0, rtol=0, atol=1e-12)


def pin_sparse_attention_masked_sdpa(orc):
    """Attention over a kept list equals SDPA with the token mask the list implies."""
    grid, block = (6, 13, 10), (4, 8, 8)
    wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, 0.6, 2, H=2, D=16, iid=False)
    N = wl.N
    tb = _token_blocks(grid, block).ravel()
    rows = np.arange(wl.H * N)
    out, ws = orc.attn_rows(g, q, k, v, scale, rows, r["kv_cnt"], r["kv_idx"])
    nb = orc.num_blocks(g)
    for h in range(wl.H):
        keep = np.zeros((nb, nb), dtype=bool)
        for i in range(nb):
            keep[i, r["kv_idx"][0, h, i, :r["kv_cnt"][0, h, i]]] = True
        mask = torch.from_numpy(keep[tb][:, tb])
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[0, h].double(), k[0, h].double(), v[0, h].double(), attn_mask=mask, scale=scale)
        np.testing.assert_allclose(out[h * N:(h + 1) * N], ref.numpy(), rtol=0, atol=1e-12)


def pin_route_order_probs_cum(orc):
    """The oracle's per-row outputs that the GPU checks read -- the ranking,
    the block probabilities and the cumulative sums -- against numpy on the
    oracle's own pooled means: order = a stable sort of the scores
    descending (equal scores keep the lower block first: numpy's lexsort),
    probs = the softmax of the scores in block order, cum = the running sum of
    probs taken in that order."""
    cases = [((12, 24, 40), (4, 8, 8), False, 0.9, 4), ((9, 20, 28), (4, 8, 8), True, 0.6, 2),
             ((8, 12, 20), (4, 4, 4), False, 0.95, 3)]
    for grid, block, iid, p, k_min in cases:
        wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, p, k_min, H=2, D=32, iid=iid, seed=13)
        s = _np_scores(qb, kb, scale)
        P = _softmax_rows(s)
        nb = s.shape[-1]
        np.testing.assert_allclose(r["probs"], P, rtol=0, atol=1e-13)
        for h in range(wl.H):
            for i in range(nb):
                expect = np.lexsort((np.arange(nb), -s[0, h, i]))
                assert r["order"][0, h, i].tolist() == expect.tolist(), (grid, h, i)
        ranked = np.take_along_axis(P, r["order"].astype(np.int64), -1)
        np.testing.assert_allclose(r["cum"], np.cumsum(ranked, axis=-1), rtol=0, atol=1e-12)


def pin_custom_scale(orc):
    """A softmax scale other than 1/sqrt(D) (the problem's softmax_scale
    override) enters the block scores and the attention logits alike: the
    probabilities are numpy's softmax of scale * Qbar.Kbar, the attention over
    the kept lists is SDPA with that scale under the lists' token mask, and
    the lists differ from those of the default scale (the value is used)."""
    grid, block, D = (6, 13, 10), (4, 8, 8), 16
    default = _route_small(orc, grid, block, 0.8, 1, H=2, D=D, iid=False, seed=17)[-1]
    for scale in (0.9, 0.04):
        wl, g, q, k, v, qb, kb, sc, r = _route_small(orc, grid, block, 0.8, 1, H=2, D=D, iid=False, seed=17,
                                                      scale=scale)
        assert sc == scale
        np.testing.assert_allclose(r["probs"], _softmax_rows(_np_scores(qb, kb, scale)), rtol=0, atol=1e-13)
        assert not np.array_equal(r["kv_cnt"], default["kv_cnt"]), scale
        N, nb = wl.N, orc.num_blocks(g)
        tb = _token_blocks(grid, block).ravel()
        out, ws = orc.attn_rows(g, q, k, v, scale, np.arange(wl.H * N), r["kv_cnt"], r["kv_idx"])
        np.testing.assert_allclose(ws, 1.0, rtol=0, atol=1e-12)
        for h in range(wl.H):
            keep = np.zeros((nb, nb), dtype=bool)
            for i in range(nb):
                keep[i, r["kv_idx"][0, h, i, :r["kv_cnt"][0, h, i]]] = True
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[0, h].double(), k[0, h].double(), v[0, h].double(), attn_mask=torch.from_numpy(keep[tb][:, tb]),
                scale=scale)
            np.testing.assert_allclose(out[h * N:(h + 1) * N], ref.numpy(), rtol=0, atol=1e-12)


def pin_invariants(orc):
    grid, block = (9, 20, 28), (4, 8, 8)
    for p, k_min in [(0.9, 4), (0.5, 1), (0.97, 10)]:
        wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, p, k_min, H=2, D=32, iid=False)
        P = _softmax_rows(_np_scores(qb, kb, scale))
        nb = P.shape[-1]
        for h in range(wl.H):
            for i in range(nb):
                cnt = r["kv_cnt"][0, h, i]
                lst = r["kv_idx"][0, h, i, :cnt]
                assert min(k_min, nb) <= cnt <= nb
                assert i in lst
                assert np.all(np.diff(lst) > 0)
                assert P[0, h, i, lst].sum() >= p - 1e-12
                # minimality: without the floor and the diagonal, dropping the
                # weakest Top-p block would fall below p
                cum = r["cum"][0, h, i]
                m_p = int(np.argmax(cum >= p)) + 1
                top = np.sort(P[0, h, i])[::-1]
                assert top[:m_p].sum() >= p - 1e-12 and (m_p == 1 or top[:m_p - 1].sum() < p + 1e-12)
        rows = np.random.default_rng(0).choice(wl.H * wl.N, size=200, replace=False)
        out, ws, lo, hi = orc.attn_rows(g, q, k, v, scale, rows, r["kv_cnt"], r["kv_idx"], want_bounds=True)
        np.testing.assert_allclose(ws, 1.0, rtol=0, atol=1e-12)
        assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)


def pin_tie_order(orc):
    """Equal scores rank the lower block index first: duplicate two key blocks."""
    grid, block = (4, 16, 16), (4, 8, 8)   # 4 blocks, all full
    wl, q, k, v = _small(grid, block, H=1, D=8, iid=True, seed=9)
    tb = _token_blocks(grid, block).ravel()
    kk = k.clone()
    kk[0, 0, tb == 3] = kk[0, 0, tb == 1]          # block 3 := block 1 (same mean)
    g = orc.geom(1, 1, grid, block, 8)
    qb, kb = orc.pool(g, q), orc.pool(g, kk)
    assert np.array_equal(kb[0, 0, 1], kb[0, 0, 3])
    s = _np_scores(qb, kb, 0.5)[0, 0]
    for i in range(4):
        # choose k_min so that the floor cuts exactly between the two tied blocks
        order = sorted(range(4), key=lambda j: (-s[i, j], j))
        pos = order.index(1)
        assert order[pos + 1] == 3
        r = orc.route(g, qb, kb, 0.5, 1e-12, pos + 1)
        lst = set(r["kv_idx"][0, 0, i, :r["kv_cnt"][0, 0, i]].tolist())
        assert 1 in lst
        assert (3 not in lst) or i == 3


def pin_nonfinite_repair(orc):
    grid, block = (8, 16, 16), (4, 8, 8)
    wl, q, k, v = _small(grid, block, H=2, D=16, iid=True)
    tb = _token_blocks(grid, block).ravel()
    qq = q.clone()
    qq[0, 1, np.where(tb == 5)[0][:3]] = float("inf")
    g = orc.geom(1, 2, grid, block, 16)
    qb, kb = orc.pool(g, qq), orc.pool(g, k)
    r = orc.route(g, qb, kb, 0.25, 0.3, 1)
    nb = orc.num_blocks(g)
    assert r["nonfinite"][0, 1, 5] == 1 and r["nonfinite"].sum() == 1
    assert r["kv_cnt"][0, 1, 5] == nb and (r["kv_idx"][0, 1, 5] == np.arange(nb)).all()
    assert (r["kv_cnt"][0, 0] < nb).any()


# ---------------------------------------------------------------- slack augmentation
def _augment_case(orc, grid, block, p, k_min, H=1, seed=17):
    wl, g, q, k, v, qb, kb, scale, r = _route_small(orc, grid, block, p, k_min, H=H, D=16, iid=True, seed=seed)
    return g, r


def pin_augment_bruteforce_equal_costs(orc):
    """All blocks hold 256 tokens, so every candidate costs the same: the
    added set must have the largest mass of all candidate subsets within the
    budget (enumerated), and never exceed it."""
    grid, block = (8, 16, 16), (4, 8, 8)          # 8 full blocks
    g, r = _augment_case(orc, grid, block, 0.3, 1, H=1)
    nb = 8
    unit = 256 * 256
    keep = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        keep[i, r["kv_idx"][0, 0, i, :r["kv_cnt"][0, 0, i]]] = True
    cand = [(i, j) for i in range(nb) for j in range(nb) if not keep[i, j]]
    P = r["probs"][0, 0]
    assert len(cand) >= 8
    for m in (0, 1, 2, 3):
        for slack in (0, unit // 2):
            budget = m * unit + slack
            cnt, idx, added, mass = orc.augment(g, r["probs"], budget, r["kv_cnt"], r["kv_idx"])
            best = max(sum(P[i, j] for i, j in comb) for comb in itertools.combinations(cand, m)) if m else 0.0
            assert added == m * unit and added <= budget
            assert abs(mass - best) <= 1e-12, (m, mass, best)
            got = sum(P[i, j] for i in range(nb) for j in idx[0, 0, i, :cnt[0, 0, i]] if not keep[i, j])
            assert abs(got - best) <= 1e-12
            for i in range(nb):
                lst = idx[0, 0, i, :cnt[0, 0, i]]
                assert np.all(np.diff(lst) > 0) and set(np.flatnonzero(keep[i])) <= set(lst.tolist())


def pin_augment_prefix_rule(orc):
    """Ragged blocks (unequal costs): the additions are a prefix of the
    candidates ordered by P descending (then row, then block): every added
    candidate comes before every candidate left out, the budget holds, and
    the first candidate left out does not fit in what remains. Budget 0
    changes nothing; a budget covering every candidate keeps every block."""
    grid, block = (9, 20, 28), (4, 8, 8)          # 3*3*4 = 36 blocks, ragged edges
    g, r = _augment_case(orc, grid, block, 0.5, 2, H=2, seed=19)
    nb = orc.num_blocks(g)
    sizes = orc.block_sizes(g).astype(np.int64)
    base = r["kv_cnt"].reshape(-1), r["kv_idx"].reshape(-1, nb)
    keep = np.zeros((base[0].size, nb), dtype=bool)
    for row in range(base[0].size):
        keep[row, base[1][row, :base[0][row]]] = True
    P = r["probs"].reshape(-1, nb)
    rows, js = np.nonzero(~keep)
    cost = sizes[rows % nb] * sizes[js]
    order = np.lexsort((js, rows, -P[rows, js]))
    total = int(cost.sum())
    for budget in (0, int(cost[order[0]]) - 1, total // 7, total // 2 + 12345, total - 1, total):
        cnt, idx, added, mass = orc.augment(g, r["probs"], budget, r["kv_cnt"], r["kv_idx"])
        cnt, idx = cnt.reshape(-1), idx.reshape(-1, nb)
        now = np.zeros_like(keep)
        for row in range(cnt.size):
            lst = idx[row, :cnt[row]]
            assert np.all(np.diff(lst) > 0)
            now[row, lst] = True
        assert (now | ~keep).all(), "a kept block was dropped"
        taken = now[rows, js][order]
        n_taken = int(taken.sum())
        assert taken[:n_taken].all() and not taken[n_taken:].any(), "additions are not a prefix of the order"
        spent = int(cost[order][:n_taken].sum())
        assert spent == added and spent <= budget
        if n_taken < order.size:
            assert spent + int(cost[order[n_taken]]) > budget
        assert abs(mass - float(P[rows, js][order][:n_taken].sum())) <= 1e-12
        if budget == 0:
            assert n_taken == 0
        if budget == total:
            assert (cnt == nb).all()


# ---------------------------------------------------------------- input types
def pin_element_decode(orc):
    """The oracle widens every one of the 65536 bit patterns exactly like
    numpy's IEEE binary16 and torch's bfloat16 conversions."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    for fp16 in (True, False):
        got = orc.widen(bits, fp16)
        if fp16:
            ref = bits.view(np.float16).astype(np.float64)
        else:
            ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got), nan), fp16
        assert np.array_equal(got[~nan], ref[~nan]), fp16


def pin_fp16_inputs(orc):
    """fp16 Q, K, V: pooling is a reshape-mean and p = 1 attention is torch's
    scaled_dot_product_attention, both on the fp16 values widened to fp64."""
    grid, block = (8, 16, 16), (4, 8, 8)
    wl, q, k, v = _small(grid, block, H=2, D=32)
    q16, k16, v16 = (t.float().to(torch.float16) for t in (q, k, v))
    g = orc.geom(wl.B, wl.H, grid, block, wl.D, fp16=True)
    qb = orc.pool(g, q16)
    x = q16.double().numpy().reshape(1, wl.H, 2, 4, 2, 8, 2, 8, wl.D)
    np.testing.assert_allclose(qb, x.mean(axis=(3, 5, 7)).reshape(1, wl.H, 8, wl.D), rtol=0, atol=1e-12)
    kb = orc.pool(g, k16)
    scale = 1.0 / math.sqrt(wl.D)
    r = orc.route(g, qb, kb, scale, 1.0, 1)
    rows = np.arange(wl.H * wl.N)
    out, ws = orc.attn_rows(g, q16, k16, v16, scale, rows, r["kv_cnt"], r["kv_idx"])
    ref = torch.nn.functional.scaled_dot_product_attention(q16.double(), k16.double(), v16.double())
    np.testing.assert_allclose(out.reshape(1, wl.H, wl.N, wl.D), ref.numpy(), rtol=0, atol=1e-12)


ALL_PINS = [
    pin_vsa_worked_example, pin_long_video_tokens, pin_pool_reshape_mean, pin_pool_ragged_bruteforce,
    pin_topp_bruteforce, pin_topk_reduction, pin_dense_reduction, pin_sparse_attention_masked_sdpa,
    pin_route_order_probs_cum, pin_custom_scale, pin_invariants, pin_tie_order, pin_nonfinite_repair, pin_element_decode, pin_fp16_inputs,
    pin_augment_bruteforce_equal_costs, pin_augment_prefix_rule,
]
