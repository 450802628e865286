"""Head costs, slack augmentation and the head-sharded layer on the GPU.

* fvattn_head_cost against the token pairs counted on the host from the
  GPU's own lists (exact integers).
* fvattn_augment: on the GPU's own fp32 block probabilities the additions
  must be exactly the longest prefix of the candidates, ordered by
  (P descending, row, block), that fits the budget; against the oracle's
  augmentation of the same base lists with its fp64 probabilities, the two
  may differ only at candidates whose probabilities lie within the
  tolerance the routing test allows for block probabilities of the
  boundary candidate; attention over the augmented lists matches the oracle.
* heads.step_emulated with the library's kernels, ranks run one after
  another on one GPU: the union of the ranks' outputs equals the whole
  layer run as one problem, bit for bit; with augmentation, every rank stays
  within its slack.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen
from tests import fvtest

pytestmark = pytest.mark.gpu

PROB_RTOL, PROB_ATOL = 2e-3, 1e-6   # GPU block probabilities vs the oracle's (routing test)


def _sizes(wl):
    import oracle
    orc = oracle.get()
    return orc.block_sizes(orc.geom(1, 1, wl.grid, wl.block, wl.D)).astype(np.int64)


def _routed(wl):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    q, k, v = fvtest.make_on_gpu(wl)
    eng = fa.FVAttn(fvtest.geometry(wl), wl.p, wl.k_min, with_probs=True)
    eng.route(q, k)
    torch.cuda.synchronize()
    return fa, eng, q, k, v


def _host_cost(cnt, idx, sizes):
    BH, nb = cnt.shape[0] * cnt.shape[1], cnt.shape[2]
    c, ix = cnt.reshape(BH, nb), idx.reshape(BH, nb, nb)
    out = np.zeros(BH, dtype=np.int64)
    for h in range(BH):
        for i in range(nb):
            out[h] += sizes[i] * sizes[ix[h, i, :c[h, i]]].sum()
    return out


@pytest.mark.parametrize("name", ["wan5b", "head_skew_64tok"])
def test_head_cost_counts_kept_token_pairs(name):
    wl = gen.WORKLOADS[name]
    fa, eng, q, k, v = _routed(wl)
    out = torch.zeros(wl.B * wl.H, dtype=torch.int64, device="cuda")
    fa.head_cost(eng.geo, eng.kv_cnt, eng.kv_idx, out)
    dense = torch.zeros_like(out)
    fa.head_cost(eng.geo, None, None, dense, dense=True)
    torch.cuda.synchronize()
    sizes = _sizes(wl)
    assert np.array_equal(out.cpu().numpy(), _host_cost(eng.kv_cnt.cpu().numpy(), eng.kv_idx.cpu().numpy(), sizes))
    assert (dense.cpu().numpy() == wl.N * wl.N).all()


def _candidates(cnt, idx, P, sizes):
    """Unkept (row, block) pairs in the order (P descending, row, block) and their costs."""
    R, nb = cnt.size, P.shape[-1]
    keep = np.zeros((R, nb), dtype=bool)
    c, ix = cnt.reshape(R), idx.reshape(R, nb)
    for r in range(R):
        keep[r, ix[r, :c[r]]] = True
    rows, js = np.nonzero(~keep)
    p = P.reshape(R, nb)[rows, js]
    order = np.lexsort((js, rows, -p))
    return keep, rows[order], js[order], p[order], (sizes[rows % nb] * sizes[js])[order]


def _added(keep, cnt, idx):
    R, nb = keep.shape
    now = np.zeros_like(keep)
    c, ix = cnt.reshape(R), idx.reshape(R, nb)
    for r in range(R):
        lst = ix[r, :c[r]]
        assert np.all(np.diff(lst) > 0)
        now[r, lst] = True
    assert (now | ~keep).all(), "a kept block was dropped"
    return now & ~keep


AUG_CASES = [
    gen.custom("aug_ragged", 1, 3, 128, (9, 20, 28), (4, 8, 8), 0.8, 3, sigma=2.0, a_range=(0.5, 4.0), seed=81),
    gen.custom("aug_64tok", 1, 4, 128, (8, 12, 20), (4, 4, 4), 0.9, 3, sigma=2.0, a_range=(0.25, 6.0), seed=82),
    gen.WORKLOADS["wan5b"],
]


@pytest.mark.parametrize("wl", AUG_CASES, ids=lambda w: w.name)
def test_augment_prefix_and_oracle(wl):
    import oracle
    orc = oracle.get()
    fa, eng, q, k, v = _routed(wl)
    sizes = _sizes(wl)
    cnt0, idx0 = eng.kv_cnt.cpu().numpy(), eng.kv_idx.cpu().numpy()
    P32 = eng.block_probs.cpu().numpy().astype(np.float64)
    keep, rows, js, p, cost = _candidates(cnt0, idx0, P32, sizes)
    total = int(cost.sum())
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    qh, kh = q.cpu(), k.cpu()
    r = orc.route(g, orc.pool(g, qh), orc.pool(g, kh), 1.0 / math.sqrt(wl.D), wl.p, wl.k_min)
    P64 = r["probs"]
    for budget in (0, total // 50, total // 7, total // 2, total, 10 * total):
        cnt = eng.kv_cnt.clone()
        idx = eng.kv_idx.clone()
        added = torch.zeros(1, dtype=torch.int64, device="cuda")
        mass = torch.zeros(1, dtype=torch.float64, device="cuda")
        fa.augment(eng.geo, eng.block_probs, budget, cnt, idx, eng.ws, added, mass)
        torch.cuda.synchronize()
        c1, i1 = cnt.cpu().numpy(), idx.cpu().numpy()
        now = _added(keep, c1, i1)
        taken = now[rows, js]
        n = int(taken.sum())
        # exact prefix of the order on the GPU's own probabilities
        assert taken[:n].all() and not taken[n:].any(), budget
        spent = int(cost[:n].sum())
        assert spent == int(added.item()) <= budget
        if n < rows.size:
            assert spent + int(cost[n]) > budget
        assert abs(mass.item() - float(p[:n].sum())) <= 1e-9 * max(1.0, float(p[:n].sum()))
        if budget >= total:
            assert (c1 == eng.nb).all()
        # the oracle's augmentation of the same base lists with fp64 probabilities
        oc, oi, opairs, _ = orc.augment(g, P64, budget, cnt0, idx0)
        onow = _added(keep, oc, oi)
        diff = np.argwhere(onow != now)
        if diff.size:
            po = P64.reshape(keep.shape)
            ko, kj = np.nonzero(onow)
            # the oracle's boundary: its smallest added probability, or its largest left out
            lo = po[ko, kj].min() if ko.size else np.inf
            left = po[~keep & ~onow]
            hi = left.max() if left.size else -np.inf
            for rr, jj in diff:
                pc = po[rr, jj]
                tol = PROB_RTOL * pc + PROB_ATOL
                near = min(abs(pc - lo), abs(pc - hi))
                assert near <= tol + PROB_RTOL * max(lo if np.isfinite(lo) else 0, hi if np.isfinite(hi) else 0) + \
                    PROB_ATOL, (budget, rr, jj, pc, lo, hi)
            assert len(diff) <= max(4, 0.01 * max(1, n)), (budget, len(diff), n)


def test_attention_over_augmented_lists_matches_the_oracle():
    import oracle
    orc = oracle.get()
    wl = AUG_CASES[0]
    fa, eng, q, k, v = _routed(wl)
    sizes = _sizes(wl)
    keep, rows, js, p, cost = _candidates(eng.kv_cnt.cpu().numpy(), eng.kv_idx.cpu().numpy(),
                                          eng.block_probs.cpu().numpy(), sizes)
    fa.augment(eng.geo, eng.block_probs, int(cost.sum()) // 5, eng.kv_cnt, eng.kv_idx, eng.ws)
    eng.schedule()
    out = torch.zeros_like(q)
    eng.attend(q, k, v, out)
    torch.cuda.synchronize()
    assert eng.status() == 0
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    rows_all = np.arange(wl.B * wl.H * wl.N)
    ref, wsum = orc.attn_rows(g, q.cpu(), k.cpu(), v.cpu(), 1.0 / math.sqrt(wl.D), rows_all,
                              eng.kv_cnt.cpu().numpy(), eng.kv_idx.cpu().numpy())
    mx, mean = fvtest.attn_errors(out, rows_all, ref, wl.D)
    assert mx <= fvtest.ATTN_MAX_ABS and mean <= fvtest.ATTN_MEAN_ABS, (mx, mean)


SHARD_WL = gen.custom("shard8", 1, 8, 128, (16, 24, 40), (4, 8, 8), 0.9, 4, sigma=2.0,
                      a_fixed=(0.4, 0.4, 0.4, 0.4, 3.0, 3.0, 3.0, 3.0), seed=83)


def _emulated(world, sasa, wl=SHARD_WL):
    from block_sparse_attention_fvattn_b200 import heads
    q, k, v = fvtest.make_on_gpu(wl)
    be = heads.GpuBackend(fvtest.geometry(wl), wl.p, wl.k_min, "cuda")
    states = [heads.RankState(r, world, wl.H, be, sasa=sasa) for r in range(world)]
    for st in states:
        for name, t in (("q", q), ("k", k), ("v", v)):
            st.buf[name][:st.S] = t[0, st.h0:st.h1]
    plan = heads.step_emulated(states)
    torch.cuda.synchronize()
    return q, k, v, states, plan, be


@pytest.mark.parametrize("world", [2, 3, 4])
def test_sharded_layer_matches_the_whole_layer(world):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    q, k, v, states, plan, be = _emulated(world, sasa=False)
    ref = fa.FVAttn(fvtest.geometry(SHARD_WL), SHARD_WL.p, SHARD_WL.k_min)(q, k, v)
    torch.cuda.synchronize()
    assert sum(a != b for a, b in zip(plan.owner_in, plan.owner_out)) >= 1
    assert max(plan.load_after) < max(plan.load_static)
    for st in states:
        assert torch.equal(st.output(), ref[0, st.h0:st.h1]), st.rank


def test_sharded_layer_augmentation_within_slack():
    import oracle
    orc = oracle.get()
    world = 4
    q, k, v, states, plan, be = _emulated(world, sasa=True)
    crit = plan.critical
    wl = SHARD_WL
    for st in states:
        added = int(st.added_pairs.item())
        assert 0 <= added <= crit - plan.load_after[st.rank]
        final = int(be.head_cost(st.buf, st.F).sum().item())
        assert final == plan.load_after[st.rank] + added <= crit
        # sampled rows of the rank's heads against the oracle on the augmented lists
        F = st.F
        g = orc.geom(1, F, wl.grid, wl.block, wl.D)
        qs, ks, vs = (st.buf[n][:F].unsqueeze(0) for n in ("q", "k", "v"))
        cnt = st.buf["cnt"][:F].unsqueeze(0)
        rows = np.random.default_rng(st.rank).choice(F * wl.N, size=256, replace=False)
        ref, _ = orc.attn_rows(g, qs.cpu(), ks.cpu(), vs.cpu(), 1.0 / math.sqrt(wl.D), rows, cnt.cpu().numpy(),
                               st.buf["idx"][:F].unsqueeze(0).cpu().numpy())
        # outputs of the slots still held here (the received head's output was sent back)
        out = torch.zeros((F, wl.N, wl.D), dtype=q.dtype, device="cuda")
        for s, h in enumerate(st.slot_head):
            if plan.owner_in[h] == st.rank:
                out[s] = st.output()[h - st.h0]
            else:
                out[s] = states[plan.owner_in[h]].output()[h - states[plan.owner_in[h]].h0]
        mx, mean = fvtest.attn_errors(out, rows, ref, wl.D)
        assert mx <= fvtest.ATTN_MAX_ABS and mean <= fvtest.ATTN_MEAN_ABS, (st.rank, mx, mean)
