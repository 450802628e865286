"""Head-sharded layer with Runtime Load Balancing and slack augmentation, on
the CPU.

The host logic of `heads` (shards, the migration plan, the slot moves, the
point-to-point exchanges and the reassembly of each rank's output) runs
with the oracle standing in for the kernels (tests/cpu_backend.py): three
ranks emulated in one process, and two real gloo ranks in two processes.
Every head is routed and attended alone wherever it runs, so the union of
the ranks' outputs must equal a single-process run bit for bit; with the
augmentation on, every rank must stay within its slack and the critical
rank must keep its lists.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# heads of very different kept work: near-dense (small a_h) and sparse
WL = gen.custom("heads7", 1, 7, 32, (8, 16, 24), (4, 8, 8), 0.9, 2, sigma=2.0,
                a_fixed=(0.3, 0.3, 0.3, 4.0, 4.0, 4.0, 4.0), seed=71)


def _reference(orc):
    """Every head of the layer in one oracle problem: lists, outputs (bf16)."""
    q, k, v = gen.make_inputs(WL, "cpu")
    g = orc.geom(1, WL.H, WL.grid, WL.block, WL.D)
    scale = 1.0 / math.sqrt(WL.D)
    r = orc.route(g, orc.pool(g, q), orc.pool(g, k), scale, WL.p, WL.k_min)
    out, _ = orc.attn_rows(g, q, k, v, scale, np.arange(WL.H * WL.N), r["kv_cnt"], r["kv_idx"])
    return q, k, v, r, torch.from_numpy(out.reshape(WL.H, WL.N, WL.D)).to(torch.bfloat16)


def _states(orc, world, q, k, v, sasa):
    from block_sparse_attention_fvattn_b200 import heads
    from tests.cpu_backend import OracleBackend
    be = OracleBackend(WL, orc)
    states = [heads.RankState(r, world, WL.H, be, sasa=sasa) for r in range(world)]
    for st in states:
        for name, t in (("q", q), ("k", k), ("v", v)):
            st.buf[name][:st.S] = t[0, st.h0:st.h1]
    return states, be


@pytest.mark.parametrize("world", [2, 3, 4])
def test_emulated_ranks_match_one_process(oracle_lib, world):
    from block_sparse_attention_fvattn_b200 import heads
    q, k, v, r, ref = _reference(oracle_lib)
    states, be = _states(oracle_lib, world, q, k, v, sasa=False)
    plan = heads.step_emulated(states)
    assert max(plan.load_after) <= max(plan.load_static)
    moved = sum(a != b for a, b in zip(plan.owner_in, plan.owner_out))
    assert moved >= 1, plan              # the skewed heads force a migration
    assert max(plan.load_after) < max(plan.load_static)
    for st in states:
        assert torch.equal(st.output(), ref[st.h0:st.h1]), st.rank
    # the gathered costs are the heads' valid token pairs under the one-process lists
    for h in range(WL.H):
        c = r["kv_cnt"][0, h]
        sizes = be.sizes
        assert plan.costs[h] == sum(int(sizes[i]) * int(sizes[r["kv_idx"][0, h, i, :c[i]]].sum())
                                    for i in range(be.nb))


def test_emulated_augmentation_stays_within_the_slack(oracle_lib):
    from block_sparse_attention_fvattn_b200 import heads
    q, k, v, r, ref = _reference(oracle_lib)
    world = 3
    states, be = _states(oracle_lib, world, q, k, v, sasa=True)
    plan = heads.step_emulated(states)
    crit = plan.critical
    some_added = False
    for st in states:
        budget = crit - plan.load_after[st.rank]
        added = int(st.added_pairs[0])
        assert 0 <= added <= budget
        if plan.load_after[st.rank] == crit:
            assert added == 0                           # the critical rank keeps its lists
        some_added |= added > 0
        # final work of the rank: never above the critical path
        final = int(be.head_cost(st.buf, st.F).sum())
        assert final == plan.load_after[st.rank] + added <= crit
        # outputs: attention of each of the rank's heads over its augmented lists
        g = oracle_lib.geom(1, st.F, WL.grid, WL.block, WL.D)
        out, _ = oracle_lib.attn_rows(g, st.buf["q"][:st.F].unsqueeze(0), st.buf["k"][:st.F].unsqueeze(0),
                                      st.buf["v"][:st.F].unsqueeze(0), 1.0 / math.sqrt(WL.D),
                                      np.arange(st.F * WL.N), st.buf["cnt"][:st.F].numpy()[None],
                                      st.buf["idx"][:st.F].numpy()[None])
        exp = torch.from_numpy(out.reshape(st.F, WL.N, WL.D)).to(torch.bfloat16)
        for s, h in enumerate(st.slot_head):
            if plan.owner_in[h] == st.rank:
                assert torch.equal(st.output()[h - st.h0], exp[s])
    assert some_added


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, sasa, qout):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle
    from block_sparse_attention_fvattn_b200 import heads
    from tests.cpu_backend import OracleBackend
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        orc = oracle.get()
        q, k, v = gen.make_inputs(WL, "cpu")
        st = heads.RankState(rank, world, WL.H, OracleBackend(WL, orc), sasa=sasa)
        for name, t in (("q", q), ("k", k), ("v", v)):
            st.buf[name][:st.S] = t[0, st.h0:st.h1]
        heads.step_distributed(st, heads.TorchComm())
        added = int(st.added_pairs[0]) if st.added_pairs is not None else 0
        # numpy copies pickle by value: the parent may read them after this process has exited
        qout.put((rank, st.output().view(torch.int16).numpy().copy(), st.plan.owner_out, st.plan.load_after, added))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sasa", [False, True])
def test_two_gloo_ranks_match_one_process(oracle_lib, sasa):
    import torch.multiprocessing as mp
    q, k, v, r, ref = _reference(oracle_lib)
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(rk, world, port, sasa, qout)) for rk in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, o, owner, load, added = qout.get(timeout=300)
        got[rank] = (torch.from_numpy(o).view(torch.bfloat16), owner, load, added)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0][1] == got[1][1]                        # every rank computed the same plan
    from block_sparse_attention_fvattn_b200 import heads
    crit = max(got[0][2])
    for rank in range(world):
        h0, h1 = heads.shard_range(WL.H, world, rank)
        if not sasa:
            assert torch.equal(got[rank][0], ref[h0:h1]), rank
        else:
            assert got[rank][3] <= crit - got[0][2][rank]
