"""Benchmark of the adaptive block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole path over one batch of synthetic input:
fvattn_route (block pooling, scores, Top-p + Top-k floor, repair, lists) ->
fvattn_schedule (balanced longest-first CTA work lists) -> fvattn_sparse_attn
(block-sparse attention over the kept blocks). The headline's inputs are
resident in HBM and larger than L2, so no flush is needed between its
steps. The default workload
is the largest single-GPU layer, the 393k-token long video (B=1, H=12,
D=128, grid 96x64x64, 4x8x8 blocks -> 1536 blocks, p=0.85, k_min=32); the
other four workloads are measured after it and reported in the same line
under "other_workloads". A buffer of twice the L2 size is written between
steps only for a layer whose Q, K and V fit in L2 (the tiny case); the
others' inputs are larger than L2 (201 MB and more). Per-kernel times are
medians of per-step CUDA events; each workload's routing lists are checked
against the fp64 oracle (counts of excused rows under "route_parity").

The metric is attention TFLOPS on kept blocks: 4*D*sum_i |i| * sum_{j in S_i} |j|
(valid query tokens x valid kept key tokens) divided by the step time. The
line also carries the sparse/dense latency ratio, routing GB/s, CTA
imbalance, the roofline of the dominant kernel (the attention kernel, bound
by the tensor cores), an end-to-end figure through host buffers, and the
fp64 CPU oracle timed on a bounded sample as a reported baseline.

Multi-GPU (torchrun): every rank runs its own copy of the workload (the path
shards by head with no exchange step), timing is the max over ranks, and
`value` sums the work of all ranks ("scaling": "weak").

--impl reference times the CPU oracle (the reference arm of this build) on
the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_attention_fvattn_b200 import inputs as gen  # noqa: E402

METRIC = "block-sparse attn TFLOPS on kept blocks & % bf16 peak; sparse/dense latency"
UNIT = "TFLOPS"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SRC = os.path.join(ROOT, "block_sparse_attention_fvattn_b200", "csrc", "attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_dram_traffic.txt")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_source_hash():
    with open(ATTN_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current attention kernel source; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    cur = attn_source_hash()
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == workload and parts[1] == cur:
                try:
                    return float(parts[2])
                except ValueError:
                    return None
    return None


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s, p in zip(sm, pw) if p is not None and p > 300] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def workload_desc(wl):
    return (f"{wl.name}: B={wl.B} H={wl.H} D={wl.D} grid(T,H,W)={wl.grid} block={wl.block} "
            f"N={wl.N} p={wl.p} k_min={wl.k_min}")


def valid_sizes(wl):
    T, Hg, W = wl.grid
    bt, bh, bw = wl.block
    nbt, nbh, nbw = -(-T // bt), -(-Hg // bh), -(-W // bw)
    out = np.zeros(nbt * nbh * nbw, dtype=np.int64)
    for j in range(out.size):
        jt, jy, jx = j // (nbh * nbw), (j // nbw) % nbh, j % nbw
        out[j] = min(bt, T - jt * bt) * min(bh, Hg - jy * bh) * min(bw, W - jx * bw)
    return out


def kept_flops(wl, cnt, idx, vs):
    B, H, nb = cnt.shape
    total = 0
    for b in range(B):
        for h in range(H):
            mask = np.arange(nb)[None, :] < cnt[b, h][:, None]
            kept = np.where(mask, vs[np.clip(idx[b, h], 0, nb - 1)], 0).sum(axis=1)
            total += int((vs * kept).sum())
    return 4 * wl.D * total


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, q, k, v, budget_s, seed=0, route=None):
    """Time the fp64 oracle on a bounded sample: full routing (pooling + scores +
    selection over every row), then attention for whole units in a seeded random
    order until the time budget is spent. Returns (flops/s extrapolated to the
    whole step, description, cores)."""
    import oracle
    orc = oracle.get()
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    scale = 1.0 / math.sqrt(wl.D)
    t0 = time.perf_counter()
    if route is None:
        qb, kb = orc.pool(g, q), orc.pool(g, k)
        route = orc.route(g, qb, kb, scale, wl.p, wl.k_min, want_detail=False)
    t_route = time.perf_counter() - t0
    cnt, idx = route["kv_cnt"], route["kv_idx"]
    vs = valid_sizes(wl)
    nb = vs.size
    T, Hg, W = wl.grid
    bt, bh, bw = wl.block
    nbh, nbw = -(-Hg // bh), -(-W // bw)
    rng = np.random.default_rng(seed)
    units = rng.permutation(wl.B * wl.H * nb)
    flops = 0
    t_attn = 0.0
    done = 0
    for u in units:
        bhh, i = divmod(int(u), nb)
        jt, jy, jx = i // (nbh * nbw), (i // nbw) % nbh, i % nbw
        toks = [((t * Hg + y) * W + x) for t in range(jt * bt, min(T, jt * bt + bt))
                for y in range(jy * bh, min(Hg, jy * bh + bh)) for x in range(jx * bw, min(W, jx * bw + bw))]
        rows = np.array(toks, dtype=np.int64) + bhh * wl.N
        b, h = divmod(bhh, wl.H)
        s0 = time.perf_counter()
        orc.attn_rows(g, q, k, v, scale, rows, cnt, idx)
        t_attn += time.perf_counter() - s0
        kept = vs[idx[b, h, i, :cnt[b, h, i]]].sum()
        flops += 4 * wl.D * vs[i] * int(kept)
        done += 1
        if t_attn >= budget_s:
            break
    frac = done / float(wl.B * wl.H * nb)
    t_equiv = t_attn + t_route * frac
    cores = len(os.sched_getaffinity(0))
    desc = (f"fp64 oracle: routing of all {wl.B * wl.H * nb} rows ({t_route:.2f} s) + attention of {done} "
            f"seeded-random units ({t_attn:.2f} s, {flops / 1e9:.1f} GFLOP); routing counted pro rata")
    return flops / t_equiv, desc, cores, done


def run_reference(args, wl, world, rank):
    """CPU oracle arm: each step is a bounded sample of the workload."""
    if rank != 0:
        return
    torch.manual_seed(0)
    q, k, v = gen.make_inputs(wl, "cpu")
    import oracle
    orc = oracle.get()
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D)
    t0 = time.perf_counter()
    qb, kb = orc.pool(g, q), orc.pool(g, k)
    route = orc.route(g, qb, kb, 1.0 / math.sqrt(wl.D), wl.p, wl.k_min, want_detail=False)
    t_route_full = time.perf_counter() - t0
    per_step = max(0.5, min(3.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    for s in range(args.warmup + args.steps):
        val, desc, cores, done = oracle_sample(wl, q, k, v, per_step, seed=s, route=route)
        if s >= args.warmup:
            vals.append(val)
    value = statistics.median(vals) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wl)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: attention of seeded-random whole units for ~{per_step:.1f} s "
                                   f"(last step: {done} units) plus the full routing ({t_route_full:.2f} s, "
                                   f"run once) counted pro rata; kept-block TFLOPS"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def l2_flusher(dev):
    """A buffer twice the L2 size; writing it evicts the previous step's data."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    return torch.empty(max(2 * l2, 1 << 20), dtype=torch.uint8, device=dev)


def use_flush(args, wl, dev, headline):
    """Whether to write an L2-sized buffer between timed steps: `--flush
    always|never`, or by default (auto) only when a step's inputs (Q, K, V)
    fit in L2. Larger inputs cannot stay resident in L2 from one step to the
    next, and the flush's dirty lines would be written back inside the next
    step's timed routing."""
    if args.flush == "always":
        return True
    if args.flush == "never":
        return False
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    elem = 2
    return 3 * wl.B * wl.H * wl.N * wl.D * elem <= l2


def route_parity(wl, q, k, cnt, idx):
    """Routing lists of the GPU vs the fp64 oracle under the parity rule of the
    tests (rows identical / excused at the Top-p boundary / excused as rounding
    ties / unexcused / invalid)."""
    import oracle
    from tests import fvtest
    orc = oracle.get()
    g = orc.geom(wl.B, wl.H, wl.grid, wl.block, wl.D, fp16=q.dtype == torch.float16)
    qh, kh = q.cpu(), k.cpu()
    qb, kb = orc.pool(g, qh), orc.pool(g, kh)
    scale = 1.0 / math.sqrt(wl.D)
    r = orc.route(g, qb, kb, scale, wl.p, wl.k_min)
    nb = cnt.shape[-1]
    bound = fvtest.score_bound(orc, g, qh, kh, qb, kb, scale, tc=nb >= fvtest.TC_SCORES_MIN_BLOCKS)
    res = fvtest.compare_lists(cnt, idx, r, bound, wl.p, wl.k_min)
    return {"rows": res.rows, "identical": res.identical, "excused_topp_window": res.excused_topp,
            "excused_rounding_tie": res.excused_tie, "unexcused": res.unexcused, "invalid": res.invalid}


def measure(args, wl, dev, rank, world, flush, steps, warmup, pk, headline):
    """Time route -> schedule -> attention on one workload.

    Returns (fields of the JSON line, timed-region total ms, kept FLOPs per
    step, engine, tensors). Per-kernel times are medians of per-step CUDA
    events on the launching stream; with `flush` an L2-sized buffer is
    written between steps (outside the events)."""
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    seed = wl.seed + 1000 * rank
    q, k, v = gen.make_inputs(wl, dev, seed=seed)
    edtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    if edtype != torch.bfloat16:
        q, k, v = (t.float().to(edtype) for t in (q, k, v))
    out = torch.empty_like(q)
    geo = fa.Geometry(wl.B, wl.H, wl.D, wl.grid, wl.block, dtype=edtype)
    eng = fa.FVAttn(geo, wl.p, wl.k_min, device=dev)
    stream = torch.cuda.current_stream()
    fl = l2_flusher(dev) if flush else None

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        eng.route(q, k)
        if evs is not None:
            evs[1].record(stream)
        eng.schedule()
        if evs is not None:
            evs[2].record(stream)
        eng.attend(q, k, v, out)
        if evs is not None:
            evs[3].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if eng.status() != 0:
        raise RuntimeError(f"{wl.name}: device status flags raised during warm-up")

    vs = valid_sizes(wl)
    cnt = eng.kv_cnt.cpu().numpy()
    idx = eng.kv_idx.cpu().numpy()
    F = kept_flops(wl, cnt, idx, vs)
    nb = eng.nb
    U = wl.B * wl.H * nb
    paired = wl.block[0] * wl.block[1] * wl.block[2] == 64
    tc_scores = nb >= 320
    dense_F = 4 * wl.D * wl.B * wl.H * wl.N * wl.N
    route_bytes = 2 * wl.B * wl.H * wl.N * wl.D * 2 + 4 * U + 4 * int(cnt.sum())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    clocks = ClockSampler(dev.index if dev.index is not None else 0) if headline else None
    if clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for s in range(steps):
        if fl is not None:
            fl.fill_(s & 0xFF)
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    total_ms = t_begin.elapsed_time(t_end)
    route_ms = statistics.median([e[0].elapsed_time(e[1]) for e in evs])
    sched_ms = statistics.median([e[1].elapsed_time(e[2]) for e in evs])
    attn_ms = statistics.median([e[2].elapsed_time(e[3]) for e in evs])
    step_ms = statistics.median([e[0].elapsed_time(e[3]) for e in evs])
    attn_tflops = F / (attn_ms * 1e-3) / 1e12

    # dense mode of the same kernel and the CTA imbalance (outside the timed region)
    dense_out = torch.empty_like(q)
    eng.dense(q, k, v, dense_out)
    dn = []
    for _ in range(3):
        if fl is not None:
            fl.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        eng.dense(q, k, v, dense_out)
        b.record(stream)
        torch.cuda.synchronize()
        dn.append(a.elapsed_time(b))
    dense_ms = statistics.median(dn)
    del dense_out
    eng.attend(q, k, v, out, timing=True)
    torch.cuda.synchronize()
    cta_ns = eng.cta_ns.cpu().numpy().astype(np.float64)
    cta_cost = eng.cta_cost.cpu().numpy().astype(np.float64)
    busy = cta_cost > 0
    imb_pred = float(cta_cost[busy].max() / cta_cost[busy].mean()) if busy.any() else 1.0
    imb_meas = float(cta_ns[busy].max() / cta_ns[busy].mean()) if busy.any() else 1.0
    status = eng.status()

    hbm = pk["hbm_gbs"]
    peak_tf = pk["bf16_tflops"]
    fields = {
        "workload": workload_desc(wl),
        "value": F / (step_ms * 1e-3) / 1e12,
        "ms_per_step": step_ms,
        "attn_tflops_kept": attn_tflops,
        "attn_frac_of_bf16_peak": attn_tflops / peak_tf,
        "attn_frac_of_bf16_sustained": attn_tflops / pk.get("bf16_tflops_sustained", peak_tf),
        "sparse_attn_ms": attn_ms, "dense_attn_ms": dense_ms, "sparse_over_dense": attn_ms / dense_ms,
        "step_over_dense": step_ms / dense_ms, "dense_tflops": dense_F / (dense_ms * 1e-3) / 1e12,
        "route_ms": route_ms, "route_gbs": route_bytes / (route_ms * 1e-3) / 1e9,
        "route_frac_of_hbm": route_bytes / (route_ms * 1e-3) / 1e9 / hbm,
        "sched_us": sched_ms * 1e3,
        "imbalance_pred": imb_pred, "imbalance_meas": imb_meas,
        "density_kept_flops": F / dense_F, "kept_flops_per_step": F, "device_status": status,
        "l2": (f"{fl.numel() / 1e6:.0f} MB written between steps (outside the events)" if fl is not None else
               f"inputs {3 * q.numel() * q.element_size() / 1e6:.0f} MB per step > L2, no flush"),
        "steps": steps, "timing": "median of per-step CUDA events on the launching stream",
    }
    if rank == 0 and not args.no_parity:
        fields["route_parity"] = route_parity(wl, q, k, cnt, idx)
    launches = 5 + int(paired) + int(tc_scores)
    return fields, total_ms, F, eng, (q, k, v, out), clk, launches, seed


def head_split_emulated(wl, q, k, v, dev, worlds, reps=3):
    """The layer's heads split over W ranks emulated one after another on this
    GPU (heads.step_emulated): the static shards, the RLB migration plan, and
    RLB plus slack augmentation. Per mode: predicted rank loads (token pairs),
    each rank's attention time (median of `reps` CUDA-event timings; a rank's
    heads run alone on the whole GPU, so its time tracks its load) and their
    max/mean, and the augmentation's additions."""
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    from block_sparse_attention_fvattn_b200 import heads
    H = wl.B * wl.H
    geo1 = fa.Geometry(1, 1, wl.D, wl.grid, wl.block, dtype=q.dtype)
    be = heads.GpuBackend(geo1, wl.p, wl.k_min, dev)
    qf, kf, vf = (t.reshape(H, wl.N, wl.D) for t in (q, k, v))
    stream = torch.cuda.current_stream()
    out = {}
    for W in worlds:
        if W > H or W < 2:
            continue
        states = [heads.RankState(r, W, H, be) for r in range(W)]
        entry = {}
        for mode in ("static", "rlb", "rlb_sasa"):
            for st in states:
                st.balance = mode != "static"
                st.sasa = mode == "rlb_sasa"
            times = [[] for _ in range(W)]
            plan = None
            for rep in range(reps + 1):
                for st in states:
                    for name, t in (("q", qf), ("k", kf), ("v", vf)):
                        st.buf[name][:st.S].copy_(t[st.h0:st.h1])
                evs = {}

                def timer(r, fn):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    fn()
                    b.record(stream)
                    evs[r] = (a, b)
                plan = heads.step_emulated(states, timer)
                torch.cuda.synchronize()
                if rep > 0:
                    for r, (a, b) in evs.items():
                        times[r].append(a.elapsed_time(b))
            ms = [statistics.median(t) for t in times]
            loads = plan.load_after
            e = {"rank_load_pairs": loads, "pred_imbalance": max(loads) / (sum(loads) / W),
                 "rank_attn_ms": ms, "meas_imbalance": max(ms) / (sum(ms) / W), "critical_attn_ms": max(ms),
                 "moves": sum(a != b for a, b in zip(plan.owner_in, plan.owner_out))}
            if mode == "rlb_sasa":
                e["added_pairs"] = sum(int(st.added_pairs.item()) for st in states)
                e["added_mass"] = sum(float(st.added_mass.item()) for st in states)
            entry[mode] = e
        out[str(W)] = entry
        del states
        torch.cuda.empty_cache()
    return out


def head_split_distributed(args, wl, world, rank, dev):
    """The layer's heads split over the torchrun ranks (strong scaling): every
    rank draws the same layer, keeps its static shard and runs
    heads.step_distributed (NCCL all-gather of the head costs, point-to-point
    migration). Timed over the whole step, max over ranks."""
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    from block_sparse_attention_fvattn_b200 import heads
    H = wl.B * wl.H
    q, k, v = gen.make_inputs(wl, dev, seed=wl.seed)
    geo1 = fa.Geometry(1, 1, wl.D, wl.grid, wl.block, dtype=q.dtype)
    st = heads.RankState(rank, world, H, heads.GpuBackend(geo1, wl.p, wl.k_min, dev), sasa=args.split_sasa)
    qf, kf, vf = (t.reshape(H, wl.N, wl.D)[st.h0:st.h1] for t in (q, k, v))
    comm = heads.TorchComm()
    stream = torch.cuda.current_stream()
    ms = []
    for s in range(args.warmup + args.steps):
        for name, t in (("q", qf), ("k", kf), ("v", vf)):
            st.buf[name][:st.S].copy_(t)
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        heads.step_distributed(st, comm)
        b.record(stream)
        torch.cuda.synchronize()
        if s >= args.warmup:
            ms.append(max_over_ranks(a.elapsed_time(b), world))
    plan = st.plan
    W = world
    return {"world": world, "ms_per_layer": statistics.median(ms), "sasa": bool(args.split_sasa),
            "pred_imbalance_static": max(plan.load_static) / (sum(plan.load_static) / W),
            "pred_imbalance_rlb": max(plan.load_after) / (sum(plan.load_after) / W),
            "moves": sum(a != b for a, b in zip(plan.owner_in, plan.owner_out))}


def run_gpu(args, wl, world, rank, local):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pk, pk_src = peaks()
    stream = torch.cuda.current_stream()
    fields, total_ms, F, eng, (q, k, v, out), clk, launches, seed = measure(
        args, wl, dev, rank, world, flush=use_flush(args, wl, dev, headline=True), steps=args.steps,
        warmup=args.warmup, pk=pk, headline=True)
    total_ms_max = max_over_ranks(total_ms, world)
    ms_per_step = total_ms_max / args.steps
    work_all = sum_over_ranks(float(F), world)
    value = work_all * args.steps / (total_ms_max * 1e-3) / 1e12

    # ---- the same step replayed as one CUDA graph (no per-kernel events inside)
    graph_ms = None
    if not args.no_graph:
        graph = eng.capture(q, k, v, out)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(a.elapsed_time(b), world) / args.steps
        del graph

    # ---- end to end through the public API with host buffers: HostPipeline
    # copies Q, K, V in and O out per group of heads, overlapped with the
    # compute of the neighbouring groups
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        pipe = fa.HostPipeline(eng.geo, wl.p, wl.k_min, groups=args.e2e_groups, device=dev, overlap_calls=True)
        n_e2e = max(2, min(args.steps, 10))
        pipe(hq, hk, hv, hout)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        pipe.restart()  # the first timed call's copies start after `a`
        for _ in range(n_e2e):
            pipe(hq, hk, hv, hout)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b), world) / n_e2e
        e2e = {"value": work_all / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
               "d2h_bytes_per_step": q.numel() * q.element_size(),
               "ms_per_step": e2e_ms, "head_groups": len(pipe.ranges), "overlap_calls": True}
        del pipe, hq, hk, hv, hout

    # ---- the layer's heads split over ranks: emulated on this GPU (N=1), or
    # over the torchrun ranks with --split
    split = None
    if world == 1 and not args.no_split:
        split = head_split_emulated(wl, q, k, v, dev, [int(x) for x in args.split_worlds.split(",") if x])
    elif world > 1 and args.split:
        split = head_split_distributed(args, wl, world, rank, dev)

    # ---- CPU oracle baseline (rank 0, N=1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        hq, hk, hv = q.cpu(), k.cpu(), v.cpu()
        val, desc, cores, _ = oracle_sample(wl, hq, hk, hv, args.cpu_budget)
        cpu = {"value": val / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        del hq, hk, hv
    del eng, q, k, v, out
    torch.cuda.empty_cache()

    # ---- the other workloads: compact results in the same line (rank 0 only
    # prints; each rank measures its own replica, N=1 only by default)
    others = {}
    extra = [] if (args.no_extra or world > 1) else [n for n in gen.WORKLOAD_ORDER if n != wl.name]
    for name in extra:
        w2 = gen.WORKLOADS[name]
        f2, _, _, e2, ts, _, _, _ = measure(args, w2, dev, rank, world, flush=use_flush(args, w2, dev, headline=False),
                                            steps=min(args.steps, 10), warmup=3, pk=pk, headline=False)
        others[name] = f2
        del e2, ts
        torch.cuda.empty_cache()

    peak_tf = pk["bf16_tflops"]
    attn_tflops = fields["attn_tflops_kept"]
    traffic = recorded_traffic(wl.name)
    paired = wl.block[0] * wl.block[1] * wl.block[2] == 64
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": workload_desc(wl), "parallelism": f"replicas x{world} (heads shard, no exchange)",
                   "l2": fields["l2"], "seed": seed, "num_ctas": fa.default_num_ctas()},
    }
    line.update({k2: v2 for k2, v2 in fields.items() if k2 not in ("workload", "value", "ms_per_step", "l2",
                                                                    "steps")})
    line.update({
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak_tf, "traffic": traffic,
                     "kernel": f"attn_kernel<{wl.D},128,{'paired' if paired else 'unpaired'}> (fvattn_sparse_attn)",
                     "peak_source": f"{pk_src} bf16 burst" + ("" if pk_src == "measured" else " (fallback)")
                     + (" x 1 (fp16 has the bf16 dense rate)" if args.dtype == "f16" else "")},
        "route_roofline": {"bound": "hbm", "achieved": fields["route_gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": fields["route_frac_of_hbm"]},
        "clocks": clk,
        "graph_ms_per_step": graph_ms,
        "gpu_launches": launches * args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "other_workloads": others or None,
        "head_split": split,
    })
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_393k", choices=sorted(gen.WORKLOADS),
                    help="headline workload (default: the largest, the 393k-token layer)")
    ap.add_argument("--no-extra", action="store_true", help="skip the compact lines of the other workloads")
    ap.add_argument("--no-parity", action="store_true", help="skip the oracle check of the routing lists")
    ap.add_argument("--no-split", action="store_true", help="skip the emulated head split (N=1)")
    ap.add_argument("--split-worlds", default="2,4,8", help="rank counts of the emulated head split")
    ap.add_argument("--split", action="store_true", help="N>1: also time the head split over the ranks")
    ap.add_argument("--split-sasa", action="store_true", help="with --split: slack augmentation on")
    ap.add_argument("--impl", default="fvattn", choices=["fvattn", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle attention work")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16"], help="element type of Q, K, V and O")
    ap.add_argument("--e2e-groups", type=int, default=12, help="head groups of the host-buffer pipeline")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--flush", default="auto", choices=["auto", "always", "never"],
                    help="L2 flush between timed steps (auto: only when a step's inputs fit in L2)")
    ap.add_argument("--heads", type=int, default=0,
                    help="keep only the first H heads of the workload (same grid, blocks and input recipe): "
                         "a slice small enough for a multi-pass ncu capture of a large layer")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = gen.WORKLOADS[args.workload]
    if args.heads:
        if not 0 < args.heads <= wl.H:
            ap.error(f"--heads must be in [1, {wl.H}]")
        wl = dataclasses.replace(wl, H=args.heads, name=f"{wl.name}_{args.heads}heads")
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        else:
            run_gpu(args, wl, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
