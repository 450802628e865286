"""Multi-rank host logic of bench.py on CPU with gloo (world size 2).

bench.py runs one process per GPU: timing is the max over ranks, work is
summed over ranks, and only rank 0 runs (and prints) the CPU oracle arm. No
GPU and no data-path collective is involved; the ranks are CPU processes.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t_max = bench.max_over_ranks(10.0 + rank, world)
        w_sum = bench.sum_over_ranks(100.0 * (rank + 1), world)
        bench.barrier(world)

        class A:
            steps, warmup, gpus = 1, 3, world
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(A, bench.gen.WORKLOADS["tiny"], world, rank)
        q.put((rank, t_max, w_sum, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_reference_arm():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, t_max, w_sum, text = q.get(timeout=300)
        out[rank] = (t_max, w_sum, text)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        assert out[rank][0] == 11.0          # max over ranks
        assert out[rank][1] == 300.0         # sum over ranks
    line = json.loads(out[0][2].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert out[1][2].strip() == ""           # only rank 0 runs the oracle arm
