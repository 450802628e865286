"""Thin ctypes binding of the C-ABI library `libfvattn.so` (include/fvattn.h).

Every function here only checks and marshals arguments (torch tensors ->
device pointers, the current CUDA stream) and calls the library; all
computation runs in the library's CUDA kernels. Importing this module loads
the library and raises if it is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfvattn.so")

OK, INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA_ERR, NONFINITE, TIMEOUT = range(7)
FLAG_NONFINITE, FLAG_TIMEOUT, FLAG_BAD_WORK = 0x1, 0x2, 0x4


class FVAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


DTYPE_BF16, DTYPE_F16 = 0, 1
_DTYPES = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}


class Problem(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "N", "D", "grid_t", "grid_h", "grid_w",
                                              "blk_t", "blk_h", "blk_w")] + [("softmax_scale", ctypes.c_float),
                                                                             ("dtype", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m block_sparse_attention_fvattn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    P = ctypes.POINTER(Problem)
    sig = {
        "fvattn_num_blocks": (i32, [P]),
        "fvattn_default_num_ctas": (i32, []),
        "fvattn_workspace_size": (sz, [P, i32]),
        "fvattn_workspace_init": (i32, [vp, sz, vp]),
        "fvattn_route": (i32, [P, vp, vp, f32, i32, vp, vp, vp, vp, sz, vp]),
        "fvattn_route_noalloc": (i32, [P, vp, vp, f32, i32, vp, vp, vp, vp]),
        "fvattn_schedule": (i32, [P, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]),
        "fvattn_sparse_attn": (i32, [P, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, sz, vp]),
        "fvattn_read_device_status": (i32, [vp, vp, ctypes.POINTER(ctypes.c_uint32)]),
        "fvattn_head_cost": (i32, [P, vp, vp, i32, vp, vp]),
        "fvattn_rlb_plan": (i32, [vp, i32, i32, vp, i32, vp, vp]),
        "fvattn_lpt_assign": (i32, [vp, i32, i32, vp, vp]),
        "fvattn_augment": (i32, [P, vp, ctypes.c_int64, vp, vp, vp, vp, vp, sz, vp]),
        "fvattn_set_wait_limit": (i32, [vp, sz, ctypes.c_uint64, vp]),
        "fvattn_test_withhold_unit": (i32, [vp, sz, i32, vp]),
        "fvattn_status_string": (ctypes.c_char_p, [i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("fvattn_num_blocks", "fvattn_default_num_ctas", "fvattn_workspace_size", "fvattn_workspace_init",
            "fvattn_route", "fvattn_route_noalloc", "fvattn_schedule", "fvattn_sparse_attn", "fvattn_read_device_status",
            "fvattn_status_string", "fvattn_head_cost", "fvattn_rlb_plan", "fvattn_lpt_assign", "fvattn_augment",
            "fvattn_set_wait_limit", "fvattn_test_withhold_unit")


def status_string(s: int) -> str:
    return _lib.fvattn_status_string(int(s)).decode()


@dataclass(frozen=True)
class Geometry:
    B: int
    H: int
    D: int
    grid: Tuple[int, int, int]
    block: Tuple[int, int, int]
    softmax_scale: float = 0.0   # <= 0 selects 1/sqrt(D)
    dtype: torch.dtype = torch.bfloat16  # element type of Q, K, V, O: bfloat16 or float16

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    def problem(self) -> Problem:
        T, Hg, W = self.grid
        bt, bh, bw = self.block
        if self.dtype not in _DTYPES:
            raise ValueError(f"unsupported element type {self.dtype}; use torch.bfloat16 or torch.float16")
        return Problem(self.B, self.H, self.N, self.D, T, Hg, W, bt, bh, bw, float(self.softmax_scale),
                       _DTYPES[self.dtype])

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / math.sqrt(self.D)


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _check(st: int, where: str):
    if st != OK:
        raise FVAttnError(st, where)


def num_blocks(geo: Geometry) -> int:
    p = geo.problem()
    return int(_lib.fvattn_num_blocks(ctypes.byref(p)))


def default_num_ctas() -> int:
    return int(_lib.fvattn_default_num_ctas())


def workspace_size(geo: Geometry, num_ctas: int = 0) -> int:
    p = geo.problem()
    return int(_lib.fvattn_workspace_size(ctypes.byref(p), int(num_ctas)))


def workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.fvattn_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)),
           "fvattn_workspace_init")


def route(geo: Geometry, q: torch.Tensor, k: torch.Tensor, p: float, k_min: int,
          kv_cnt: torch.Tensor, kv_idx: torch.Tensor, ws: torch.Tensor,
          block_probs: Optional[torch.Tensor] = None, stream=None):
    prob = geo.problem()
    st = _lib.fvattn_route(ctypes.byref(prob), _ptr(q, geo.dtype, "q"), _ptr(k, geo.dtype, "k"),
                           float(p), int(k_min), _ptr(kv_cnt, torch.int32, "kv_cnt"),
                           _ptr(kv_idx, torch.int32, "kv_idx"), _ptr(block_probs, torch.float32, "block_probs"),
                           _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "fvattn_route")


def route_noalloc(geo: Geometry, q: torch.Tensor, k: torch.Tensor, p: float, k_min: int,
                  kv_cnt: torch.Tensor, kv_idx: torch.Tensor, block_probs: Optional[torch.Tensor] = None,
                  stream=None):
    """fvattn_route without a workspace, for callers that cannot allocate device
    memory: the library's own fixed 16 MiB per-device array holds the scratch.
    Calls that may overlap on the GPU race on that array; order them on one
    stream, and make the first call on a device before any stream capture."""
    prob = geo.problem()
    st = _lib.fvattn_route_noalloc(ctypes.byref(prob), _ptr(q, geo.dtype, "q"), _ptr(k, geo.dtype, "k"),
                                   float(p), int(k_min), _ptr(kv_cnt, torch.int32, "kv_cnt"),
                                   _ptr(kv_idx, torch.int32, "kv_idx"),
                                   _ptr(block_probs, torch.float32, "block_probs"), _stream(stream))
    _check(st, "fvattn_route_noalloc")


def schedule(geo: Geometry, kv_cnt: Optional[torch.Tensor], kv_idx: Optional[torch.Tensor], dense: bool,
             num_ctas: int, work: torch.Tensor, cta_range: torch.Tensor, ws: torch.Tensor,
             cta_cost: Optional[torch.Tensor] = None, stream=None):
    prob = geo.problem()
    st = _lib.fvattn_schedule(ctypes.byref(prob), _ptr(kv_cnt, torch.int32, "kv_cnt"),
                              _ptr(kv_idx, torch.int32, "kv_idx"), int(bool(dense)), int(num_ctas),
                              _ptr(work, torch.int32, "work"), _ptr(cta_range, torch.int32, "cta_range"),
                              _ptr(cta_cost, torch.int64, "cta_cost"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                              _stream(stream))
    _check(st, "fvattn_schedule")


def sparse_attn(geo: Geometry, q, k, v, kv_cnt, kv_idx, work, cta_range, num_ctas: int, dense: bool,
                out: torch.Tensor, ws: torch.Tensor, cta_ns: Optional[torch.Tensor] = None, stream=None):
    prob = geo.problem()
    st = _lib.fvattn_sparse_attn(ctypes.byref(prob), _ptr(q, geo.dtype, "q"), _ptr(k, geo.dtype, "k"),
                                 _ptr(v, geo.dtype, "v"), _ptr(kv_cnt, torch.int32, "kv_cnt"),
                                 _ptr(kv_idx, torch.int32, "kv_idx"), _ptr(work, torch.int32, "work"),
                                 _ptr(cta_range, torch.int32, "cta_range"), int(num_ctas), int(bool(dense)),
                                 _ptr(out, geo.dtype, "out"), _ptr(cta_ns, torch.int64, "cta_ns"),
                                 _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream))
    _check(st, "fvattn_sparse_attn")


def head_cost(geo: Geometry, kv_cnt: Optional[torch.Tensor], kv_idx: Optional[torch.Tensor], out: torch.Tensor,
              dense: bool = False, stream=None):
    """out[b*H + h] (int64) = valid (query, key) token pairs of head (b, h) under its kept lists."""
    prob = geo.problem()
    st = _lib.fvattn_head_cost(ctypes.byref(prob), _ptr(kv_cnt, torch.int32, "kv_cnt"),
                               _ptr(kv_idx, torch.int32, "kv_idx"), int(bool(dense)), _ptr(out, torch.int64, "out"),
                               _stream(stream))
    _check(st, "fvattn_head_cost")


def rlb_plan(head_cost_host, world: int, owner_in=None, max_moves: int = 1):
    """Head migration plan (host): returns (owner_out, rank_load) as int lists.
    head_cost_host: sequence of int64 costs; owner_in: None for the static shards."""
    n = len(head_cost_host)
    costs = (ctypes.c_int64 * max(n, 1))(*[int(c) for c in head_cost_host])
    own_in = None if owner_in is None else (ctypes.c_int32 * max(n, 1))(*[int(o) for o in owner_in])
    own_out = (ctypes.c_int32 * max(n, 1))()
    load = (ctypes.c_int64 * max(int(world), 1))()
    st = _lib.fvattn_rlb_plan(costs, int(n), int(world), own_in, int(max_moves), own_out, load)
    _check(st, "fvattn_rlb_plan")
    return [int(own_out[h]) for h in range(n)], [int(load[r]) for r in range(int(world))]


def lpt_assign(head_cost_host, world: int):
    """Longest-processing-time assignment of heads to ranks (host): (owner, rank_load)."""
    n = len(head_cost_host)
    costs = (ctypes.c_int64 * max(n, 1))(*[int(c) for c in head_cost_host])
    own_out = (ctypes.c_int32 * max(n, 1))()
    load = (ctypes.c_int64 * max(int(world), 1))()
    _check(_lib.fvattn_lpt_assign(costs, int(n), int(world), own_out, load), "fvattn_lpt_assign")
    return [int(own_out[h]) for h in range(n)], [int(load[r]) for r in range(int(world))]


def augment(geo: Geometry, block_probs: torch.Tensor, budget: int, kv_cnt: torch.Tensor, kv_idx: torch.Tensor,
            ws: torch.Tensor, added_pairs: Optional[torch.Tensor] = None, added_mass: Optional[torch.Tensor] = None,
            stream=None):
    """Add the highest-probability unkept blocks to the lists, within `budget` token pairs (in place)."""
    prob = geo.problem()
    st = _lib.fvattn_augment(ctypes.byref(prob), _ptr(block_probs, torch.float32, "block_probs"), int(budget),
                             _ptr(kv_cnt, torch.int32, "kv_cnt"), _ptr(kv_idx, torch.int32, "kv_idx"),
                             _ptr(added_pairs, torch.int64, "added_pairs"),
                             _ptr(added_mass, torch.float64, "added_mass"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
                             _stream(stream))
    _check(st, "fvattn_augment")


def set_wait_limit(ws: torch.Tensor, limit_ns: int, stream=None):
    """Time limit (ns) of every wait inside the kernels of later calls on `ws` (0: default 2 s)."""
    _check(_lib.fvattn_set_wait_limit(_ptr(ws, torch.uint8, "ws"), ws.numel(), int(limit_ns), _stream(stream)),
           "fvattn_set_wait_limit")


def test_withhold_unit(ws: torch.Tensor, rank: int, stream=None):
    """Failure-path test hook: the next attention call on `ws` withholds unit rank `rank` (-1: off)."""
    _check(_lib.fvattn_test_withhold_unit(_ptr(ws, torch.uint8, "ws"), ws.numel(), int(rank), _stream(stream)),
           "fvattn_test_withhold_unit")


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check(_lib.fvattn_read_device_status(_ptr(ws, torch.uint8, "ws"), _stream(stream), ctypes.byref(flags)),
           "fvattn_read_device_status")
    return int(flags.value)


class FVAttn:
    """The whole path for one problem: route -> schedule -> block-sparse attention.

    Buffers (lists, schedule, workspace) are allocated once through torch and
    reused; `__call__` enqueues the three library calls on the current stream.
    """

    def __init__(self, geo: Geometry, p: float, k_min: int, device="cuda", num_ctas: int = 0,
                 with_probs: bool = False):
        self.geo, self.p, self.k_min = geo, float(p), int(k_min)
        self.nb = num_blocks(geo)
        if self.nb < 0:
            raise FVAttnError(INVALID_ARG, "FVAttn")
        self.num_ctas = num_ctas if num_ctas > 0 else default_num_ctas()
        dev = torch.device(device)
        B, H, nb = geo.B, geo.H, self.nb
        self.kv_cnt = torch.zeros((B, H, nb), dtype=torch.int32, device=dev)
        self.kv_idx = torch.zeros((B, H, nb, nb), dtype=torch.int32, device=dev)
        self.block_probs = torch.zeros((B, H, nb, nb), dtype=torch.float32, device=dev) if with_probs else None
        self.work = torch.zeros(B * H * nb, dtype=torch.int32, device=dev)
        self.cta_range = torch.zeros(self.num_ctas + 1, dtype=torch.int32, device=dev)
        self.cta_cost = torch.zeros(self.num_ctas, dtype=torch.int64, device=dev)
        self.cta_ns = torch.zeros(self.num_ctas, dtype=torch.int64, device=dev)
        self.dense_work = torch.zeros_like(self.work)
        self.dense_range = torch.zeros_like(self.cta_range)
        self.ws = torch.zeros(max(workspace_size(geo, self.num_ctas), 256), dtype=torch.uint8, device=dev)
        workspace_init(self.ws)
        self._dense_scheduled = False

    def route(self, q, k, stream=None):
        route(self.geo, q, k, self.p, self.k_min, self.kv_cnt, self.kv_idx, self.ws, self.block_probs, stream)

    def schedule(self, stream=None):
        schedule(self.geo, self.kv_cnt, self.kv_idx, False, self.num_ctas, self.work, self.cta_range, self.ws,
                 self.cta_cost, stream)

    def attend(self, q, k, v, out, stream=None, timing=False):
        sparse_attn(self.geo, q, k, v, self.kv_cnt, self.kv_idx, self.work, self.cta_range, self.num_ctas,
                    False, out, self.ws, self.cta_ns if timing else None, stream)

    def dense(self, q, k, v, out, stream=None, timing=False):
        if not self._dense_scheduled:
            schedule(self.geo, None, None, True, self.num_ctas, self.dense_work, self.dense_range, self.ws,
                     None, stream)
            self._dense_scheduled = True
        sparse_attn(self.geo, q, k, v, None, None, self.dense_work, self.dense_range, self.num_ctas, True, out,
                    self.ws, self.cta_ns if timing else None, stream)

    def __call__(self, q, k, v, out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        self.route(q, k, stream)
        self.schedule(stream)
        self.attend(q, k, v, out, stream)
        return out

    def status(self, stream=None) -> int:
        return read_device_status(self.ws, stream)

    def capture(self, q, k, v, out) -> torch.cuda.CUDAGraph:
        """Record route -> schedule -> attention on fixed q, k, v, out as one CUDA
        graph; `graph.replay()` then runs the whole step with one launch call.
        The kernels' programmatic launch dependencies become graph edges, and
        the counters they share through the workspace reset themselves, so
        the graph can be replayed any number of times."""
        self(q, k, v, out)  # first use outside the capture: attributes and tensor-map encoder
        torch.cuda.synchronize(q.device)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=q.device)
        side.wait_stream(torch.cuda.current_stream(q.device))
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                self(q, k, v, out)
        torch.cuda.current_stream(q.device).wait_stream(side)
        return graph


class HostPipeline:
    """The whole path on host-resident (pinned) Q, K, V, O, with the
    host<->device copies overlapped with the compute.

    Heads are independent all along the path, so the B*H heads are split into
    `groups` contiguous ranges, each run as its own problem (B=1, H=its heads)
    through the same three library calls. Group c+1 is copied in on one stream
    while group c computes on the caller's stream and group c-1 is copied out
    on a third, so a call takes about the host->device copy time plus one
    group's compute and copy-out. The result is the same as FVAttn on the
    whole problem (every head is routed, scheduled and attended alone).

    overlap_calls: by default a call's copies in start only after all work
    enqueued before it on the current stream, which includes the previous
    call's last compute and copy-out. With overlap_calls, a call's copy of head
    group c waits only for the previous call's compute of group c (the reader
    of those device buffers), so consecutive calls keep the host->device
    link busy. The host inputs must then be ready when the call is made: no
    work still pending on a stream may be writing them.
    """

    def __init__(self, geo: Geometry, p: float, k_min: int, groups: int = 4, device="cuda", num_ctas: int = 0,
                 overlap_calls: bool = False):
        BH = geo.B * geo.H
        groups = max(1, min(int(groups), BH))
        self.geo, self.dev = geo, torch.device(device)
        self.ranges = [(BH * c // groups, BH * (c + 1) // groups) for c in range(groups)]
        self.engines = [FVAttn(Geometry(1, h1 - h0, geo.D, geo.grid, geo.block, geo.softmax_scale, geo.dtype),
                               p, k_min, device=device, num_ctas=num_ctas) for h0, h1 in self.ranges]
        shape = (BH, geo.N, geo.D)
        self.dq, self.dk, self.dv, self.dout = (torch.empty(shape, dtype=geo.dtype, device=self.dev) for _ in range(4))
        self.s_in = torch.cuda.Stream(device=self.dev)
        self.s_out = torch.cuda.Stream(device=self.dev)
        self.overlap_calls = bool(overlap_calls)
        self._prev_done = None  # the previous call's compute events, per group

    def __call__(self, hq: torch.Tensor, hk: torch.Tensor, hv: torch.Tensor, hout: torch.Tensor):
        """hq, hk, hv, hout: pinned host tensors [B, H, N, D] of the problem's dtype.
        Enqueued on the current stream; returns without waiting, like the
        library calls (synchronise before reading hout)."""
        for t, name in ((hq, "q"), (hk, "k"), (hv, "v"), (hout, "out")):
            if t.is_cuda or not t.is_pinned():
                raise ValueError(f"{name} must be a pinned host tensor")
            if t.dtype != self.geo.dtype or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous {self.geo.dtype} tensor")
            if tuple(t.shape) != (self.geo.B, self.geo.H, self.geo.N, self.geo.D):
                raise ValueError(f"{name} has shape {tuple(t.shape)}")
        BH = self.geo.B * self.geo.H
        views = [t.view(BH, self.geo.N, self.geo.D) for t in (hq, hk, hv, hout)]
        compute = torch.cuda.current_stream(self.dev)
        prev = self._prev_done if self.overlap_calls else None
        if prev is None:
            self.s_in.wait_stream(compute)   # the device buffers are free once earlier work is done
        self.s_out.wait_stream(compute)
        copied, done = [], []
        for c, (h0, h1) in enumerate(self.ranges):
            with torch.cuda.stream(self.s_in):
                if prev is not None:
                    # the previous call's compute of this group has read its inputs
                    self.s_in.wait_event(prev[c])
                for dst, src in zip((self.dq, self.dk, self.dv), views[:3]):
                    dst[h0:h1].copy_(src[h0:h1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_in)
                copied.append(ev)
        for (h0, h1), eng, ev in zip(self.ranges, self.engines, copied):
            compute.wait_event(ev)
            eng(self.dq[h0:h1], self.dk[h0:h1], self.dv[h0:h1], out=self.dout[h0:h1])
            d = torch.cuda.Event()
            d.record(compute)
            done.append(d)
        for (h0, h1), d in zip(self.ranges, done):
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(d)
                views[3][h0:h1].copy_(self.dout[h0:h1], non_blocking=True)
        compute.wait_stream(self.s_out)
        self._prev_done = done
        return hout

    def restart(self):
        """Make the next call wait for all work enqueued before it on the
        current stream, as the first call does (overlap_calls only)."""
        self._prev_done = None

    def status(self) -> int:
        flags = 0
        for eng in self.engines:
            flags |= eng.status()
        return flags
