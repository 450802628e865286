"""fp64 CPU oracle of the adaptive block-sparse attention path -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package. It shares no code with the CUDA library: the arithmetic
lives in `fvattn_oracle.c` (plain C, fp64, OpenMP over independent items), and
this module only compiles it with gcc and marshals numpy arrays through ctypes.

Functions follow the steps written at the top of `fvattn_oracle.c`:
pooling, block scores, softmax, Top-p with a Top-k floor, diagonal/non-finite
repair, ascending kept lists, and masked softmax attention for chosen query
tokens; and the slack augmentation of the lists (oracle_augment). Which parts are pinned to something other than the oracle itself is
listed in the test module `tests/test_oracle_pins.py`; the score temperature
(scale = 1/sqrt(D) for routing) and the synthetic-input recipe are readings
with no printed value to pin against ("parity unpinned" for those choices).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fvattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


class Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "T", "Hg", "W", "D", "bt", "bh", "bw", "fp16")]


def compile_oracle(src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle source into a shared library with gcc (-O2, OpenMP)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_oracle()
    return _LIB


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_u16(x) -> np.ndarray:
    """bf16 or fp16 tensor/array -> contiguous uint16 view of the raw bits (no rounding)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype in (torch.bfloat16, torch.float16)
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, lib_path: Optional[str] = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        L = self.lib
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
        L.oracle_num_blocks.argtypes = [ctypes.POINTER(Geom)]
        L.oracle_num_blocks.restype = i32
        L.oracle_block_sizes.argtypes = [ctypes.POINTER(Geom), vp]
        L.oracle_pool.argtypes = [ctypes.POINTER(Geom), vp, vp]
        L.oracle_widen.argtypes = [i32, vp, vp, ctypes.c_int64]
        L.oracle_route.argtypes = [ctypes.POINTER(Geom), vp, vp, f64, f64, i32, vp, vp, vp, vp, vp, vp]
        L.oracle_attn_rows.argtypes = [ctypes.POINTER(Geom), vp, vp, vp, f64, vp, vp,
                                       ctypes.c_int64, vp, vp, vp, vp, vp]
        L.oracle_augment.argtypes = [ctypes.POINTER(Geom), vp, ctypes.c_int64, vp, vp, vp, vp]

    @staticmethod
    def geom(B, H, grid, block, D, fp16=False) -> Geom:
        T, Hg, W = grid
        bt, bh, bw = block
        return Geom(B, H, T, Hg, W, D, bt, bh, bw, 1 if fp16 else 0)

    def widen(self, bits: np.ndarray, fp16: bool) -> np.ndarray:
        """The oracle's exact decode of raw 16-bit elements to fp64."""
        b = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.zeros(b.size, dtype=np.float64)
        self.lib.oracle_widen(ctypes.c_int32(1 if fp16 else 0), _ptr(b), _ptr(out), ctypes.c_int64(b.size))
        return out

    def num_blocks(self, g: Geom) -> int:
        return int(self.lib.oracle_num_blocks(ctypes.byref(g)))

    def block_sizes(self, g: Geom) -> np.ndarray:
        out = np.zeros(self.num_blocks(g), dtype=np.int32)
        self.lib.oracle_block_sizes(ctypes.byref(g), _ptr(out))
        return out

    def pool(self, g: Geom, x) -> np.ndarray:
        xu = _as_u16(x)
        nb = self.num_blocks(g)
        out = np.zeros((g.B, g.H, nb, g.D), dtype=np.float64)
        self.lib.oracle_pool(ctypes.byref(g), _ptr(xu), _ptr(out))
        return out

    def route(self, g: Geom, qbar: np.ndarray, kbar: np.ndarray, scale: float, p: float, k_min: int,
              want_detail: bool = True):
        """Returns dict(kv_cnt, kv_idx, probs, order, cum, nonfinite) as numpy arrays."""
        nb = self.num_blocks(g)
        qb = np.ascontiguousarray(qbar, dtype=np.float64)
        kb = np.ascontiguousarray(kbar, dtype=np.float64)
        cnt = np.zeros((g.B, g.H, nb), dtype=np.int32)
        idx = np.full((g.B, g.H, nb, nb), -1, dtype=np.int32)
        probs = order = cum = None
        if want_detail:
            probs = np.zeros((g.B, g.H, nb, nb), dtype=np.float64)
            order = np.zeros((g.B, g.H, nb, nb), dtype=np.int32)
            cum = np.zeros((g.B, g.H, nb, nb), dtype=np.float64)
        nonf = np.zeros((g.B, g.H, nb), dtype=np.uint8)
        self.lib.oracle_route(ctypes.byref(g), _ptr(qb), _ptr(kb), float(scale), float(p), int(k_min),
                              _ptr(cnt), _ptr(idx), _ptr(probs), _ptr(order), _ptr(cum), _ptr(nonf))
        return dict(kv_cnt=cnt, kv_idx=idx, probs=probs, order=order, cum=cum, nonfinite=nonf)

    def augment(self, g: Geom, probs: np.ndarray, budget: int, kv_cnt: np.ndarray, kv_idx: np.ndarray):
        """Slack augmentation of copies of the lists within `budget` token pairs.
        Returns (kv_cnt, kv_idx, added_pairs, added_mass)."""
        pr = np.ascontiguousarray(probs, dtype=np.float64)
        cnt = np.ascontiguousarray(kv_cnt, dtype=np.int32).copy()
        idx = np.ascontiguousarray(kv_idx, dtype=np.int32).copy()
        pairs = ctypes.c_int64(0)
        mass = ctypes.c_double(0.0)
        self.lib.oracle_augment(ctypes.byref(g), _ptr(pr), ctypes.c_int64(int(budget)), _ptr(cnt), _ptr(idx),
                                ctypes.byref(pairs), ctypes.byref(mass))
        return cnt, idx, int(pairs.value), float(mass.value)

    def attn_rows(self, g: Geom, q, k, v, scale: float, rows: np.ndarray,
                  kv_cnt: Optional[np.ndarray] = None, kv_idx: Optional[np.ndarray] = None,
                  want_bounds: bool = False):
        """Attention output [len(rows), D] for flat query rows (b*H+h)*N+n.

        kv_cnt/kv_idx None means every block is kept (dense attention)."""
        qu, ku, vu = _as_u16(q), _as_u16(k), _as_u16(v)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        out = np.zeros((n, g.D), dtype=np.float64)
        ws = np.zeros(n, dtype=np.float64)
        lo = hi = None
        if want_bounds:
            lo = np.zeros((n, g.D), dtype=np.float64)
            hi = np.zeros((n, g.D), dtype=np.float64)
        c = None if kv_cnt is None else np.ascontiguousarray(kv_cnt, dtype=np.int32)
        ix = None if kv_idx is None else np.ascontiguousarray(kv_idx, dtype=np.int32)
        self.lib.oracle_attn_rows(ctypes.byref(g), _ptr(qu), _ptr(ku), _ptr(vu), float(scale),
                                  _ptr(c), _ptr(ix), ctypes.c_int64(n), _ptr(rows),
                                  _ptr(out), _ptr(ws), _ptr(lo), _ptr(hi))
        if want_bounds:
            return out, ws, lo, hi
        return out, ws


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
