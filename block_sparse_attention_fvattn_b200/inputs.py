"""Seeded synthetic inputs for the adaptive block-sparse attention path.

This module only draws tensors. It holds none of the method's arithmetic
(no pooling, scoring, selection or attention), so both the CUDA path and the
CPU oracle can be fed from it without sharing any of the computation.

The five workloads mirror the video-DiT layers the FVAttn pages evaluate on
(Wan2.2 I2V, step-distilled; ai-feeds.com summary, "Experiments") and the
FastVideo VSA block geometry (zskr.cn guide, section 1: (T,H,W) latent grid cut
into (4,8,8) = 256-token blocks; section 5: the 64-token (4,4,4) route). Real
activations need model weights that are not available, so the query/key
tensors are built from a smooth spatio-temporal field: neighbouring tokens get
correlated queries and keys, which gives locality-shaped block scores and a
per-head sparsity that ranges from near-dense to very sparse.

Recipe per (b, h), in this draw order on one torch.Generator:
  a_h (if drawn), S [D,T,Hg,W] ~ N(0,1), eps_q [N,D], eps_k [N,D], V [N,D].
  S is blurred by a separable Gaussian (same sigma along T, H and W, radius
  ceil(3 sigma), weights normalised to 1, mirror boundary) and renormalised to
  zero mean / unit variance per channel over the grid.
  Q = a_h * S + 0.5 * eps_q,  K = a_h * S + 0.5 * eps_k,  V ~ N(0,1).
  Everything is rounded to bf16 (round-to-nearest-even) at the end.
The tiny workload draws Q, K, V i.i.d. N(0,1) instead.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    grid: Tuple[int, int, int]          # (T, Hg, W) latent grid
    block: Tuple[int, int, int]         # (bt, bh, bw)
    p: float                            # Top-p threshold
    k_min: int                          # Top-k safety floor
    sigma: Optional[float] = None       # blur sigma in tokens; None -> i.i.d. inputs
    a_range: Optional[Tuple[float, float]] = None   # log-uniform a_h range
    a_fixed: Optional[Tuple[float, ...]] = None     # explicit a_h per head
    seed: int = 0

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (8, 16, 16), (4, 8, 8), 0.9, 2, seed=1001),
    "wan5b": Workload("wan5b", 1, 24, 128, (31, 22, 40), (4, 8, 8), 0.9, 8,
                      sigma=2.0, a_range=(0.5, 4.0), seed=1002),
    "wan14b_i2v_720p": Workload("wan14b_i2v_720p", 1, 40, 128, (21, 45, 80), (4, 8, 8), 0.9, 16,
                                sigma=2.0, a_range=(0.5, 4.0), seed=1003),
    "head_skew_64tok": Workload("head_skew_64tok", 1, 16, 128, (16, 32, 32), (4, 4, 4), 0.95, 4,
                                sigma=2.0, a_fixed=tuple([0.25] * 4 + [6.0] * 12), seed=1004),
    "long_393k": Workload("long_393k", 1, 12, 128, (96, 64, 64), (4, 8, 8), 0.85, 32,
                          sigma=3.0, a_range=(1.0, 4.0), seed=1005),
}
# Positional aliases in the order the workloads are listed.
WORKLOAD_ORDER = ["tiny", "wan5b", "wan14b_i2v_720p", "head_skew_64tok", "long_393k"]


def custom(name, B, H, D, grid, block, p, k_min, sigma=None, a_range=None, a_fixed=None, seed=7):
    """A workload of arbitrary shape built with the same recipe (tests use small ones)."""
    return Workload(name, B, H, D, tuple(grid), tuple(block), p, k_min, sigma, a_range, a_fixed, seed)


def _gauss_taps(sigma: float, device) -> torch.Tensor:
    r = int(math.ceil(3.0 * sigma))
    x = torch.arange(-r, r + 1, dtype=torch.float64)
    w = torch.exp(-(x * x) / (2.0 * sigma * sigma))
    return (w / w.sum()).to(torch.float32).to(device)


def _blur_axis(s: torch.Tensor, taps: torch.Tensor, axis: int) -> torch.Tensor:
    """Blur s [D, T, Hg, W] along one grid axis with mirror padding."""
    r = (taps.numel() - 1) // 2
    x = s.movedim(axis, -1)
    shp = x.shape
    x = x.reshape(-1, 1, shp[-1])
    n = shp[-1]
    if n == 1:
        return s
    # Mirror padding without repeating the edge; reflect as often as needed.
    idx = torch.arange(-r, n + r, device=s.device)
    period = 2 * (n - 1)
    idx = torch.remainder(idx, period)
    idx = torch.where(idx >= n, period - idx, idx)
    x = x[..., idx]
    x = torch.nn.functional.conv1d(x, taps.view(1, 1, -1))
    return x.reshape(shp).movedim(-1, axis)


def smooth_field(gen: torch.Generator, D: int, grid, sigma: float, device) -> torch.Tensor:
    """Blurred, per-channel renormalised N(0,1) field, returned as [N, D] fp32."""
    T, Hg, W = grid
    s = torch.randn((D, T, Hg, W), generator=gen, device=device, dtype=torch.float32)
    taps = _gauss_taps(sigma, device)
    for ax in (1, 2, 3):
        s = _blur_axis(s, taps, ax)
    flat = s.reshape(D, -1)
    mean = flat.mean(dim=1, keepdim=True)
    std = flat.std(dim=1, unbiased=False, keepdim=True).clamp_min(1e-12)
    flat = (flat - mean) / std
    return flat.t().contiguous()


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None,
                with_v: bool = True, return_a: bool = False):
    """Build Q, K, V as bf16 [B, H, N, D] on `device` from a seeded generator.

    The random stream depends on the device type (CPU and CUDA generators
    differ); callers that need the same tensors on both sides copy them.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed if seed is None else seed)
    B, H, D, N = wl.B, wl.H, wl.D, wl.N
    q = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=dev)
    k = torch.empty_like(q)
    v = torch.empty_like(q) if with_v else None
    a_all = []
    for b in range(B):
        for h in range(H):
            if wl.sigma is None:
                q[b, h] = torch.randn((N, D), generator=gen, device=dev).to(torch.bfloat16)
                k[b, h] = torch.randn((N, D), generator=gen, device=dev).to(torch.bfloat16)
                vv = torch.randn((N, D), generator=gen, device=dev)
                a_all.append(0.0)
            else:
                if wl.a_fixed is not None:
                    a = float(wl.a_fixed[h % len(wl.a_fixed)])
                else:
                    lo, hi = wl.a_range
                    u = torch.rand((1,), generator=gen, device=dev, dtype=torch.float64).item()
                    a = math.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
                a_all.append(a)
                S = smooth_field(gen, D, wl.grid, wl.sigma, dev)
                eq = torch.randn((N, D), generator=gen, device=dev)
                q[b, h] = (a * S + 0.5 * eq).to(torch.bfloat16)
                del eq
                ek = torch.randn((N, D), generator=gen, device=dev)
                k[b, h] = (a * S + 0.5 * ek).to(torch.bfloat16)
                del ek, S
                vv = torch.randn((N, D), generator=gen, device=dev)
            if with_v:
                v[b, h] = vv.to(torch.bfloat16)
            del vv
    if return_a:
        return q, k, v, a_all
    return q, k, v
