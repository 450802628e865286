"""Shared helpers for the GPU parity tests and the benchmark's checks.

Inputs come from the seeded generator (`block_sparse_attention_fvattn_b200.inputs`),
are drawn on the GPU and copied to the host, so the CUDA path and the fp64
oracle see the same bf16 tensors. Nothing here computes any step of the method
itself except through the oracle (expected values) or the library (results).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from block_sparse_attention_fvattn_b200 import inputs as gen

# Tolerances stated by the target: attention output vs the oracle run on the
# GPU's own lists; Top-p boundary window for list differences.
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
TOPP_WINDOW = 1e-5
# Rounding-tie window for list differences at the rank boundary: the fp32
# pooled scores can differ from the fp64 ones by at most about
# (D + 2*256) * 2^-24 * scale * |Qbar_i| * |Kbar_j| (dot-product and pooled-sum
# error bounds; the three-product TF32 split used for long rows adds at most
# 3 * 2^-22 of the same scale), so two blocks whose oracle scores are closer
# than that may legitimately swap ranks.
TIE_FACTOR = 4e-5


def geometry(wl, dtype=torch.bfloat16):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    return fa.Geometry(wl.B, wl.H, wl.D, wl.grid, wl.block, dtype=dtype)


def make_on_gpu(wl, seed=None, dtype=torch.bfloat16):
    """The seeded bf16 inputs; for fp16 they are converted (through fp32)."""
    q, k, v = gen.make_inputs(wl, "cuda", seed=seed)
    if dtype != torch.bfloat16:
        q, k, v = (t.float().to(dtype) for t in (q, k, v))
    torch.cuda.synchronize()
    return q, k, v


@dataclass
class ListCompare:
    rows: int
    identical: int
    excused_topp: int
    excused_tie: int
    unexcused: int
    first_unexcused: object = None


def compare_lists(gpu_cnt, gpu_idx, orc, qbar, kbar, scale, p, k_min):
    """Compare GPU kept lists with the oracle's, row by row.

    A differing row is excused only if every block in the symmetric difference
    sits at an oracle rank whose inclusive cumulative probability (or the one
    before it) lies within TOPP_WINDOW of p, or ties (within the rounding
    window) with the oracle's boundary block."""
    ocnt, oidx = orc["kv_cnt"], orc["kv_idx"]
    B, H, nb = ocnt.shape
    gc = gpu_cnt.reshape(B, H, nb)
    gi = gpu_idx.reshape(B, H, nb, nb)
    same_cnt = gc == ocnt
    col = np.arange(nb)[None, None, None, :]
    valid = col < ocnt[..., None]
    same_idx = np.where(valid, gi == oidx, True).all(axis=-1)
    same = same_cnt & same_idx
    res = ListCompare(rows=B * H * nb, identical=int(same.sum()), excused_topp=0, excused_tie=0, unexcused=0)
    bad = np.argwhere(~same)
    qn = np.linalg.norm(qbar, axis=-1)     # [B,H,nb]
    kn = np.linalg.norm(kbar, axis=-1)
    for b, h, i in bad:
        o = orc["order"][b, h, i]
        cum = orc["cum"][b, h, i]
        probs = orc["probs"][b, h, i]
        so = set(oidx[b, h, i, :ocnt[b, h, i]].tolist())
        sg = set(gi[b, h, i, :gc[b, h, i]].tolist())
        diff = so ^ sg
        rank = np.empty(nb, dtype=np.int64)
        rank[o] = np.arange(nb)
        # oracle count before the diagonal repair
        m_p = nb if p >= 1 else int(np.argmax(cum >= p)) + 1 if (cum >= p).any() else nb
        m = min(nb, max(m_p, k_min))
        s = scale * (qbar[b, h, i] @ kbar[b, h].T)
        tau = TIE_FACTOR * scale * qn[b, h, i] * kn[b, h].max()
        ex_topp = ex_tie = unexcused = False
        for j in diff:
            r = rank[j]
            c_prev = cum[r - 1] if r > 0 else 0.0
            if abs(cum[r] - p) <= TOPP_WINDOW or abs(c_prev - p) <= TOPP_WINDOW:
                ex_topp = True
                continue
            near = [o[x] for x in (m - 1, m) if 0 <= x < nb]
            if any(abs(s[j] - s[q]) <= tau for q in near):
                ex_tie = True
                continue
            unexcused = True
            break
        if unexcused:
            res.unexcused += 1
            if res.first_unexcused is None:
                res.first_unexcused = dict(b=int(b), h=int(h), i=int(i), oracle=sorted(so), gpu=sorted(sg),
                                           diff=sorted(int(x) for x in diff))
        elif ex_topp:
            res.excused_topp += 1
        else:
            res.excused_tie += 1
    return res


def sample_rows(wl, kv_cnt, n_random=96, seed=0):
    """Query tokens to check: random ones, every token class of the edge
    blocks (last t/y/x block), and rows of the heaviest and lightest unit of a
    few heads. Returns flat indices (b*H + h)*N + n."""
    rng = np.random.default_rng(seed)
    B, H, N = wl.B, wl.H, wl.N
    T, Hg, W = wl.grid
    bt, bh, bw = wl.block
    nbh, nbw = -(-Hg // bh), -(-W // bw)
    rows = set(rng.choice(B * H * N, size=min(n_random, B * H * N), replace=False).tolist())
    # the very last token (corner of the last block) and last-frame tokens
    for bhh in rng.choice(B * H, size=min(4, B * H), replace=False):
        for n in (N - 1, (T - 1) * Hg * W, (T - 1) * Hg * W + Hg * W // 2, rng.integers(N)):
            rows.add(int(bhh) * N + int(n))
    cnt = kv_cnt.reshape(B * H, -1)
    for bhh in rng.choice(B * H, size=min(6, B * H), replace=False):
        for i in (int(cnt[bhh].argmax()), int(cnt[bhh].argmin())):
            jt, jy, jx = i // (nbh * nbw), (i // nbw) % nbh, i % nbw
            for _ in range(3):
                t = min(T - 1, jt * bt + int(rng.integers(bt)))
                y = min(Hg - 1, jy * bh + int(rng.integers(bh)))
                x = min(W - 1, jx * bw + int(rng.integers(bw)))
                rows.add(int(bhh) * N + (t * Hg + y) * W + x)
    return np.array(sorted(rows), dtype=np.int64)


def attn_errors(gpu_out, rows, ref, D):
    got = gpu_out.reshape(-1, D)[torch.from_numpy(rows).to(gpu_out.device)].float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    return float(err.max()), float(err.mean())


def kept_flops(wl, kv_cnt, kv_idx, valid_sizes):
    """Algorithmic attention FLOPs on kept blocks: 4*D*sum_i |i| * sum_{j in S_i} |j|."""
    B, H, nb = kv_cnt.shape
    total = 0
    vs = valid_sizes.astype(np.int64)
    for b in range(B):
        for h in range(H):
            cnt = kv_cnt[b, h]
            idx = kv_idx[b, h]
            mask = np.arange(nb)[None, :] < cnt[:, None]
            kept = np.where(mask, vs[np.clip(idx, 0, nb - 1)], 0).sum(axis=1)
            total += int((vs * kept).sum())
    return 4 * wl.D * total
