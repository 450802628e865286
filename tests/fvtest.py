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
# At most this share of rows may differ from the oracle under the two excuses.
EXCUSED_MAX_SHARE = 0.02

# fp32 unit roundoff and the standard bound gamma_n = n*u / (1 - n*u) on the
# error of any n-term fp32 sum, whatever its order (Higham, "Accuracy and
# Stability of Numerical Algorithms", 2nd ed., section 3.1).
U32 = 2.0 ** -24


def gamma(n):
    return n * U32 / (1.0 - n * U32)


def geometry(wl, dtype=torch.bfloat16, softmax_scale=0.0):
    from block_sparse_attention_fvattn_b200 import fvattn as fa
    return fa.Geometry(wl.B, wl.H, wl.D, wl.grid, wl.block, softmax_scale=softmax_scale, dtype=dtype)


def make_on_gpu(wl, seed=None, dtype=torch.bfloat16):
    """The seeded bf16 inputs; for fp16 they are converted (through fp32)."""
    q, k, v = gen.make_inputs(wl, "cuda", seed=seed)
    if dtype != torch.bfloat16:
        q, k, v = (t.float().to(dtype) for t in (q, k, v))
    torch.cuda.synchronize()
    return q, k, v


def abs_bits(x):
    """|x| of a bf16/fp16 tensor as raw 16-bit patterns (the sign bit cleared, exact)."""
    b = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(b & np.uint16(0x7FFF))


@dataclass
class ScoreBound:
    """Inputs of the per-pair rounding bound of the GPU's fp32 block scores.

    qbar, kbar: the oracle's fp64 block means [B,H,nb,D]; qabs, kabs: block
    means of |Q| and |K| (the same pooling on the absolute values); sizes:
    valid tokens per block; tc: the scores come from the three-product TF32
    split (rows of >= 320 blocks)."""
    qbar: np.ndarray
    kbar: np.ndarray
    qabs: np.ndarray
    kabs: np.ndarray
    sizes: np.ndarray
    scale: float
    tc: bool

    def row(self, b, h, i):
        """e[j] >= |s_fp32[i, j] - s_fp64[i, j]| for every key block j of row (b, h, i).

        The GPU pools each mean as an fp32 sum of n bf16 values (any order:
        error <= gamma_{n-1} * n * mean|x|), times an fp32 reciprocal of n (two
        more roundings); then a D-term fp32 dot product (gamma_D of the sum of
        |q_d k_d|; with the TF32 split, 3D products plus the dropped and
        rounded low parts, below 2^-20 of each |q_d k_d|), and one rounding
        of the scale product. The bound adds these terms up, keeping the
        products of two error terms."""
        D = self.qbar.shape[-1]
        n_i = int(self.sizes[i])
        qm, qa = np.abs(self.qbar[b, h, i]), self.qabs[b, h, i]
        km, ka = np.abs(self.kbar[b, h]), self.kabs[b, h]
        eq = gamma(max(n_i - 1, 1)) * qa + 3 * U32 * qm
        ek = gamma(np.maximum(self.sizes - 1, 1).astype(np.float64))[:, None] * ka + 3 * U32 * km
        g_dot = (gamma(3 * D) + 2.0 ** -20) if self.tc else gamma(D)
        e1 = km @ eq + ek @ qm + ek @ eq
        e2 = (km + ek) @ (qm + eq)
        s = self.scale * (self.kbar[b, h] @ self.qbar[b, h, i])
        return self.scale * (e1 + g_dot * e2) * (1 + 1e-6) + 2 * U32 * np.abs(s)


@dataclass
class ListCompare:
    rows: int
    identical: int
    excused_topp: int
    excused_tie: int
    unexcused: int
    invalid: int
    first_unexcused: object = None
    first_invalid: object = None

    def summary(self):
        return (f"rows {self.rows}: identical {self.identical}, excused at the Top-p boundary "
                f"{self.excused_topp}, excused as rounding ties {self.excused_tie}, unexcused {self.unexcused}, "
                f"invalid {self.invalid}")


def _row_validity(gc, gi, orc, p, k_min):
    """Checks every GPU row must pass whatever the oracle chose: count in
    [min(k_min, nb), nb], indices strictly ascending inside [0, nb), the
    diagonal block present, and a kept count consistent with the oracle's
    probabilities (enough mass, and minimal unless the floor binds). Returns a
    bool array [B,H,nb] marking invalid rows."""
    B, H, nb = gc.shape
    kp = min(k_min, nb)
    out = np.zeros((B, H, nb), dtype=bool)
    col = np.arange(nb)[None, :]
    diag = np.arange(nb)[:, None]
    for b in range(B):
        for h in range(H):
            c, idx = gc[b, h], gi[b, h]
            valid = col < c[:, None]
            bad = (c < kp) | (c > nb)
            last = np.take_along_axis(idx, (np.clip(c, 1, nb) - 1)[:, None], -1)[:, 0]
            asc = np.where(valid[:, 1:], np.diff(idx, axis=-1) > 0, True).all(-1)
            bad |= ~asc | (idx[:, 0] < 0) | (last >= nb)
            bad |= ~np.where(valid, idx == diag, False).any(-1)
            if p >= 1.0:
                out[b, h] = bad | (c != nb)
                continue
            probs = orc["probs"][b, h]
            nonf = orc["nonfinite"][b, h].astype(bool)
            P = np.take_along_axis(probs, np.clip(idx, 0, nb - 1), -1)
            mass = np.where(valid, P, 0.0).sum(-1)
            pmin = np.where(valid, P, np.inf).min(-1)
            pmin_wo = np.where(valid & (idx != diag), P, np.inf).min(-1)
            mass_wo = mass - np.diagonal(probs)

            def consistent(m, ms, pm):
                # m blocks kept by Top-p + floor: at least the floor, enough
                # mass, and minimal unless the floor binds: without the weakest
                # kept block the mass would fall short of p
                return (m >= kp) & ((m == nb) | (ms >= p - TOPP_WINDOW)) & ((m == kp) | (ms - pm < p + TOPP_WINDOW))

            # the diagonal block is one of the ranked blocks, or added by the repair
            ok = consistent(c, mass, pmin) | consistent(c - 1, mass_wo, pmin_wo)
            out[b, h] = bad | (~ok & ~nonf)
    return out


def compare_lists(gpu_cnt, gpu_idx, orc, bound: ScoreBound, p, k_min):
    """Compare GPU kept lists with the oracle's, row by row.

    Every GPU row must be valid on its own (see _row_validity). A row that
    differs from the oracle's is excused only if every block in the symmetric
    difference sits at an oracle rank whose inclusive cumulative probability
    (or the one before it) lies within TOPP_WINDOW of p, or its fp64 score
    lies within the rounding bound of the pair (the GPU scores are fp32) of
    the oracle's boundary block; and if the GPU's kept set is still a prefix
    of some ranking that orders no pair of blocks against their fp64 scores
    by more than that pair's rounding bound."""
    ocnt, oidx = orc["kv_cnt"], orc["kv_idx"]
    B, H, nb = ocnt.shape
    gc = np.asarray(gpu_cnt).reshape(B, H, nb).astype(np.int64)
    gi = np.asarray(gpu_idx).reshape(B, H, nb, nb).astype(np.int64)
    invalid = _row_validity(gc, gi, orc, p, k_min)
    same_cnt = gc == ocnt
    col = np.arange(nb)[None, None, None, :]
    valid = col < ocnt[..., None]
    same_idx = np.where(valid, gi == oidx, True).all(axis=-1)
    same = same_cnt & same_idx
    res = ListCompare(rows=B * H * nb, identical=int(same.sum()), excused_topp=0, excused_tie=0, unexcused=0,
                      invalid=int(invalid.sum()))
    if res.invalid:
        b, h, i = np.argwhere(invalid)[0]
        res.first_invalid = dict(b=int(b), h=int(h), i=int(i), cnt=int(gc[b, h, i]),
                                 gpu=gi[b, h, i, :max(0, min(int(gc[b, h, i]), nb))].tolist())
    for b, h, i in np.argwhere(~same):
        o = orc["order"][b, h, i]
        cum = orc["cum"][b, h, i]
        so = set(oidx[b, h, i, :ocnt[b, h, i]].tolist())
        sg = set(gi[b, h, i, :min(max(gc[b, h, i], 0), nb)].tolist())
        diff = so ^ sg
        rank = np.empty(nb, dtype=np.int64)
        rank[o] = np.arange(nb)
        # oracle count before the diagonal repair
        m_p = nb if p >= 1 else int(np.argmax(cum >= p)) + 1 if (cum >= p).any() else nb
        m = min(nb, max(m_p, k_min))
        s = bound.scale * (bound.kbar[b, h] @ bound.qbar[b, h, i])
        e = bound.row(b, h, i)
        ex_topp = ex_tie = unexcused = False
        for j in diff:
            r = rank[j]
            c_prev = cum[r - 1] if r > 0 else 0.0
            if abs(cum[r] - p) <= TOPP_WINDOW or abs(c_prev - p) <= TOPP_WINDOW:
                ex_topp = True
                continue
            # a rounding tie across the oracle's boundary: a block the oracle
            # kept against the first one it dropped, or the other way round
            other = int(o[m]) if r < m and m < nb else int(o[m - 1]) if r >= m and m >= 1 else None
            if other is not None and other != j and abs(s[j] - s[other]) <= e[j] + e[other]:
                ex_tie = True
                continue
            unexcused = True
            break
        if not unexcused:
            # prefix check: no dropped block beats a kept one (the diagonal
            # aside) by more than the pair's rounding bound
            kept = np.array(sorted(sg - {int(i)}), dtype=np.int64)
            drop = np.array(sorted(set(range(nb)) - sg), dtype=np.int64)
            if kept.size and drop.size:
                gap = s[drop][:, None] - s[kept][None, :]
                unexcused = bool((gap > e[drop][:, None] + e[kept][None, :]).any())
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


# The library scores rows of at least this many blocks on the tensor cores
# (three-product TF32 split); shorter rows on the CUDA cores in fp32.
TC_SCORES_MIN_BLOCKS = 320

# List comparisons of this test session, by workload, for the terminal summary.
RECORDED = {}


def record(name, res: ListCompare):
    RECORDED[name] = res


def score_bound(orc, g, q, k, qbar, kbar, scale, tc):
    """ScoreBound for inputs q, k (bf16/fp16 tensors) and the oracle's means."""
    qabs = orc.pool(g, abs_bits(q))
    kabs = orc.pool(g, abs_bits(k))
    return ScoreBound(qbar, kbar, qabs, kabs, orc.block_sizes(g).astype(np.int64), scale, tc)


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


def attn_excess(gpu_out, rows, ref, D, rel):
    """max over the checked elements of |gpu - ref| - rel * |ref|: the error
    left after each element's own output rounding (rel = the element type's
    unit roundoff) is taken off."""
    got = gpu_out.reshape(-1, D)[torch.from_numpy(rows).to(gpu_out.device)].float().cpu().numpy().astype(np.float64)
    return float((np.abs(got - ref) - rel * np.abs(ref)).max())


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
