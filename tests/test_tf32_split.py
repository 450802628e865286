"""Error bound of the three-product TF32 split used for long score rows (CPU).

From 320 blocks on, the routing scores s = Qbar_i . Kbar_j are formed on the
tensor cores from means split as x = hi + lo, hi = tf32(x), lo = tf32(x - hi),
with tf32() rounding an fp32 to 10 fraction bits, to nearest, ties away from
zero (PTX cvt.rna.tf32.f32), and s ~= hi_q.hi_k + hi_q.lo_k + lo_q.hi_k.
The list comparison of the GPU parity tests allows rank swaps within a window
that takes this split's error as at most 3 * 2^-22 * sum_d |q_d k_d| (on top
of the fp32 dot-product and pooling bounds). This test rebuilds the split
from that definition with numpy, forms the three products exactly in fp64,
and checks the bound, including the values where the rounding is worst.
"""
import numpy as np


def tf32_rna(x):
    """fp32 -> nearest fp32 with 13 low fraction bits clear, ties away from zero."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    sign = u & np.uint64(0x80000000)
    mag = u & np.uint64(0x7FFFFFFF)
    mag = (mag + np.uint64(0x1000)) & np.uint64(0x7FFFE000)   # add half an ulp of tf32, truncate
    return (sign | mag).astype(np.uint32).view(np.float32)


def split(x):
    x = np.asarray(x, dtype=np.float32)
    hi = tf32_rna(x)
    lo = tf32_rna((x - hi).astype(np.float32))
    return hi, lo


def three_product(q, k):
    qh, ql = split(q)
    kh, kl = split(k)
    f = lambda a: a.astype(np.float64)
    return (f(qh) * f(kh) + f(qh) * f(kl) + f(ql) * f(kh)).sum(axis=-1)


def test_rounding_definition():
    # 1 + 2^-11 is a tie between 1 and 1 + 2^-10: away from zero
    one = np.float32(1.0)
    tie = np.float32(1.0 + 2.0 ** -11)
    assert tf32_rna(tie) == np.float32(1.0 + 2.0 ** -10)
    assert tf32_rna(-tie) == -np.float32(1.0 + 2.0 ** -10)
    assert tf32_rna(np.float32(1.0 + 2.0 ** -12)) == one
    # already representable values are unchanged, and the result has 13 clear bits
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    r = tf32_rna(x)
    assert np.all((r.view(np.uint32) & np.uint32(0x1FFF)) == 0)
    assert np.array_equal(tf32_rna(r), r)
    assert np.all(np.abs(r.astype(np.float64) - x) <= 2.0 ** -11 * np.abs(x.astype(np.float64)))


def test_split_parts_are_exact_and_small():
    x = np.random.default_rng(1).standard_normal(100000).astype(np.float32) * np.float32(3.0)
    hi, lo = split(x)
    for part in (hi, lo):
        assert np.all((part.view(np.uint32) & np.uint32(0x1FFF)) == 0)
    resid = x.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64)
    assert np.all(np.abs(resid) <= 2.0 ** -22 * np.abs(x.astype(np.float64)))


def test_three_product_error_bound():
    rng = np.random.default_rng(2)
    for D in (64, 128):
        # block means: small, mixed-sign values of varied magnitude
        q = (rng.standard_normal((2000, D)) * rng.uniform(0.01, 3.0, (2000, 1))).astype(np.float32)
        k = (rng.standard_normal((2000, D)) * rng.uniform(0.01, 3.0, (2000, 1))).astype(np.float32)
        exact = (q.astype(np.float64) * k.astype(np.float64)).sum(axis=-1)
        got = three_product(q, k)
        scale = (np.abs(q.astype(np.float64)) * np.abs(k.astype(np.float64))).sum(axis=-1)
        assert np.all(np.abs(got - exact) <= 3 * 2.0 ** -22 * scale)


def test_worst_case_values():
    # mantissas whose low 13 bits sit at or next to the tf32 rounding tie, and
    # whose rest then rounds at its own tie: the largest residuals of the split
    worst = []
    for e in (0, -3, 5):
        for pattern in (0x1000, 0x0800 | 0x0001, 0x1FFF, 0x0FFF, 0x17FF | 0x0800):
            worst.append(np.ldexp(1.0 + pattern * 2.0 ** -23, e))
    x = np.array(worst, dtype=np.float32)
    assert np.array_equal(x.astype(np.float64), np.array(worst))   # exact in fp32
    q = np.stack([x, -x])
    k = np.stack([x[::-1], x[::-1]])
    exact = (q.astype(np.float64) * k.astype(np.float64)).sum(axis=-1)
    got = three_product(q, k)
    scale = (np.abs(q.astype(np.float64)) * np.abs(k.astype(np.float64))).sum(axis=-1)
    assert np.all(np.abs(got - exact) <= 3 * 2.0 ** -22 * scale)
