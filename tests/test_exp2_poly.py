"""The polynomial exponential used for part of the softmax columns (CPU).

The attention kernel computes some 2^a values as 2^round(a) * p(a - round(a))
with the degree-3 minimax polynomial of csrc/exp2_poly.h, applying 2^j by
adding j to the float's exponent field. This test replays that arithmetic
bit for bit in float32 with numpy (same constants, same operation order,
same rounding constant and clamp) and checks it against exp2 over the range
the softmax produces, including masked columns (-inf) and very small values.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_fvattn_b200", "csrc", "exp2_poly.h")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"FV_EXP2_C{i}\s+([0-9.eE+-]+)f", text).group(1))) for i in range(4)]


def emulate(a):
    c0, c1, c2, c3 = coeffs()
    a = np.maximum(a.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (a + magic).astype(np.float32)
    f = (a - (t - magic).astype(np.float32)).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)      # fma in the kernel; one extra rounding here is harmless
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) \
        & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_softmax_range():
    a = np.linspace(-125.0, 9.0, 2_000_001, dtype=np.float32)   # results in the normal range
    got = emulate(a).astype(np.float64)
    ref = np.exp2(a.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert np.isfinite(got).all()
    assert rel.max() < 1.0e-4, rel.max()


def test_masked_and_underflowing_arguments_are_tiny_not_nan():
    a = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.5, -126.0], dtype=np.float32)
    got = emulate(a)
    assert np.isfinite(got).all() and (got >= 0).all()
    assert (got <= np.float32(2.0 ** -125)).all()


def test_exact_powers_of_two():
    a = np.arange(-120, 9, dtype=np.float32)
    got = emulate(a).astype(np.float64)
    c0 = float(coeffs()[0])
    np.testing.assert_allclose(got / np.exp2(a.astype(np.float64)), c0, rtol=1e-7)
