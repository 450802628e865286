"""Fit of the polynomial used for part of the softmax exponentials (exp2_poly.h).

The attention kernel computes 2^x for some softmax columns on the FMA/ALU
pipes instead of the MUFU unit: x = j + f with j = round(x), f in [-1/2, 1/2],
2^x = 2^j * p(f). p is the minimax polynomial for the *relative* error of 2^f on
[-1/2, 1/2], found with the Remez exchange algorithm (equioscillation of the
relative error at deg+2 points). Run: python exp2_poly_fit.py
Degree 3 gives max relative error 7.5e-5, below the bf16 rounding (2^-9) that
P receives before the PV product.
"""
import numpy as np
from numpy.polynomial import polynomial as P
def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        t = np.linspace(a, b, 200001)
        err = (P.polyval(t, c) - f(t)) / f(t)
        # new extrema: sign changes partition
        idx = [0]
        s = np.sign(err)
        for k in range(1, len(t)):
            if s[k] != s[idx[-1]]:
                idx.append(k)
            elif abs(err[k]) > abs(err[idx[-1]]):
                idx[-1] = k
        if len(idx) >= n:
            # keep n points with largest |err| alternating (take first n)
            x = t[idx[:n]] if len(idx) == n else t[sorted(idx, key=lambda k: -abs(err[k]))[:n]]
            x = np.sort(x)
    return c, np.max(np.abs(err))
for d in (3, 4):
    c, e = remez(d)
    c32 = c.astype(np.float32)
    t = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    # evaluate in float32 Horner like the kernel
    p = np.float32(c32[-1])
    for k in range(d - 1, -1, -1):
        p = (p * t + c32[k]).astype(np.float32)
    rel = np.max(np.abs(p.astype(np.float64) - np.exp2(t.astype(np.float64))) / np.exp2(t.astype(np.float64)))
    print(d, [float(v) for v in c32], "minimax rel err %.3e, float32 Horner rel err %.3e" % (e, rel))
    print("   hex:", [hex(np.float32(v).view(np.uint32)) for v in c32])
