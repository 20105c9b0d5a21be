"""Reproduce the 2^f coefficients of exp2_poly.cuh: the degree-3 polynomial
minimising max |p(f) / 2^f - 1| on [0, 1], by a Remez exchange, then its
maximum relative error when evaluated in float32 with Horner's rule.

    python fit_exp2_poly.py
"""
import numpy as np


def remez_relative(deg: int, iters: int = 40):
    n = deg + 2
    x = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))  # Chebyshev start
    g = np.linspace(0.0, 1.0, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[: deg + 1]
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        d = np.diff(err)
        ext = [0] + [i for i in range(1, len(g) - 1) if (d[i - 1] > 0) != (d[i] > 0)] + [len(g) - 1]
        if len(ext) >= n:
            ext = sorted(sorted(ext, key=lambda i: -abs(err[i]))[:n])
            x = g[ext]
    return c


def f32_error(c):
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(0.0, 1.0, 1000001).astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max())


if __name__ == "__main__":
    c = remez_relative(3)
    print("coefficients c0..c3:", [float(np.float32(v)) for v in c])
    print("max relative error (float32 Horner):", f32_error(c))
