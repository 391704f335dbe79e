"""Derives the polynomial the tensor-core kernel uses for part of its 2^x.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite
range reduction: the integer part goes into the exponent field, only the
fraction needs approximating).  2^f on [-1/2, 1/2] is approximated by the
degree-3 polynomial that minimises the maximum RELATIVE error, found with the
Remez exchange algorithm (equioscillation at degree+2 points).  The kernel
rounds P to bf16 (relative precision 2^-9) right after, so the polynomial's
error only has to stay well below that.

    python -m attention_sdpa_fwd_b200.csrc.fit_exp2_poly      (prints the coefficients)
"""
from __future__ import annotations

import numpy as np

LO, HI = -0.5, 0.5


def remez_relative(degree: int = 3, iters: int = 30):
    """Minimax polynomial for 2^f with weight 1/2^f (relative error)."""
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    xs = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    f = lambda x: np.exp2(x)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)   (relative error equioscillates)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: the extrema of the error between sign changes
        sign = np.sign(err)
        idx = []
        start = 0
        for j in range(1, len(grid) + 1):
            if j == len(grid) or sign[j] != sign[start]:
                seg = np.arange(start, j)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = j
        if len(idx) < n:
            break
        idx = np.array(idx)
        if len(idx) > n:  # keep the n largest alternating extrema
            while len(idx) > n:
                drop = np.argmin(np.abs(err[idx]))
                idx = np.delete(idx, drop)
        xs = grid[idx]
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative(3)
    print("coefficients c0..c3:", ", ".join(f"{x:.9e}" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
    c32 = np.float32(c)
    g = np.linspace(LO, HI, 100001, dtype=np.float32)
    p = ((c32[3] * g + c32[2]) * g + c32[1]) * g + c32[0]
    print(f"in float32 (Horner): {np.max(np.abs(p / np.exp2(g.astype(np.float64)) - 1)):.3e}")
