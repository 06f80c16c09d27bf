"""Coefficients of the cubic that the forward kernel (csrc/fwd2.cu, exp2_fma)
evaluates on the FMA pipe for part of its exponentials.

Method: Cody and Waite's range reduction (W. J. Cody and W. Waite, "Software
Manual for the Elementary Functions", 1980): 2^x = 2^n * 2^f with n = round(x)
and |f| <= 1/2; 2^f by the polynomial of degree 3 with the smallest maximum
relative error on [-1/2, 1/2], found by the Remez exchange algorithm (E. Ya.
Remez, 1934). The kernel adds n to the exponent bits of the polynomial's value.

    python -m split_kv_block_b200.exp2_poly     # prints the coefficients and the error bound
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int = 3, iters: int = 30, grid: int = 200001):
    """(coefficients c0..c_degree, max relative error) of the minimax
    polynomial for 2^f on [-1/2, 1/2]."""
    a, b = -0.5, 0.5
    n = degree
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * (n + 1 - k) / (n + 1))  # Chebyshev extrema as the start
    g = np.linspace(a, b, grid)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the n + 2 reference points
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:n + 1]
        err = (np.polyval(c[::-1], g) - np.exp2(g)) / np.exp2(g)
        # the new reference: the local extrema of the error (and the end points), the n + 2 largest
        idx = [0] + [j for j in range(1, grid - 1) if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) < 0] + [grid - 1]
        if len(idx) >= n + 2:
            x = np.sort(g[sorted(idx, key=lambda j: -abs(err[j]))[:n + 2]])
    err = (np.polyval(c[::-1], g) - np.exp2(g)) / np.exp2(g)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    coef, e = remez_exp2()
    print("coefficients (float32):", ", ".join(f"{float(np.float32(v)):.9g}f" for v in coef))
    print("max relative error on [-1/2, 1/2]:", e)
