"""Fit the polynomial that fa_fwd.cu uses to evaluate 2^x on the FMA pipe.

Method: Cody-Waite style range reduction x = n + f with n = round(x), f in [-1/2, 1/2],
2^x = 2^n * 2^f, and a minimax approximation of 2^f on [-1/2, 1/2] in the relative-error
sense, found with the Remez exchange algorithm (E. Remez, 1934). The constant term is not
constrained. Run: python gen_exp2_poly.py [degree]; prints the coefficients (c0..cd) and
the max relative error of the float32 Horner evaluation over a dense grid.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_rel(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 30) -> np.ndarray:
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # Solve p(x_i) + (-1)^i E f(x_i) = f(x_i) for coefficients and E (relative error E)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return c


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    c32 = c.astype(np.float32)
    p = np.full_like(f, c32[-1], dtype=np.float32)
    for ci in c32[-2::-1]:
        p = (p * f + ci).astype(np.float32)  # the kernel uses fused multiply-add
    return p


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_rel(deg)
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    rel = np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    print("coefficients c0..c%d:" % deg, ", ".join(f"{float(np.float32(ci)):.9e}f" for ci in c))
    print("max relative error (float32 Horner):", rel.max())
