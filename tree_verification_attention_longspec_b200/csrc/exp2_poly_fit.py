"""Derive the polynomial used by the prefix kernel's software 2^x.

Method (Cody-Waite range reduction followed by a minimax polynomial):
  2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2];
  2^f is approximated on [-1/2, 1/2] by the degree-3 polynomial that minimises the
  maximum RELATIVE error (Remez exchange algorithm), and 2^n is applied by adding n
  to the exponent field of the result.

    python exp2_poly_fit.py      # prints the coefficients and their error

The coefficients are rounded to fp32; the printed bound is for fp32 Horner
evaluation, checked on a dense grid.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(deg=DEGREE, lo=LO, hi=HI, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (relative error equioscillation)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        sign = np.sign(err)
        for j in range(1, len(grid)):
            if sign[j] != sign[idx[-1]] and sign[j] != 0:
                idx.append(j)
            elif abs(err[j]) > abs(err[idx[-1]]):
                idx[-1] = j
        if len(idx) >= n:
            # keep the n alternating extrema with the largest magnitude window
            best = max(range(len(idx) - n + 1), key=lambda s: min(abs(err[idx[s:s + n]])))
            xs = grid[idx[best:best + n]]
    return c


def horner_f32(c, f):
    f = f.astype(np.float32)
    r = np.float32(c[-1])
    for a in c[-2::-1]:
        r = (r * f + np.float32(a)).astype(np.float32)
    return r


def main():
    c = remez_relative()
    c32 = np.array(c, dtype=np.float32)
    grid = np.linspace(LO, HI, 2_000_001)
    rel = np.abs(horner_f32(c32, grid).astype(np.float64) / np.exp2(grid) - 1.0)
    print("coefficients (c0 + c1 f + c2 f^2 + c3 f^3), fp32:")
    for i, a in enumerate(c32):
        print(f"  c{i} = {float(a):.9e}f  ({float(a).hex()})")
    print(f"max relative error of fp32 Horner on [{LO}, {HI}]: {rel.max():.3e}")


if __name__ == "__main__":
    main()
