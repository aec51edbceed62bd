"""Derive the polynomial used for exp2 on the FMA pipes in the scoring epilogue.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]; 2^f is approximated by a
polynomial p(f) whose coefficients minimise the maximum RELATIVE error on [-1/2, 1/2]
(Remez exchange algorithm, E. Ya. Remez 1934, in its textbook form for a weighted
polynomial fit).  The coefficients are then rounded to fp32 and the fp32 Horner
evaluation is checked against exp2 in fp64.

Run:  python exp2_poly.py [degree]     (prints the fp32 coefficients and the error bound)
"""
import sys

import numpy as np


def remez_relative(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 60):
    f = np.exp2
    # start from Chebyshev extrema
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i) for coefficients c and level E (relative weight 1/f)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.flatnonzero(np.diff(s) != 0)
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) < deg + 2:
            break
        # keep deg+2 alternating extrema with the largest magnitudes
        while len(ext) > deg + 2:
            mags = np.abs(err[ext])
            drop = 0 if mags[0] < mags[-1] else len(ext) - 1
            ext.pop(drop)
        x = grid[ext]
    return c, np.max(np.abs(err))


def check_fp32(c32: np.ndarray, n: int = 2_000_001):
    """fp32 Horner evaluation of p(f) against 2^f in fp64: max relative error on [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for ci in c32[-2::-1]:
        acc = (acc * f + ci).astype(np.float32)   # the kernel uses fused multiply-adds; this is a bound check
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c, e = remez_relative(deg)
    c32 = c.astype(np.float32)
    print(f"degree {deg}: minimax relative error {e:.3e}; fp32 Horner {check_fp32(c32):.3e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci)!r}f  // {ci.view(np.uint32):#010x}")
