"""Fit the polynomial the kernels use for 2^f on [-1/2, 1/2].

Method: Cody-Waite style range reduction (x = n + f with n = round(x),
2^x = 2^n * 2^f, 2^n applied by adding n to the float's exponent field) and a
minimax polynomial for 2^f on [-1/2, 1/2], found with the Remez exchange
algorithm (relative error, equioscillation on degree + 2 points).  Everything
here is computed from the mathematics; no library's constants are used.

Run:  python io_aware_exact_33_b200/csrc/fit_exp2.py [degree]
It prints the coefficients (float32-rounded) and the achieved maximum
relative error of the float32 Horner evaluation; the values are pasted into
sm100.cuh (exp2_poly2).
"""
from __future__ import annotations

import sys

import numpy as np


def remez_relative(degree: int, iters: int = 60):
    """Minimax (relative error) polynomial for 2^f on [-1/2, 1/2]."""
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    xs = -0.5 * np.cos(np.pi * k / (n - 1))
    grid = np.linspace(-0.5, 0.5, 200001)
    target = np.exp2(grid)
    coef = None
    for _ in range(iters):
        # Solve sum_j c_j x_i^j + (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(xs))
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - target) / target
        # new reference: alternating extrema of the error
        sign = np.sign(err)
        idx = []
        start = 0
        for j in range(1, len(grid) + 1):
            if j == len(grid) or sign[j] != sign[start]:
                seg = slice(start, j)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = j
        idx = np.array(idx)
        if len(idx) > n:  # keep the n largest alternating extrema
            while len(idx) > n:
                drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
                idx = np.delete(idx, drop)
        if len(idx) == n:
            xs = grid[idx]
    return coef


def horner_f32(coef32, f):
    acc = np.float32(coef32[-1])
    for c in coef32[-2::-1]:
        acc = np.float32(acc * f + np.float32(c))  # fma approximated in float64 then rounded
    return acc


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = remez_relative(degree)
    coef32 = [np.float32(c) for c in coef]
    f = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    approx = np.array([horner_f32(coef32, x) for x in f[::10]], dtype=np.float64)
    exact = np.exp2(f[::10].astype(np.float64))
    rel = np.max(np.abs(approx - exact) / exact)
    print(f"degree {degree}: max relative error {rel:.3e} (float32 Horner)")
    for i, c in enumerate(coef32):
        print(f"  c{i} = {float(c):.9e}f  (bits 0x{np.float32(c).view(np.uint32):08x})")


if __name__ == "__main__":
    main()
