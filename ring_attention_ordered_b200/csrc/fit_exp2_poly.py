"""Fit the polynomial the kernels can use for part of their 2^x evaluations.

Method: Remez exchange (minimax in relative error) for p(f) ~ 2^f on
f in [-1/2, 1/2], degree 3.  The kernel splits x = j + f with j = round(x)
(the 1.5 * 2^23 add-and-subtract trick) and scales p(f) by 2^j by adding
j << 23 to the float's bits.  Coefficients are rounded to float32 and the
reported error bound is measured on the rounded coefficients with float32
Horner evaluation.

Run: ``python ring_attention_ordered_b200/csrc/fit_exp2_poly.py`` -- prints
the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the maximum relative
error; the values are copied into ``ra_exp2.cuh`` (EXP2_C0..C3), which
``tests/test_exp2_poly.py`` checks against this fit.
"""

from __future__ import annotations

import numpy as np


def remez_relative(func, lo, hi, degree, iters=40):
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * func(x[i])
        sol = np.linalg.solve(A, func(x))
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - func(grid)) / func(grid)
        # new reference: extrema of the error between its sign changes
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest magnitudes
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return coef


def horner_f32(coef32, f):
    f = f.astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p * f + c).astype(np.float32)
    return p


def main():
    coef = remez_relative(lambda t: np.exp2(t), -0.5, 0.5, 3)
    c32 = coef.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001)
    rel = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f) - 1.0)
    for i, c in enumerate(c32):
        print(f"EXP2_C{i} = {float(c):.9e}f  ({c.view(np.uint32):#010x})")
    print(f"max relative error (float32 Horner, rounded coefficients): {rel.max():.3e}")


if __name__ == "__main__":
    main()
