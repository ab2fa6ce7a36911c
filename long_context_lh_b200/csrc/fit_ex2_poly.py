"""Fit of the cubic that approximates 2^f on [-1/2, 1/2] in ex2_fma2 (tc_common.cuh).

ex2_fma2 computes 2^x as 2^n * p(f) with n = rint(x), f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction: W. J. Cody and W. Waite, "Software Manual
for the Elementary Functions", Prentice-Hall, 1980).  p is the degree-3
polynomial of least maximum RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2],
found by the Remez exchange algorithm (E. Remez, 1934): start from the
Chebyshev extrema, solve for the coefficients and the levelled error E on
deg + 2 reference points, move the references to the extrema of the error
curve, repeat until they stop moving.  The coefficients are then rounded to
fp32, the type the kernel evaluates them in.

Run:  python fit_ex2_poly.py   (prints the four fp32 constants, c0 first, and
the maximum relative error of the fp32 polynomial on a fine grid).
Nothing here is used at run time; the kernel holds the printed constants.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(deg: int = DEGREE, iters: int = 50, grid: int = 400001):
    """Coefficients c[0..deg] (c0 first) minimising max |p/2^f - 1| on [LO, HI]."""
    n = deg + 2
    k = np.arange(n)
    x = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    g = np.linspace(LO, HI, grid)
    c = None
    for _ in range(iters):
        # p(x_i) - (-1)^i E 2^x_i = 2^x_i  <=>  p(x_i)/2^x_i - 1 = (-1)^i E
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = -((-1.0) ** k) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        e = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
        # one extremum of |e| between consecutive sign changes
        cuts = [0] + list(np.where(np.diff(np.sign(e)) != 0)[0] + 1) + [grid]
        xn = np.array([g[a + np.argmax(np.abs(e[a:b]))] for a, b in zip(cuts[:-1], cuts[1:])])
        if len(xn) != n or np.allclose(xn, x, rtol=0, atol=1e-12):
            break
        x = xn
    return c


def fp32_poly_max_rel_error(c32: np.ndarray, grid: int = 400001) -> float:
    """Max relative error of the Horner evaluation in fp32, each step a fused
    multiply-add (the fp32 product is exact in fp64; the sum is rounded once to
    fp32 after an fp64 addition, which can differ from a true fused rounding by
    an ulp in rare cases -- far below the bound this checks)."""
    f = np.linspace(LO, HI, grid).astype(np.float32)
    p = np.full_like(f, c32[3])
    for j in (2, 1, 0):
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c32[j])).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def fitted_constants() -> np.ndarray:
    return remez_relative().astype(np.float32)


if __name__ == "__main__":
    c32 = fitted_constants()
    for j, v in enumerate(c32):
        print(f"c{j} = {float(v):.8g}f")
    print(f"max relative error (fp32 Horner): {fp32_poly_max_rel_error(c32):.4g}")
