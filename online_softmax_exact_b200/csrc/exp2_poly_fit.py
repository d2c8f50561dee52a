"""Fit the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by exp2_poly_f32x2 (sm100_ptx.cuh).

The Remez exchange algorithm for the minimax polynomial in relative error: start from
Chebyshev extrema, solve for coefficients that make the relative error equioscillate
on the current reference points, move the points to the error's extrema, repeat.
The coefficients are then rounded to fp32, as the kernel stores them, and the
maximum relative error of the rounded polynomial is measured on a fine grid.

    python online_softmax_exact_b200/csrc/exp2_poly_fit.py [--degree 3]
"""

from __future__ import annotations

import argparse

import numpy as np


def remez_exp2(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 50):
    """Coefficients c[0..degree] (constant term first) of the minimax relative-error
    approximation of 2^f on [lo, hi], and that error."""
    n = degree + 2
    k = np.arange(n)
    pts = 0.5 * (lo + hi) - 0.5 * (hi - lo) * np.cos(np.pi * k / (n - 1))
    grid = np.linspace(lo, hi, 400_001)
    c = np.zeros(degree + 1)
    for _ in range(iters):
        a = np.zeros((n, n))
        a[:, : degree + 1] = pts[:, None] ** np.arange(degree + 1)[None, :]
        a[:, -1] = (-1.0) ** k * 2.0**pts          # p(x_i) - 2^x_i = (-1)^i E 2^x_i
        sol = np.linalg.solve(a, 2.0**pts)
        c = sol[:-1]
        err = np.polynomial.polynomial.polyval(grid, c) / 2.0**grid - 1.0
        # the new reference: the extremum of each run of equal sign
        sign = np.sign(err)
        runs = np.flatnonzero(np.diff(sign) != 0) + 1
        bounds = np.concatenate([[0], runs, [grid.size]])
        if bounds.size - 1 != n:
            break
        pts = np.array([grid[a0 + np.argmax(np.abs(err[a0:b0]))]
                        for a0, b0 in zip(bounds[:-1], bounds[1:])])
    c32 = c.astype(np.float32)
    err32 = np.polynomial.polynomial.polyval(grid, c32.astype(np.float64)) / 2.0**grid - 1.0
    return c32, float(np.abs(err32).max())


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--degree", type=int, default=3)
    a = ap.parse_args()
    c, e = remez_exp2(a.degree)
    for i, v in enumerate(c):
        print(f"constexpr float kExp2C{i} = {float(v)!r}f;")
    print(f"// max relative error after rounding to fp32: {e:.3e}")


if __name__ == "__main__":
    main()
