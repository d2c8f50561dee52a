"""Fit the polynomial the attention kernel uses for part of its exponentials.

Method (Cody-Waite style range reduction with a fitted polynomial): for x <= 8,
    n = round(x),  f = x - n in [-1/2, 1/2],  2^x = 2^n * p(f),
where p is a degree-DEG polynomial fitted here to minimise the maximum RELATIVE error of
p(f) against 2^f on [-1/2, 1/2] (a discrete Remez exchange on a dense grid, seeded by a
Chebyshev least-squares fit), with p(0) constrained to 1 so that exact powers of two come
out exact. 2^n is applied by adding n to the exponent field.

    python online_softmax_exact_b200/csrc/exp2_poly_fit.py
prints the coefficients (fp32, lowest order first) and the achieved relative error in
fp64 and when evaluated in fp32 with Horner's rule, as the kernel does.
"""

from __future__ import annotations

import numpy as np

DEG = 3


def fit(deg: int = DEG, iters: int = 60):
    x = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(x)
    # p(f) = 1 + f * q(f): fit q, weights 1/y for relative error
    def design(xs):
        return np.stack([xs ** (k + 1) for k in range(deg)], axis=1)

    A = design(x)
    w = 1.0 / y
    q, *_ = np.linalg.lstsq(A * w[:, None], (y - 1.0) * w, rcond=None)
    # iteratively re-weighted least squares towards the minimax relative error
    weights = np.ones_like(x)
    for _ in range(iters):
        err = (1.0 + A @ q - y) / y
        weights *= (1.0 + 50.0 * np.abs(err) / np.abs(err).max())
        weights /= weights.mean()
        ww = weights * w
        q, *_ = np.linalg.lstsq(A * ww[:, None], (y - 1.0) * ww, rcond=None)
    coeffs = np.concatenate([[1.0], q])
    return coeffs


def horner_f32(coeffs, f):
    c = coeffs.astype(np.float32)
    f = f.astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return p


def main():
    coeffs = fit()
    x = np.linspace(-0.5, 0.5, 200001)
    rel64 = np.abs(np.polyval(coeffs[::-1], x) / np.exp2(x) - 1).max()
    rel32 = np.abs(horner_f32(coeffs, x).astype(np.float64) / np.exp2(x) - 1).max()
    print("coefficients (fp32, c0..c%d):" % DEG)
    for k, c in enumerate(coeffs.astype(np.float32)):
        print(f"  c{k} = {float(c):.9e}f")
    print(f"max relative error: fp64 {rel64:.3e}, fp32 Horner {rel32:.3e}")


if __name__ == "__main__":
    main()
