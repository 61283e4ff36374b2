"""Fit the polynomial of the FMA-pipe exp2 used by the forward's softmax.

2^x is evaluated as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(range reduction by an integer shift of the exponent field).  This script fits
p(f) = 1 + f (c1 + f (c2 + f c3)), constrained to p(0) = 1 so that whole-number
arguments (and the clamped -127 of masked scores) are exact, for the least
maximum relative error on [-1/2, 1/2]: a Lawson iteration of weighted least
squares, which converges to the minimax (equioscillating) solution.  It prints
the float32 coefficients and the error of the float32 Horner evaluation; the
values are copied into ``csrc/ptx.cuh`` (ex2_poly).

    python mask_skipping_flashattention_b200/fit_exp2_poly.py
"""

import numpy as np


def fit(deg=3, iters=200, npts=20001):
    f = np.linspace(-0.5, 0.5, npts)
    y = np.exp2(f)
    a = np.stack([f ** k for k in range(1, deg + 1)], 1)
    w = np.full_like(f, 1.0 / npts)
    for _ in range(iters):
        sw = np.sqrt(w) / y  # relative error weighting
        c, *_ = np.linalg.lstsq(a * sw[:, None], (y - 1.0) * sw, rcond=None)
        e = np.abs((1.0 + a @ c - y) / y)
        w = w * (e / e.max() + 1e-12)
        w /= w.sum()
    return c.astype(np.float32)


def horner32(c, f):
    f = f.astype(np.float32)
    q = np.full_like(f, c[-1])
    for ck in c[-2::-1]:
        q = (q * f + ck).astype(np.float32)
    return (np.float32(1.0) + f * q).astype(np.float32)


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(horner32(c, f).astype(np.float64) / np.exp2(f) - 1.0).max()
    print("c1..c3 =", ", ".join(f"{float(x):.9e}f" for x in c))
    print(f"max relative error (float32 Horner) on [-1/2, 1/2]: {err:.3e}")
