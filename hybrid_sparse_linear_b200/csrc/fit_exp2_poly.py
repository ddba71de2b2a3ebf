"""Fits the polynomial used by fastexp.cuh: p(f) ~ 2^f on [-1/2, 1/2], minimax in relative error.

Method: Lawson's iteration (iteratively reweighted least squares whose weights converge to the
minimax solution) on a dense grid, then a check of the fp32 Horner evaluation.  Run it to
reproduce the coefficients in fastexp.cuh:  python fit_exp2_poly.py
"""
import numpy as np


def fit(deg: int, n: int = 20001, iters: int = 500):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True) / y[:, None]  # rows give (p(f) - 2^f) / 2^f + 1
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        w = w * np.abs(V @ c - 1.0)
        w /= w.sum()
    c32 = c.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(deg - 1, -1, -1):
        p = p * f.astype(np.float32) + c32[k]
    return c32, float(np.max(np.abs(p.astype(np.float64) / y - 1.0)))


if __name__ == "__main__":
    c, err = fit(3)
    print("coefficients (c0..c3):", [float(v) for v in c])
    print("max relative error of the fp32 Horner evaluation:", err)
