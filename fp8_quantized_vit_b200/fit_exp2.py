"""Fit the polynomial the attention kernel uses for part of its exp2 work.

2^x = 2^n * 2^f with n = rint(x) and f = x - n in [-0.5, 0.5] (Cody-Waite
range reduction).  2^f is approximated by a polynomial whose coefficients
minimise the maximum RELATIVE error on [-0.5, 0.5] (Lawson's iteratively
reweighted least squares converging to the minimax fit), then rounded to
fp32.  Run: python -m fp8_quantized_vit_b200.fit_exp2 [degree]
"""
import sys

import numpy as np


def fit(degree: int = 3, iters: int = 400, npts: int = 4001):
    f = np.cos(np.linspace(np.pi, 0.0, npts)) * 0.5  # Chebyshev-spaced nodes
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error
    b = np.ones_like(f)
    w = np.ones_like(f) / npts
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 200001)
    approx = np.polyval(c32[::-1].astype(np.float64), fine)
    rel = np.abs(approx / np.exp2(fine) - 1.0).max()
    return c32, rel


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, rel = fit(deg)
    print("coefficients (c0..c%d):" % deg, ", ".join(f"{float(v)!r}f" for v in c))
    print("max relative error on [-0.5, 0.5]: %.3e (2^%.2f)" % (rel, np.log2(rel)))
