"""Derive the cubic used by the forward kernel's software exp2 (attn_fwd.cuh, exp2_poly).

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is replaced by a cubic
c0 + c1 f + c2 f^2 + c3 f^3. The coefficients minimise the maximum relative error on [-1/2, 1/2]: a
least-squares start on Chebyshev nodes refined by iterative reweighting (Lawson's method). Run this file to
reprint them and the error bound; the kernel's constants were copied from its output.
"""
import numpy as np


def fit(degree=3, iters=200):
    f = np.cos(np.linspace(0, np.pi, 4001)) * 0.5           # Chebyshev-spaced points on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]  # relative-error design matrix
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * np.sqrt(w)[:, None], np.sqrt(w), rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * (err + 1e-30)
        w /= w.sum()
    return c


if __name__ == "__main__":
    c = fit()
    grid = np.linspace(-0.5, 0.5, 200001)
    p = np.polynomial.polynomial.polyval(grid, c)
    print("coefficients:", ", ".join(f"{x:.9g}f" for x in c))
    print("max relative error on [-1/2, 1/2]: %.3e" % np.max(np.abs(p / np.exp2(grid) - 1)))
