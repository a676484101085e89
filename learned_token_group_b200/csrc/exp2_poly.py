"""Coefficients of the polynomial 2^f used by the attention softmax.

The attention kernel evaluates part of its exponentials on the FMA pipe
instead of the MUFU unit: t = n + f with n = round(t) and f in [-1/2, 1/2]
(Cody-Waite style range reduction with one rounding step), 2^t = 2^n * p(f),
where p is a degree-3 polynomial fitted to 2^f in the minimax sense for
RELATIVE error by Lawson's iteratively re-weighted least squares on Chebyshev
points.  Run this file to reproduce the constants in ptx.cuh (exp2_poly_x2).
"""
import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    y = np.exp2(f)
    V = np.vstack([f ** k for k in range(degree + 1)]).T
    w = np.ones_like(f)
    c = None
    for it in range(iters):
        W = w / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = (V @ c - y) / y
        if it:
            w = w * np.sqrt(np.abs(err))
        w /= w.sum()
    grid = np.linspace(-0.5, 0.5, 200001)
    rel = (np.vstack([grid ** k for k in range(degree + 1)]).T @ c - np.exp2(grid)) / np.exp2(grid)
    return c, float(np.abs(rel).max())


if __name__ == "__main__":
    c, e = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9g}f" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
