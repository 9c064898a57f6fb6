"""Coefficients of the cubic that approximates 2^f on [-1/2, 1/2] in
exp2_poly() (csrc/sm100.cuh).

Method: weighted least squares of the relative error on Chebyshev nodes of the
interval, followed by a few iterations of Lawson's algorithm (iteratively
re-weighted least squares), which drives the fit towards the minimax
(equioscillating) relative-error polynomial.  The constant term is pinned to 1
so that 2^0 is exact.  Run as a script to print the coefficients and the
maximum relative error on a dense grid.
"""

import numpy as np


def fit(degree: int = 3, nodes: int = 2000, iters: int = 60):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)       # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    # p(f) = 1 + c1 f + ... ; relative residual (p - y) / y
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    w = np.ones(nodes)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * (r + 1e-18)
        w /= w.sum()
    return np.concatenate([[1.0], c])


def max_rel_error(coef, points: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, points)
    p = np.polyval(coef[::-1], f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    print("coefficients (c0..c3):", ", ".join(f"{float(x):.9e}f" for x in c32))
    print("max relative error (fp64 coefficients):", max_rel_error(c))
    print("max relative error (fp32 coefficients):", max_rel_error(c32.astype(np.float64)))
