"""Fit the degree-3 polynomial the kernels use for 2^f on f in [-1/2, 1/2].

    python -m exact_tiled_attention_42_b200.fit_exp2_poly

Iteratively reweighted least squares on Chebyshev-spaced points, weighting
toward the points of largest relative error (Lawson's method), then rounding
the coefficients to float32. Prints the coefficients (as C float literals) and
the resulting maximum relative error over a dense grid. The kernels'
exp2_poly (csrc/common.cuh) holds the printed values.
"""

import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = w / y
        c, *_ = np.linalg.lstsq(a * sw[:, None], y * sw, rcond=None)
        err = np.abs(a @ c - y) / y
        w = w * np.sqrt(err / err.max()) + 1e-12
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error(c32) -> float:
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(f)
    for coef in c32[::-1]:
        p = p * f + float(coef)
    return float(np.max(np.abs(p - np.exp2(f)) / np.exp2(f)))


if __name__ == "__main__":
    c = fit()
    for i, v in enumerate(c):
        print(f"C{i} = {float(v).hex()}  ({float(v):.9g}f)")
    print("max relative error", max_rel_error(c))
