"""Fit the degree-3 polynomial the kernels use for 2^f on f in [-1/2, 1/2].

    python -m exact_tiled_attention_42_b200.fit_exp2_poly

The constant term is fixed at 1, so 2^0 is exactly 1: a row's largest score
has x = 0 exactly, and P = 1 must stay 1 (a block weight times P can sit on an
e4m3 rounding tie, where 1 - 7e-5 and 1 round apart). The other three
coefficients come from iteratively reweighted least squares on
Chebyshev-spaced points, weighting toward the points of largest relative error
(Lawson's method), rounded to float32. Prints the coefficients (as C float
literals) and the resulting maximum relative error over a dense grid. The
kernels' exp2_poly (csrc/common.cuh) holds the printed values.
"""

import numpy as np


def fit(degree: int = 3, iters: int = 200):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True)[:, 1:]   # f, f^2, f^3: the constant term is 1
    w = np.ones_like(f)
    for _ in range(iters):
        sw = w / y
        c, *_ = np.linalg.lstsq(a * sw[:, None], (y - 1.0) * sw, rcond=None)
        err = np.abs(1.0 + a @ c - y) / y
        w = w * np.sqrt(err / err.max()) + 1e-12
        w /= w.sum()
    return np.concatenate([[1.0], c]).astype(np.float32)


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
