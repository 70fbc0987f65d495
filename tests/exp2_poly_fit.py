"""Derive the coefficients of the FMA-pipe exp2 used by the prefill softmax.

Method (Cody & Waite style argument reduction): x = n + f with n = round(x)
and f in [-1/2, 1/2]; 2^x = 2^n * 2^f, where 2^n is applied by adding n to
the float's exponent field and 2^f is a cubic polynomial. The cubic is fitted
here by weighted least squares on Chebyshev nodes, minimising the relative
error, then refined by a few Lawson (iteratively reweighted) steps towards the
minimax solution. The probabilities it produces are rounded to bf16 (relative
step 2^-8), so a relative error near 1e-4 is far below what is kept.

Run: python tests/exp2_poly_fit.py  -> prints the coefficients c0..c3 and the max
relative error over [-1/2, 1/2].
"""

import numpy as np


def fit(degree=3, n_nodes=2000, lawson_steps=200):
    k = np.arange(n_nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n_nodes)          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(lawson_steps):
        W = w / target                                          # relative error weighting
        c, *_ = np.linalg.lstsq(V * W[:, None], target * W, rcond=None)
        err = np.abs(V @ c / target - 1.0)
        w = w * err / (w * err).sum() * len(f) + 1e-12
    grid = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0).max()
    return c, rel


if __name__ == "__main__":
    c, rel = fit()
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}  # {ci:.17g}")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
