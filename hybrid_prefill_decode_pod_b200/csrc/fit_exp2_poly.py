"""Fit the polynomial used by pod_exp2.cuh: p(f) ~ 2^f on f in [-0.5, 0.5].

Method: iteratively reweighted least squares on Chebyshev points, weighting by
relative error, which converges towards the minimax (equiripple) relative-error
fit. Prints the fp32 coefficients c0..c3 (p = c0 + c1 f + c2 f^2 + c3 f^3) and
the worst relative error on a dense grid. Run: python fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, iters=60):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = 2.0 ** f
    w = 1.0 / y
    for _ in range(iters):
        A = np.vander(f, deg + 1, increasing=True) * w[:, None]
        c, *_ = np.linalg.lstsq(A, y * w, rcond=None)
        err = (np.polyval(c[::-1], f) - y) / y
        w = w * (1.0 + 4.0 * np.abs(err) / np.abs(err).max())
    c32 = np.array(c, dtype=np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    worst = np.abs(np.polyval(c32.astype(np.float64)[::-1], grid) / 2.0 ** grid - 1.0).max()
    return c32, worst


if __name__ == "__main__":
    c, worst = fit()
    for i, x in enumerate(c):
        print("c%d = %.9ef" % (i, x))
    print("max relative error on [-0.5, 0.5]: %.3e" % worst)
