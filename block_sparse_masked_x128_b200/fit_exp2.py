"""Fit of the degree-3 polynomial behind exp2_fma2 (csrc/sm100_ptx.cuh).

exp2_fma2 computes 2^a as 2^n * p(f) with n = round(a) and f = a - n in [-1/2, 1/2].  The
coefficients of p minimise the maximum RELATIVE error |p(f) - 2^f| / 2^f on that interval.
They come from Lawson's algorithm: weighted least squares on a dense grid, where after each
solve every point's weight is multiplied by its current error, which drives the solution to
the minimax (equi-oscillating) one.  Run this file to print the coefficients and their error.
"""
import numpy as np


def fit(degree: int = 3, points: int = 20001, iterations: int = 200):
    x = np.linspace(-0.5, 0.5, points)
    y = np.exp2(x)
    A = np.vstack([x ** k for k in range(degree + 1)]).T
    w = np.ones_like(x)
    for _ in range(iterations):
        sw = np.sqrt(w) / y                      # relative error: divide each row by 2^x
        c, *_ = np.linalg.lstsq(A * sw[:, None], y * sw, rcond=None)
        err = np.abs(A @ c - y) / y
        w = w * err
        w /= w.sum()
    return c, float((np.abs(A @ c - y) / y).max())


if __name__ == "__main__":
    coeffs, rel = fit()
    for i, c in enumerate(coeffs):
        print(f"kExp2C{i} = {c:.16f}")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
