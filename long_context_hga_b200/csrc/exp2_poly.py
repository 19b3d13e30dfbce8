"""Fits the polynomial behind tc::exp2_fma2 (tc.cuh): 2^f on [-1/2, 1/2].

Method: least squares, relative-error weighted, on Chebyshev nodes of the
interval (a near-minimax fit), for the Cody-Waite style reduction
2^x = 2^j * 2^f, j = round(x) (W. J. Cody and W. Waite, "Software Manual for
the Elementary Functions", 1980).  Prints the float32 coefficients (constant
term first) and the worst relative error of float32 Horner evaluation.

    python long_context_hga_b200/csrc/exp2_poly.py [degree]
"""
import sys

import numpy as np


def fit(deg: int, n: int = 4000):
    k = np.arange(n)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n)
    y = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    c32 = c.astype(np.float32)
    xs = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    acc = np.full_like(xs, c32[-1])
    for cc in c32[-2::-1]:
        acc = (acc * xs + cc).astype(np.float32)
    err = np.abs(acc.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1).max()
    return c32, err


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, err = fit(deg)
    print("coefficients:", ", ".join(f"{float(x):.9g}f" for x in c))
    print(f"max relative error (float32 Horner): {err:.3e}")
