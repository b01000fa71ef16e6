"""Coefficients of the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the
kernels' FMA-pipe exp2 (2^x = p(x - rint(x)) * 2^rint(x), the range
reduction of Cody and Waite, "Software Manual for the Elementary Functions",
1980).

The fit: least squares in relative error on 2001 Chebyshev nodes of
[-1/2, 1/2], with p(0) pinned to 1 so that 2^n is exact. Run to print the
coefficients and the maximum relative error of the float64 polynomial:
    python exact_tiled_attention_softmax_b200/csrc/gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def fit(degree: int = 3):
    k = np.arange(2001)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / 2001)          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    # p(f) = 1 + c1 f + ... + cd f^d, relative residual (p - 2^f) / 2^f
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / target[:, None]
    rhs = (target - 1.0) / target
    c, *_ = np.linalg.lstsq(A, rhs, rcond=None)
    coeffs = np.concatenate([[1.0], c])
    xs = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(coeffs[::-1], xs)
    err = np.max(np.abs(p / np.exp2(xs) - 1.0))
    return coeffs, err


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coeffs, err = fit(d)
    for i, c in enumerate(coeffs):
        print(f"c{i} = {float(np.float32(c))!r}f")
    print(f"max relative error (float64 evaluation) = {err:.3e}")
