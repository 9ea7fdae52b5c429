"""Fits the polynomial used for the FMA-pipe share of exp2 in the softmax.

Method: Cody-Waite style range reduction, x = n + f with n = round(x) and
f in [-1/2, 1/2], so 2^x = 2^n * 2^f; 2^n is applied by adding n to the
exponent field.  2^f is approximated by a cubic p(f) fitted here by weighted
least squares of the relative error on 2001 Chebyshev nodes of [-1/2, 1/2]
(numpy.linalg.lstsq), with p(0) = 1 imposed so that exact-max entries give
exactly 1.  The kernel stores P in bf16 (relative step 2^-8), so a relative
error of a few 1e-5 is far below the rounding P receives anyway.

Run: python fit_exp2_poly.py  -> prints the coefficients c1, c2, c3 and the
max relative error; the constants in attn_kernel.cuh are these values.
"""

import numpy as np


def fit(degree: int = 3, nodes: int = 2001):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    # p(f) = 1 + c1 f + c2 f^2 + c3 f^3; minimise sum(((p - y) / y)^2)
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    return c


def max_rel_error(c, n: int = 200001):
    f = np.linspace(-0.5, 0.5, n)
    p = 1.0 + sum(ci * f ** (i + 1) for i, ci in enumerate(c))
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients:", ", ".join(f"{x:.9e}" for x in c))
    print("float32:", ", ".join(repr(float(np.float32(x))) for x in c))
    print("max relative error:", max_rel_error(c))
