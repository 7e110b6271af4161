"""Coefficients of the degree-3 polynomial the attention softmax uses for part
of its exp2 evaluations (ex2_poly2 in qi21_attn_tc.cuh, every 8th pair of a
row; the rest run on the MUFU unit).

Method: Cody-Waite style argument split 2^x = 2^n * 2^f with n = rint(x),
f = x - n in [-1/2, 1/2]; 2^f is approximated by the cubic that minimises the
relative error in the least-squares sense on 4001 Chebyshev nodes of
[-1/2, 1/2] (weights 1/2^f), with the constant term pinned to 1 so that
2^0 = 1 exactly. Run this file to print the coefficients and the maximum
relative error; the kernel's constants are the printed values rounded to
float32. P is stored in bf16 (relative step 2^-8), so an approximation error
near 1e-4 is far below the rounding that follows.
"""
import numpy as np


def fit(deg=3, n=4001):
    k = np.arange(n)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n)          # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    # y ~ 1 + c1 f + c2 f^2 + c3 f^3, relative error weights 1/y
    A = np.stack([f ** i for i in range(1, deg + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    coef = np.concatenate([[1.0], c])
    g = np.linspace(-0.5, 0.5, 200001)
    approx = np.polyval(coef[::-1], g)
    err = np.max(np.abs(approx / np.exp2(g) - 1.0))
    return coef, err


if __name__ == "__main__":
    coef, err = fit()
    for i, c in enumerate(coef):
        print(f"c{i} = {np.float32(c)!r}")
    print("max relative error", err)
