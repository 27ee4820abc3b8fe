"""Coefficients of the polynomial 2^f ~ p(f) on f in [-1/2, 1/2] used by the
forward kernel to compute part of its exponentials on the FMA pipe.

Method: the argument of 2^x is split Cody-Waite style into x = n + f with
n = round(x) (so |f| <= 1/2) and 2^x = 2^n * p(f), where 2^n is applied by
adding n to the float's exponent field.  p is fitted for minimum *relative*
error with p(0) = 1 exactly, by Lawson's iteratively reweighted least squares
(which converges to the minimax fit) on a dense grid, in float64.

Run: python exp2_poly_fit.py [degree]   (prints C++ constants and the error)
"""

import sys

import numpy as np


def fit(degree=4, n=20001, iters=200):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    # p(f) = 1 + sum_{k>=1} c_k f^k, fitted to 2^f with relative weighting
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    coeffs = np.concatenate([[1.0], c])
    p = np.polyval(coeffs[::-1], f)
    rel = np.abs(p / y - 1.0).max()
    # the same evaluation in float32 Horner form, as the kernel does it
    c32 = coeffs.astype(np.float32)
    f32 = f.astype(np.float32)
    acc = np.full_like(f32, c32[-1])
    for k in range(degree - 1, -1, -1):
        acc = (acc * f32 + c32[k]).astype(np.float32)
    rel32 = np.abs(acc.astype(np.float64) / y - 1.0).max()
    return coeffs, rel, rel32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    coeffs, rel, rel32 = fit(deg)
    print(f"// degree {deg}: max relative error {rel:.3e} (float64), {rel32:.3e} (float32 Horner)")
    for k, c in enumerate(coeffs):
        print(f"constexpr float kExp2C{k} = {float(np.float32(c)):.9g}f;  // {c:.17g}")
