"""Fit the cubic used by the attention kernel to evaluate 2^f on the FMA pipe.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-0.5, 0.5].  This script
finds the degree-3 polynomial p(f) minimising the maximum RELATIVE error of p(f) against
2^f on that interval (Lawson's iteratively reweighted least squares, which converges to the
minimax fit), rounds the coefficients to float32 and reports the error of the float32
polynomial.  The attention kernel rounds P to bf16 (8 significand bits), so a relative error
near 1e-4 is far below what the result can represent.

Usage: python block_sparse_attention_31_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(degree: int = 3, iters: int = 400, n: int = 20001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones(n) / n
    coef = None
    for _ in range(iters):
        sw = np.sqrt(w) / y                      # relative-error weighting
        coef, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ coef - y) / y
        w = w * err
        w /= w.sum()
    return coef


def float32_error(coef32, n: int = 200001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.zeros_like(f)
    for c in coef32[::-1]:                       # Horner in float32, as on the device
        p = (p * f + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    print("coefficients (c0 + c1 f + c2 f^2 + c3 f^3):")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v)!r:>24}f  ({float(v).hex()})")
    print(f"max relative error of the float32 cubic on [-0.5, 0.5]: {float32_error(c32):.3e}")
