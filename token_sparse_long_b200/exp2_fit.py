"""Coefficients of the cubic behind the FMA-pipe exponential (exp2_fma in csrc/common.cuh).

2^x is split as 2^j * 2^f with j the integer nearest x and |f| <= 1/2.  2^j goes straight
into the float's exponent field; 2^f comes from a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose
relative error is made equal-ripple (minimax) on [-1/2, 1/2] by Lawson's iteratively
reweighted least squares on Chebyshev nodes.  Result: max relative error 7.48e-5 in float64,
and the same in float32 evaluation.

    python -m token_sparse_long_b200.exp2_fit
"""
import numpy as np


def fit(deg=3, nodes=4001, iters=400):
    f = np.cos(np.linspace(0.0, np.pi, nodes)) * 0.5
    y = 2.0 ** f
    a = np.vander(f, deg + 1, increasing=True) / y[:, None]  # relative-error design matrix
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], sw, rcond=None)
        e = np.abs(a @ c - 1.0)
        w = w * e
        w /= w.sum()
    return c


def max_rel_err_f32(c):
    c32 = np.asarray(c, dtype=np.float32)
    fx = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(fx)
    for ci in c32[::-1]:
        p = p * fx + ci
    return float(np.abs(p.astype(np.float64) / 2.0 ** fx.astype(np.float64) - 1.0).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", [float(np.float32(x)).hex() for x in c])
    print("max relative error (float32 evaluation): %.3e" % max_rel_err_f32(c))
