"""Provenance of the cubic behind the FMA-pipe exponential (exp2_fma in csrc/common.cuh).

2^x is split as 2^j * 2^f with j the integer nearest x and |f| <= 1/2; 2^j goes into the
float's exponent field and 2^f comes from a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose relative
error is made equal-ripple (minimax) on [-1/2, 1/2] by Lawson's iteratively reweighted least
squares on Chebyshev nodes (C. L. Lawson, 1961; see also J.-M. Muller, "Elementary
Functions", on minimax polynomial approximation).  This test refits the cubic and checks
that the four constants compiled into the kernels are that fit, rounded to float32, and
that their float32 evaluation keeps the stated 7.5e-5 relative error bound."""
import os
import re

import numpy as np

CUH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "token_sparse_long_b200", "csrc",
                   "common.cuh")


def lawson_minimax_rel(deg=3, nodes=4001, iters=400):
    f = np.cos(np.linspace(0.0, np.pi, nodes)) * 0.5
    y = 2.0 ** f
    a = np.vander(f, deg + 1, increasing=True) / y[:, None]  # relative-error design matrix
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], sw, rcond=None)
        w = w * np.abs(a @ c - 1.0)
        w /= w.sum()
    return c


def max_rel_err_f32(c):
    c32 = np.asarray(c, dtype=np.float32)
    fx = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(fx)
    for ci in c32[::-1]:
        p = (p * fx + ci).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** fx.astype(np.float64) - 1.0).max())


def kernel_constants():
    """c0..c3 as written in exp2_fma (the Horner chain starts from c3 f + c2)."""
    src = open(CUH).read()
    body = src[src.index("__device__ __forceinline__ float exp2_fma("):]
    body = body[:body.index("return")]
    hexes = re.findall(r"0x1\.[0-9a-f]+p-?\d+f", body)
    vals = [float.fromhex(h[:-1]) for h in hexes]
    c3, c2, c1, c0 = vals[0], vals[1], vals[2], vals[3]
    return np.array([c0, c1, c2, c3])


def test_kernel_cubic_is_the_lawson_fit():
    fit = lawson_minimax_rel()
    got = kernel_constants()
    assert np.allclose(got, fit.astype(np.float32).astype(np.float64), rtol=2e-6, atol=0), (got, fit)


def test_kernel_cubic_error_bound():
    assert max_rel_err_f32(kernel_constants()) < 7.5e-5
    # equal ripple: the minimax error of a cubic for 2^f on [-1/2, 1/2] is not much smaller
    assert max_rel_err_f32(kernel_constants()) > 6e-5
