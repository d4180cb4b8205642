"""Permutation-free token movement (oracle).

Jenga notes §4.4 / Jenga summary §4.4.1 (Fig. 9): retained tokens are read straight
from the original input, and the sub-block output is added in place into the
original input rows (padding and residual add in one step); eliminated rows are
untouched.  Here the two halves are written as plain row copies.

Row expansion: kept block b covers token rows [b*blk, (b+1)*blk); the retained row
list is the concatenation over the ascending kept blocks.
"""
import numpy as np


def retained_rows(idx, n_kept, blk):
    idx = np.asarray(idx)[: int(n_kept)].astype(np.int64)
    return (idx[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)


def gather(x, idx, n_kept, blk):
    """out[t] = x[row(t)] for the retained rows; x is [S, h]."""
    return np.array(x[retained_rows(idx, n_kept, blk)], copy=True)


def scatter_add(x, y, idx, n_kept, blk, alpha, dtype):
    """x[row(t)] <- round_dtype(x[row(t)] + alpha * y[t]); other rows unchanged.

    ``dtype`` is "f32" or "bf16"; the sum is formed in float64 and rounded once to
    fp32 (then, for bf16 storage, to bf16).  x and y hold the stored values as
    float64.  Returns a new array.
    """
    from .bf16 import round_bf16, round_f32
    out = np.array(x, dtype=np.float64, copy=True)
    rows = retained_rows(idx, n_kept, blk)
    s = round_f32(out[rows] + float(np.float32(alpha)) * np.asarray(y, np.float64)[: rows.size])
    if dtype == "bf16":
        s = round_bf16(s)
    out[rows] = s
    return out
