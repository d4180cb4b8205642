"""Block selection (oracle).

Jenga notes §4.2 ("layer-specific threshold") / Jenga summary §4.2.3 and Algorithm 1:
each token block's score B^T_n is compared with a layer threshold T_i; blocks that
clear it are kept, the rest are eliminated.  Algorithm 1 step 1 initialises T_i to
the average block score of the layer.

Modes (readings stated where the pages are silent):

* ``mean_ge``  - T = average block score (Algorithm 1, step 1); keep n iff
  score[n] >= T.  The average is the float64 sum in index order divided by nb;
  each fp32 score is compared as float64.
* ``topk``     - keep exactly k blocks, ranked by (score descending, block index
  ascending) -- the tie-break is a reading (the pages do not discuss ties).
* ``abs_ge``   - keep n iff score[n] >= a given threshold (fp32 compare).

``topk_count(p, nb)`` turns a keep fraction p into k = ceil(p * nb - 1e-6), clamped
to [0, nb] ("keep at least a fraction p", with a 1e-6 guard so that fractions
written in decimal, e.g. 0.3 * 10, do not round up by one).

NaN scores compare as -inf (never kept by a threshold, ranked last by top-k).
Outputs: ascending kept block indices (padded with -1 to nb), the count, and a
0/1 mask.
"""
import math

import numpy as np


def topk_count(p, nb):
    k = math.ceil(float(p) * nb - 1e-6)
    return max(0, min(nb, k))


def _clean(scores):
    s = np.asarray(scores, dtype=np.float32).astype(np.float64)
    return np.where(np.isnan(s), -np.inf, s)


def _pack(keep):
    nb = keep.shape[0]
    idx = np.full(nb, -1, dtype=np.int32)
    kept = np.nonzero(keep)[0].astype(np.int32)
    idx[:kept.size] = kept
    return idx, int(kept.size), keep.astype(np.uint8)


def select_mean_ge(scores):
    s = _clean(scores)
    total = 0.0
    for v in s:                      # float64, index order
        total += v
    mean = total / s.shape[0]
    return _pack(s >= mean), mean


def select_abs_ge(scores, threshold):
    s = _clean(scores)
    thr = float(np.float32(threshold))
    return _pack(s >= thr)


def select_topk(scores, k):
    s = _clean(scores)
    nb = s.shape[0]
    order = sorted(range(nb), key=lambda n: (-s[n], n))
    keep = np.zeros(nb, dtype=bool)
    for n in order[:k]:
        keep[n] = True
    return _pack(keep)


def select(scores, mode, param):
    """Batched front end: scores [B, nb] -> idx [B, nb], n_kept [B], mask [B, nb]."""
    scores = np.atleast_2d(scores)
    B, nb = scores.shape
    idx = np.zeros((B, nb), np.int32)
    nk = np.zeros(B, np.int32)
    mask = np.zeros((B, nb), np.uint8)
    for b in range(B):
        if mode == "mean_ge":
            (i, n, m), _ = select_mean_ge(scores[b])
        elif mode == "topk_frac":
            i, n, m = select_topk(scores[b], topk_count(param, nb))
        elif mode == "topk":
            i, n, m = select_topk(scores[b], int(param))
        elif mode == "abs_ge":
            i, n, m = select_abs_ge(scores[b], param)
        else:
            raise ValueError(mode)
        idx[b], nk[b], mask[b] = i, n, m
    return idx, nk, mask
