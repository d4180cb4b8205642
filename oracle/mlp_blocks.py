"""MLP-block token elimination criterion (oracle) -- TEST INFRASTRUCTURE ONLY.

Jenga notes §4.2 / Jenga summary §4.2.4 (extend to the MLP block): as with the
attention scores, the informativeness of a token for the MLP block comes from the
block's intermediate activation; for a SiLU-gated MLP that activation is the
elementwise product of the gate projection (after SiLU) and the up projection,
a = SiLU(x Wg^T) * (x Wu^T).  Readings of the unstated points: a token's MLP
informativeness is the sum of |a| over the intermediate neurons (the L1 mass, in the
spirit of the attention-mass score), a token block's score is the sum over its tokens
(as the attention scores are summed over a key block), the criterion runs on the
attention-retained blocks (compact order), and the MLP keeps a subset of them, so the
second index list is the attention list composed with the positions the MLP keeps.
float64 throughout.
"""
import numpy as np


def mlp_block_scores(a, blk, n_kept=None):
    """a [n, F] (rows in compact retained order) -> [n / blk] block scores; blocks at or
    past n_kept (if given) score -inf so that no selection keeps them."""
    a = np.asarray(a, dtype=np.float64)
    n, F = a.shape
    s = np.abs(a).sum(axis=1).reshape(n // blk, blk).sum(axis=1)
    if n_kept is not None:
        s[int(n_kept):] = -np.inf
    return s


def compose_indices(idx_outer, pos, n_pos):
    """out[i] = idx_outer[pos[i]] for i < n_pos, -1 after (the inner list in the outer
    list's numbering)."""
    idx_outer = np.asarray(idx_outer, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    out = np.full(pos.size, -1, dtype=np.int64)
    out[:n_pos] = idx_outer[pos[:n_pos]]
    return out
