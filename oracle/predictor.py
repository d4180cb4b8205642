"""Block-score predictor MLP (oracle).

Jenga notes §4.3 / Jenga summary §4.3.1 (Fig. 8): lightweight per-layer predictors
take block-organised token embeddings X, extract a representative embedding per
block and output an approximate informativeness score per block; the predictor is
sized to one block, not to the whole sequence.

Form used here (a reading: the pages' predictor is three low-rank matrices with
ReLU per Q/K side; this is the single-MLP block-score form): the representative
embedding of block n is the mean of the block's raw layer-input rows,
    xbar_n = (1/blk) sum_{t in block n} x_t,
and the score is s_n = W2 . GELU(W1 xbar_n + b1) + b2 with W1 [m, h], b1 [m],
W2 [1, m], b2 [1], GELU(z) = z * Phi(z) = z/2 (1 + erf(z / sqrt 2)) (exact erf form).
"""
import numpy as np
from scipy.special import erf


def gelu(z):
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def block_means(x, blk):
    x = np.asarray(x, np.float64)
    S, h = x.shape
    return x.reshape(S // blk, blk, h).mean(axis=1)


def predict_blocks(x, blk, w1, b1, w2, b2):
    """x [S, h] -> predicted block scores [S / blk] (float64)."""
    xb = block_means(x, blk)
    hid = gelu(xb @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64)[None, :])
    return (hid @ np.asarray(w2, np.float64).T)[:, 0] + float(np.asarray(b2, np.float64).reshape(-1)[0])
