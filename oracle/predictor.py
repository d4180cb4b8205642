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


# ------------------------------------------------------------------ Q/K predictor pair
# Jenga summary §4.3.1 Eq. (3) and Fig. 8: each layer has a pair of predictors, one for
# the query side and one for the key side.  Each is three trainable low-rank matrices
# with ReLU between consecutive ones; its input is the block-organised embedding X (one
# representative embedding per block) and its output the block's approximate
# informativeness.  The score-block informativeness is the product
#     I(B^S_mn) = I(B^Q_m) I(B^K_n)^T,
# and (§4.2.3) a key block's score is the sum of its column of score blocks.
# Readings of the unstated points: the representative embedding is the block mean of the
# raw layer input (as for the single-MLP predictor above); the matrices carry no biases;
# the predictor outputs are d-vectors (d = 1 gives scalar informativeness), so I(B^S_mn)
# is their dot product; with causal attention only query blocks m >= n contribute to key
# block n.

def predictor_pair_side(xb, w1, w2, w3):
    """One side: W3 ReLU(W2 ReLU(W1 xbar)) for every block.  xb [nb, h] -> [nb, d]."""
    a = np.maximum(xb @ np.asarray(w1, np.float64).T, 0.0)
    a = np.maximum(a @ np.asarray(w2, np.float64).T, 0.0)
    return a @ np.asarray(w3, np.float64).T


def predict_blocks_qk(x, blk, q_w, k_w, causal=True):
    """x [S, h]; q_w, k_w: (W1 [r1, h], W2 [r2, r1], W3 [d, r2]) -> scores [nb] (float64).

    The nb x nb score-block matrix I(B^S) = Qhat Khat^T is formed explicitly and summed
    down its columns (causal: rows m >= n only)."""
    xb = block_means(x, blk)
    qh = predictor_pair_side(xb, *q_w)
    kh = predictor_pair_side(xb, *k_w)
    blocks = qh @ kh.T                      # [m, n]
    nb = blocks.shape[0]
    if causal:
        blocks = np.where(np.arange(nb)[:, None] >= np.arange(nb)[None, :], blocks, 0.0)
    return blocks.sum(axis=0)
