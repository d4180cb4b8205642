"""Causal-LM loss over the vocabulary (oracle) -- TEST INFRASTRUCTURE ONLY.

Jenga summary §4.4.2 (segment-based peak cutting, Fig. 10): for every token the model
produces a next-token distribution over the whole vocabulary and the loss compares it
with the true next token; with a large vocabulary and a long context these transient
activations make the memory peak.  The pages' remedy processes the token sequence in
smaller segments, one after the other, dropping each segment's activations once its
gradient is computed.  That changes only the memory peak, not the result, so the
oracle is the unsegmented definition:

  logits_t = hidden_t . W^T                    (W [V, h], the frozen output embedding)
  loss     = (1 / n) sum_{t valid} ( logsumexp(logits_t) - logits_t[label_t] )
  dhidden_t = (1 / n) (softmax(logits_t) - onehot(label_t)) . W   for valid t, else 0

with valid tokens 0 <= label_t < V (any other label, e.g. -100, is ignored) and n the
number of valid tokens (the mean reduction of the usual cross-entropy).  Reading for the
unstated points: mean over valid tokens; labels are the already-shifted next-token ids;
only the hidden-state gradient is formed (the output embedding is frozen, as the base
weights are in LoRA fine-tuning).  float64 throughout.
"""
import numpy as np


def _valid(labels, V):
    labels = np.asarray(labels, dtype=np.int64)
    return (labels >= 0) & (labels < V)


def lm_loss(hidden, w, labels, rows=None):
    """(loss, dhidden) for hidden [S, h], w [V, h], labels [S] (see module docstring).

    ``rows`` (optional index array) restricts dhidden to those rows (returned as
    [len(rows), h]); the loss is always over all rows.
    """
    hidden = np.asarray(hidden, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    V = w.shape[0]
    labels = np.asarray(labels, dtype=np.int64)
    valid = _valid(labels, V)
    n = int(valid.sum())
    total = 0.0
    S = hidden.shape[0]
    want = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    dh = np.zeros((want.size, hidden.shape[1]), dtype=np.float64)
    pos = {int(r): i for i, r in enumerate(want)}
    chunk = 256  # rows at a time only to bound memory
    for c0 in range(0, S, chunk):
        z = hidden[c0:c0 + chunk] @ w.T                      # [c, V]
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        ssum = e.sum(axis=1, keepdims=True)
        lse = (m + np.log(ssum))[:, 0]
        for i in range(z.shape[0]):
            t = c0 + i
            if not valid[t]:
                continue
            total += lse[i] - z[i, labels[t]]
            if t in pos:
                p = e[i] / ssum[i, 0]
                p[labels[t]] -= 1.0
                dh[pos[t]] = (p / n) @ w
    loss = total / n if n > 0 else 0.0
    return loss, dh
