"""Block informativeness scores (oracle).

Jenga notes §4.2 / Jenga summary §4.2.1 Eq. (1): a token's informativeness is the
sum over all other tokens i of its interaction S_ij with them.  §4.2.2 (Fig. 6):
scores are aggregated across heads, partitioned into b x b score blocks, and §4.2.3
sums score blocks down a key-block column, B^T_n = sum_m B^S_mn, to give one score per
token block.

Reading used for the primary mode (``softmax_mass``): S_ij is the causal softmax
attention probability of query i on key j (the pages say the scores pass through
softmax), the diagonal i == j is included (so each query row sums to 1 and the
total mass is the number of queries per head), heads are summed without the
1/N_head factor, and the per-token values are summed over the tokens of each key
block.  This is Eq. (1) with softmax probabilities, summed over the block.

``paper_blockmax`` is Eq. (2) literally: for every (query block m, key block n) the
maximum over causal entries (i >= j) of sum_h max(S^h_ij, 0) / N_head, with raw
scaled logits S^h_ij = q_i . k_j / sqrt(D); then B^T_n = sum_m I(B^S_mn) over the
query blocks that have at least one causal entry in column n.
"""
import numpy as np


def _as_f64(a):
    return np.asarray(a, dtype=np.float64)


def head_column_mass(args):
    """Softmax column mass of ONE head: args = (qh [S, D], kh [S, D], causal, chunk).

    Returns [S] with mass[j] = sum_i P_ij, P_i. = softmax_j(q_i . k_j / sqrt(D)) over
    j <= i (all j if not causal).  The softmax is the textbook one (subtract the row max,
    exponentiate, divide by the row sum); rows are processed in chunks only to bound
    memory, and a causal chunk of rows [i0, i1) only forms the keys j < i1 (the others
    have probability exactly 0)."""
    qh, kh, causal, chunk = args
    qh = _as_f64(qh)
    kh = _as_f64(kh)
    S, D = qh.shape
    scale = 1.0 / np.sqrt(D)
    mass = np.zeros(S, dtype=np.float64)
    for i0 in range(0, S, chunk):
        i1 = min(S, i0 + chunk)
        kend = i1 if causal else S
        s = (qh[i0:i1] @ kh[:kend].T) * scale            # [c, kend]
        if causal:  # keys j < i0 are visible to every row of the chunk: mask the diagonal block
            ii = np.arange(i0, i1)[:, None]
            s[:, i0:] = np.where(np.arange(i0, kend)[None, :] <= ii, s[:, i0:], -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        p /= p.sum(axis=1, keepdims=True)
        mass[:kend] += p.sum(axis=0)
    return mass


def column_mass(q, k, causal=True, chunk=512, pmap=map):
    """Per-key softmax column mass, summed over heads (in head order).

    q, k: [S, H, D].  Returns [S] with mass[j] = sum_h sum_i P^h_ij (``head_column_mass``
    per head).  ``pmap`` maps the per-head function over the heads (the builtin ``map`` by
    default; a process pool's ``map`` gives the same result, since heads are independent)."""
    q = _as_f64(q)
    k = _as_f64(k)
    S, H, D = q.shape
    mass = np.zeros(S, dtype=np.float64)
    tasks = [(np.ascontiguousarray(q[:, h, :]), np.ascontiguousarray(k[:, h, :]), causal, chunk) for h in range(H)]
    for mh in pmap(head_column_mass, tasks):
        mass += mh
    return mass


def block_scores_softmax_mass(q, k, blk, causal=True, pmap=map):
    """Score of each token block: sum of ``column_mass`` over the block's keys.

    q, k: [S, H, D] (one sequence) or [B, S, H, D].  S must be a multiple of blk.
    Returns [nb] or [B, nb] float64.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    if q.ndim == 4:
        return np.stack([block_scores_softmax_mass(q[b], k[b], blk, causal, pmap) for b in range(q.shape[0])])
    S = q.shape[0]
    assert S % blk == 0
    mass = column_mass(q, k, causal, pmap=pmap)
    return mass.reshape(S // blk, blk).sum(axis=1)


def block_scores_paper_blockmax(q, k, blk, causal=True):
    """Eq. (2) + §4.2.3 aggregation (see module docstring).  q, k: [S, H, D]."""
    q = _as_f64(q)
    k = _as_f64(k)
    if q.ndim == 4:
        return np.stack([block_scores_paper_blockmax(q[b], k[b], blk, causal) for b in range(q.shape[0])])
    S, H, D = q.shape
    nb = S // blk
    scale = 1.0 / np.sqrt(D)
    out = np.zeros(nb, dtype=np.float64)
    for m in range(nb):
        rows = slice(m * blk, (m + 1) * blk)
        agg = np.zeros((blk, S), dtype=np.float64)
        for h in range(H):
            s = (q[rows, h, :] @ k[:, h, :].T) * scale
            agg += np.maximum(s, 0.0)
        agg /= H
        ii = np.arange(m * blk, (m + 1) * blk)[:, None]
        valid = (np.arange(S)[None, :] <= ii) if causal else np.ones_like(agg, dtype=bool)
        for n in range(nb):
            cols = slice(n * blk, (n + 1) * blk)
            v = valid[:, cols]
            if v.any():
                out[n] += agg[:, cols][v].max()
    return out


def row_lse(qh, kh, rows, causal=True):
    """Natural log-sum-exp of the scaled logits of the given query rows of ONE head:
    lse_i = log sum_{j <= i} exp(q_i . k_j / sqrt(D)) (all j if not causal), with the
    textbook max shift.  qh, kh: [S, D]; rows: query indices.  Returns [len(rows)]."""
    qh = _as_f64(qh)
    kh = _as_f64(kh)
    S, D = qh.shape
    out = np.zeros(len(rows))
    for n, i in enumerate(rows):
        kend = int(i) + 1 if causal else S
        s = (kh[:kend] @ qh[int(i)]) / np.sqrt(D)
        m = s.max()
        out[n] = m + np.log(np.exp(s - m).sum())
    return out
