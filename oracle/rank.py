"""Rank agreement between predicted and exact block scores (oracle).

Jenga notes §6 (predictor evaluation) / Jenga summary §6: the predictors are judged
by how well they recover the exact informative blocks (recall).  With untrained
random weights the paper's recall value cannot be reproduced, so this module only
defines the statistics: Spearman's rho (Pearson correlation of average ranks),
Kendall's tau-b, and the recall of the exact top-k set inside the predicted top-k
set (ties broken by block index).
"""
import numpy as np


def average_ranks(a):
    """Ranks 1..n, tied values sharing the mean of their positions."""
    a = np.asarray(a, np.float64)
    order = sorted(range(a.size), key=lambda i: a[i])
    ranks = np.zeros(a.size)
    i = 0
    while i < a.size:
        j = i
        while j + 1 < a.size and a[order[j + 1]] == a[order[i]]:
            j += 1
        avg = (i + j) / 2.0 + 1.0
        for t in range(i, j + 1):
            ranks[order[t]] = avg
        i = j + 1
    return ranks


def spearman(a, b):
    ra, rb = average_ranks(a), average_ranks(b)
    ra -= ra.mean()
    rb -= rb.mean()
    den = np.sqrt((ra * ra).sum() * (rb * rb).sum())
    return float((ra * rb).sum() / den) if den > 0 else float("nan")


def kendall_tau_b(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    n = a.size
    conc = disc = ties_a = ties_b = 0
    for i in range(n):
        for j in range(i + 1, n):
            da = np.sign(a[i] - a[j])
            db = np.sign(b[i] - b[j])
            if da == 0 and db == 0:
                continue
            if da == 0:
                ties_a += 1
            elif db == 0:
                ties_b += 1
            elif da == db:
                conc += 1
            else:
                disc += 1
    den = np.sqrt((conc + disc + ties_a) * (conc + disc + ties_b))
    return float((conc - disc) / den) if den > 0 else float("nan")


def topk_set(a, k):
    a = np.asarray(a, np.float64)
    order = sorted(range(a.size), key=lambda i: (-a[i], i))
    return set(order[:k])


def topk_recall(pred, exact, k):
    """|topk(exact) & topk(pred)| / k."""
    if k == 0:
        return 1.0
    return len(topk_set(exact, k) & topk_set(pred, k)) / k
