"""Pins for oracle.select and oracle.movement (no GPU)."""
from fractions import Fraction
from itertools import combinations

import numpy as np
import pytest

from oracle import movement as omv
from oracle import select as osel
from oracle.bf16 import round_bf16
from synth import gen_score_case, gen_scores


def _brute_topk(s, k):
    # enumerate every k-subset; the answer is the one whose sorted (-score, index)
    # key list is lexicographically smallest
    nb = len(s)
    best = None
    for sub in combinations(range(nb), k):
        key = sorted((-s[i], i) for i in sub)
        if best is None or key < best[0]:
            best = (key, sub)
    return sorted(best[1]) if best else []


@pytest.mark.parametrize("seed,dist", [(0, "normal"), (1, "ties"), (2, "ties"), (3, "normal")])
def test_topk_brute_force(seed, dist):
    sc = gen_scores(seed, 1, 8, dist)[0]
    for k in range(0, 9):
        idx, n, mask = osel.select_topk(sc, k)
        assert n == k
        assert list(idx[:n]) == _brute_topk([float(v) for v in sc], k)
        assert all(idx[n:] == -1)
        assert mask.sum() == k and all(mask[idx[:n]] == 1)


@pytest.mark.parametrize("seed,dist", [(4, "normal"), (5, "ties")])
def test_mean_threshold_exact_rational(seed, dist):
    sc = gen_scores(seed, 1, 7, dist)[0]
    (idx, n, mask), mean = osel.select_mean_ge(sc)
    fr = [Fraction(float(v)) for v in sc]
    m = sum(fr) / len(fr)
    want = [i for i, v in enumerate(fr) if v >= m]
    assert list(idx[:n]) == want
    assert abs(mean - float(m)) <= 1e-15 * max(1.0, abs(float(m)))


def test_keep_all_keep_none_and_counts():
    sc = gen_scores(9, 1, 256)[0]
    assert osel.select_topk(sc, osel.topk_count(1.0, 256))[1] == 256
    assert osel.select_topk(sc, osel.topk_count(0.0, 256))[1] == 0
    # per-layer keep fractions of the 32K four-layer workload
    assert [osel.topk_count(p, 256) for p in (0.8, 0.6, 0.5, 0.4)] == [205, 154, 128, 103]
    assert [osel.topk_count(p, 64) for p in (0.25, 0.5, 0.75)] == [16, 32, 48]
    assert osel.topk_count(0.3, 10) == 3
    idx, n, _ = osel.select_abs_ge(sc, np.inf)
    assert n == 0 and all(idx == -1)


def test_nan_scores_never_kept():
    sc = np.array([1.0, np.nan, 3.0, 2.0], np.float32)
    idx, n, _ = osel.select_abs_ge(sc, -1e30)
    assert list(idx[:n]) == [0, 2, 3]
    idx, n, _ = osel.select_topk(sc, 3)
    assert list(idx[:n]) == [0, 2, 3]


def test_batched_front_end():
    sc = gen_scores(12, 3, 40)
    idx, nk, mask = osel.select(sc, "topk_frac", 0.5)
    for b in range(3):
        i, n, m = osel.select_topk(sc[b], 20)
        assert nk[b] == n and (idx[b] == i).all() and (mask[b] == m).all()


def test_gather_scatter_identity():
    rng = np.random.default_rng(0)
    S, h, blk = 64, 12, 8
    x = rng.standard_normal((S, h)).astype(np.float32).astype(np.float64)
    idx = np.array([1, 4, 5, 7, -1, -1, -1, -1], np.int32)
    g = omv.gather(x, idx, 4, blk)
    assert g.shape == (32, h)
    z = omv.scatter_add(np.zeros_like(x), g, idx, 4, blk, 1.0, "f32")
    rows = omv.retained_rows(idx, 4, blk)
    np.testing.assert_array_equal(z[rows], x[rows])
    other = np.setdiff1d(np.arange(S), rows)
    assert (z[other] == 0).all()
    assert list(rows[:3]) == [8, 9, 10] and rows[-1] == 63


def test_score_fp32_scatter_is_three_x():
    c = gen_score_case(0)
    x = c.x.astype(np.float64)
    idx = np.array([0, 3, 9, -1], np.int32)
    y = omv.gather(x, idx, 3, c.blk)
    out = omv.scatter_add(x, y, idx, 3, c.blk, 2.0, "f32")
    rows = omv.retained_rows(idx, 3, c.blk)
    np.testing.assert_array_equal(out[rows], (3.0 * c.x[rows].astype(np.float32)).astype(np.float64))
    other = np.setdiff1d(np.arange(c.S), rows)
    np.testing.assert_array_equal(out[other], x[other])


def test_scatter_add_bf16_rounds_once():
    x = np.array([[1.0, 256.0]])
    y = np.array([[2.0 ** -8, 1.0]])          # 1 + 2^-8 is a tie -> even (1.0); 257 -> 256 (tie, even)
    out = omv.scatter_add(x, y, np.array([0], np.int32), 1, 1, 1.0, "bf16")
    assert out[0, 0] == 1.0 and out[0, 1] == 256.0
    y2 = np.array([[3 * 2.0 ** -8, 3.0]])     # 1 + 3*2^-8 -> 1 + 2^-6 ; 259 -> 260
    out2 = omv.scatter_add(x, y2, np.array([0], np.int32), 1, 1, 1.0, "bf16")
    assert out2[0, 0] == 1.0 + 2.0 ** -6 and out2[0, 1] == 260.0
    assert round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
