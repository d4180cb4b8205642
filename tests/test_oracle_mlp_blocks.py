"""Pins for oracle.mlp_blocks (no GPU)."""
import numpy as np

from oracle import mlp_blocks as omb
from oracle import select as osel


def test_block_scores_brute_force_loops():
    rng = np.random.default_rng(0)
    a = rng.standard_normal((24, 7))
    want = [sum(abs(a[t, f]) for t in range(b * 4, b * 4 + 4) for f in range(7)) for b in range(6)]
    np.testing.assert_allclose(omb.mlp_block_scores(a, 4), want, rtol=1e-14)


def test_block_scores_closed_forms():
    # constant activation c: every block scores blk * F * |c|; the sign does not matter;
    # zero activation scores 0; blocks past n_kept are never selectable
    a = np.full((32, 5), -1.5)
    np.testing.assert_array_equal(omb.mlp_block_scores(a, 8), np.full(4, 8 * 5 * 1.5))
    np.testing.assert_array_equal(omb.mlp_block_scores(-a, 8), omb.mlp_block_scores(a, 8))
    assert np.all(omb.mlp_block_scores(np.zeros((16, 3)), 4) == 0)
    s = omb.mlp_block_scores(a, 8, n_kept=2)
    assert np.all(np.isneginf(s[2:])) and np.all(s[:2] == 60.0)


def test_compose_indices():
    outer = np.array([3, 5, 8, 13, 21, -1, -1])
    pos = np.array([0, 2, 4, -1, -1, -1, -1])
    np.testing.assert_array_equal(omb.compose_indices(outer, pos, 3), [3, 8, 21, -1, -1, -1, -1])


def test_second_list_is_subset_of_first():
    rng = np.random.default_rng(1)
    nb, blk, F = 32, 4, 6
    outer, n_out, _ = osel.select_topk(rng.standard_normal(nb), 20)
    a = rng.standard_normal((n_out * blk, F))
    s = omb.mlp_block_scores(a, blk)
    pos, n_pos, _ = osel.select_topk(s, 10)
    inner = omb.compose_indices(outer, pos, n_pos)
    assert set(inner[:n_pos].tolist()) <= set(outer[:n_out].tolist())
    assert np.all(np.diff(inner[:n_pos]) > 0)
