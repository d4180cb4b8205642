"""Pins for oracle.scores (no GPU).

Each test ties the oracle to something other than itself: a closed form, an
invariant of the softmax, or a library softmax / pure-Python brute force on tiny
inputs.
"""
from fractions import Fraction
from itertools import permutations

import numpy as np
import pytest
import torch

from oracle import scores as osc
from synth import gen_score_case


def _rand_qk(seed, S, H, D, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((S, H, D)) * scale, rng.standard_normal((S, H, D)) * scale)


@pytest.mark.parametrize("S,H,D,blk", [(64, 3, 16, 8), (96, 2, 32, 32), (17 * 4, 1, 8, 4)])
def test_total_mass_equals_queries_times_heads(S, H, D, blk):
    q, k = _rand_qk(S + H, S, H, D, 2.0)
    sc = osc.block_scores_softmax_mass(q, k, blk)
    assert sc.shape == (S // blk,)
    assert abs(sc.sum() - H * S) < 1e-9 * H * S


def test_zero_queries_give_harmonic_closed_form():
    # Q = 0 -> every causal row is uniform over j <= i: P_ij = 1/(i+1); key j's mass is
    # sum_{i=j}^{S-1} 1/(i+1) = Harm(S) - Harm(j), per head.
    S, H, D, blk = 48, 3, 16, 6
    _, k = _rand_qk(1, S, H, D)
    q = np.zeros((S, H, D))
    harm = [Fraction(0)]
    for i in range(1, S + 1):
        harm.append(harm[-1] + Fraction(1, i))
    mass = [H * (harm[S] - harm[j]) for j in range(S)]
    want = [float(sum(mass[n * blk:(n + 1) * blk])) for n in range(S // blk)]
    got = osc.block_scores_softmax_mass(q, k, blk)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_first_key_block_receives_query_zero():
    # With S == blk there is one block and it receives every query's full row: H*S.
    q, k = _rand_qk(3, 8, 2, 4)
    assert abs(osc.block_scores_softmax_mass(q, k, 8)[0] - 16.0) < 1e-12


def test_brute_force_against_library_softmax():
    S, H, D, blk = 40, 3, 16, 5
    q, k = _rand_qk(7, S, H, D, 1.5)
    qt, kt = torch.tensor(q), torch.tensor(k)
    logits = torch.einsum("ihd,jhd->hij", qt, kt) / np.sqrt(D)
    mask = torch.ones(S, S, dtype=torch.bool).triu(1)
    p = torch.softmax(logits.masked_fill(mask, float("-inf")), dim=-1)
    want = p.sum(dim=(0, 1)).reshape(S // blk, blk).sum(-1).numpy()
    np.testing.assert_allclose(osc.block_scores_softmax_mass(q, k, blk), want, rtol=1e-12)
    # non-causal variant
    pn = torch.softmax(logits, dim=-1)
    want_nc = pn.sum(dim=(0, 1)).reshape(S // blk, blk).sum(-1).numpy()
    np.testing.assert_allclose(osc.block_scores_softmax_mass(q, k, blk, causal=False), want_nc, rtol=1e-12)


def test_head_permutation_invariance_and_batch():
    S, H, D, blk = 32, 4, 8, 8
    q, k = _rand_qk(11, S, H, D)
    base = osc.block_scores_softmax_mass(q, k, blk)
    for perm in list(permutations(range(H)))[:5]:
        np.testing.assert_allclose(osc.block_scores_softmax_mass(q[:, perm], k[:, perm], blk), base, rtol=1e-13)
    qb = np.stack([q, q[::-1].copy()])
    kb = np.stack([k, k[::-1].copy()])
    sb = osc.block_scores_softmax_mass(qb, kb, blk)
    np.testing.assert_allclose(sb[0], base, rtol=1e-13)


def test_salient_key_raises_its_block():
    # A key aligned with every query collects more mass than its neighbours.
    S, H, D, blk = 64, 1, 16, 8
    q, k = _rand_qk(5, S, H, D, 0.1)
    d = np.ones(D) / np.sqrt(D)
    q[:, 0, :] += 3 * d
    k[20, 0, :] = 10 * d
    sc = osc.block_scores_softmax_mass(q, k, blk)
    assert np.argmax(sc) == 20 // blk


def test_score_fp32_workload_mean_is_closed_form():
    c = gen_score_case(0)
    q = c.q.reshape(c.S, c.H, c.D)
    k = c.k.reshape(c.S, c.H, c.D)
    sc = osc.block_scores_softmax_mass(q, k, c.blk)
    # mean block score = H * S / nb = 4 * 512 / 16 = 128
    assert abs(sc.mean() - 128.0) < 1e-9


def _blockmax_loops(q, k, blk):
    # Pure-Python Eq. (2) on tiny inputs: per causal entry sum positive head scores / H,
    # max inside each (m, n) score block, sum over m.
    S, H, D = q.shape
    nb = S // blk
    out = [0.0] * nb
    for m in range(nb):
        for n in range(nb):
            best = None
            for i in range(m * blk, (m + 1) * blk):
                for j in range(n * blk, (n + 1) * blk):
                    if j > i:
                        continue
                    tot = 0.0
                    for h in range(H):
                        sij = sum(q[i, h, d] * k[j, h, d] for d in range(D)) / D ** 0.5
                        if sij > 0:
                            tot += sij
                    v = tot / H
                    best = v if best is None else max(best, v)
            if best is not None:
                out[n] += best
    return out


def test_paper_blockmax_brute_force():
    q, k = _rand_qk(21, 12, 2, 4)
    np.testing.assert_allclose(osc.block_scores_paper_blockmax(q, k, 3), _blockmax_loops(q, k, 3), rtol=1e-12)


def test_golden_score_fp32_regression():
    # tests/golden/score_fp32_oracle.json was written by tests/golden/make_golden.py
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "score_fp32_oracle.json")) as f:
        gold = json.load(f)
    c = gen_score_case(0)
    sc = osc.block_scores_softmax_mass(c.q.reshape(c.S, c.H, c.D), c.k.reshape(c.S, c.H, c.D), c.blk)
    np.testing.assert_allclose(sc, gold["scores"], rtol=1e-12)
    assert abs(sum(gold["scores"]) - 4 * 512) < 1e-9
    assert list(c.salient) == gold["salient_rows"]


def test_row_lse_against_library_logsumexp_and_softmax_normalisation():
    from scipy.special import logsumexp
    S, D = 50, 16
    q, k = _rand_qk(9, S, 1, D, 3.0)
    rows = [0, 1, 7, 49]
    got = osc.row_lse(q[:, 0], k[:, 0], rows)
    for n, i in enumerate(rows):
        s = (q[i, 0] @ k[: i + 1, 0].T) / np.sqrt(D)
        assert abs(got[n] - logsumexp(s)) < 1e-12
        assert abs(np.exp(s - got[n]).sum() - 1.0) < 1e-12
    assert abs(osc.row_lse(q[:, 0], k[:, 0], [0])[0] - (q[0, 0] @ k[0, 0]) / np.sqrt(D)) < 1e-12
    full = osc.row_lse(q[:, 0], k[:, 0], [3], causal=False)[0]
    assert abs(full - logsumexp((k[:, 0] @ q[3, 0]) / np.sqrt(D))) < 1e-12
