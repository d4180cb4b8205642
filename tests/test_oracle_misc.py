"""Pins for oracle.bf16, oracle.predictor and oracle.rank (no GPU)."""
import numpy as np
import pytest
import scipy.stats
import torch

from oracle import predictor as opr
from oracle import rank as ork
from oracle.bf16 import from_bits, round_bf16
from synth import bf16_bits_to_f32, f32_to_bf16_bits


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_bf16(x.astype(np.float64)), want)


def test_round_bf16_ties_to_even():
    assert round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert round_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -40)) == -(1.0 + 2.0 ** -7)
    assert round_bf16(0.0) == 0.0


def test_synth_bits_roundtrip_agrees():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(5000).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    np.testing.assert_array_equal(from_bits(bits), round_bf16(x.astype(np.float64)))
    np.testing.assert_array_equal(bf16_bits_to_f32(bits).astype(np.float64), from_bits(bits))


def test_predictor_matches_torch_modules():
    rng = np.random.default_rng(2)
    S, h, m, blk = 64, 24, 8, 8
    x = rng.standard_normal((S, h))
    w1, b1 = rng.standard_normal((m, h)) * 0.3, rng.standard_normal(m) * 0.1
    w2, b2 = rng.standard_normal((1, m)) * 0.3, rng.standard_normal(1) * 0.1
    l1 = torch.nn.Linear(h, m).double()
    l2 = torch.nn.Linear(m, 1).double()
    with torch.no_grad():
        l1.weight.copy_(torch.tensor(w1)); l1.bias.copy_(torch.tensor(b1))
        l2.weight.copy_(torch.tensor(w2)); l2.bias.copy_(torch.tensor(b2))
        pooled = torch.nn.functional.avg_pool1d(torch.tensor(x).T[None], blk, blk)[0].T
        want = l2(torch.nn.functional.gelu(l1(pooled), approximate="none"))[:, 0].numpy()
    np.testing.assert_allclose(opr.predict_blocks(x, blk, w1, b1, w2, b2), want, rtol=1e-12, atol=1e-14)


def test_predictor_constant_blocks_score_equal():
    rng = np.random.default_rng(3)
    row = rng.standard_normal(16)
    x = np.tile(row, (32, 1))
    w1 = rng.standard_normal((4, 16))
    s = opr.predict_blocks(x, 8, w1, np.zeros(4), rng.standard_normal((1, 4)), np.zeros(1))
    assert np.ptp(s) == 0.0


@pytest.mark.parametrize("ties", [False, True])
def test_rank_statistics_match_scipy(ties):
    rng = np.random.default_rng(4)
    a = rng.standard_normal(60)
    b = a + rng.standard_normal(60)
    if ties:
        a = np.round(a)
        b = np.round(b)
    assert abs(ork.spearman(a, b) - scipy.stats.spearmanr(a, b).statistic) < 1e-12
    assert abs(ork.kendall_tau_b(a, b) - scipy.stats.kendalltau(a, b).statistic) < 1e-12


def test_topk_recall():
    exact = np.arange(10.0)
    assert ork.topk_recall(exact, exact, 5) == 1.0
    assert ork.topk_recall(-exact, exact, 5) == 0.0
    assert ork.topk_recall(np.array([9, 8, 0, 0, 0, 0, 0, 0, 0, 7.0]), exact, 3) == pytest.approx(1 / 3)
