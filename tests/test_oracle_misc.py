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


# ------------------------------------------------------------------ Q/K predictor pair
def _pair_case(seed, S=64, h=24, blk=8, r1=10, r2=6, d=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, h))
    mk = lambda: (rng.standard_normal((r1, h)) * 0.3, rng.standard_normal((r2, r1)) * 0.3,
                  rng.standard_normal((d, r2)) * 0.3)
    return x, blk, mk(), mk()


def test_predictor_pair_brute_force_loops():
    x, blk, qw, kw = _pair_case(0)
    nb = x.shape[0] // blk
    want = np.zeros(nb)
    for n in range(nb):
        for m in range(n, nb):
            xm = x[m * blk:(m + 1) * blk].sum(axis=0) / blk
            xn = x[n * blk:(n + 1) * blk].sum(axis=0) / blk
            qv = np.zeros(qw[2].shape[0])
            kv = np.zeros(kw[2].shape[0])
            for side, xv, out in ((qw, xm, qv), (kw, xn, kv)):
                a1 = [max(0.0, sum(side[0][i, c] * xv[c] for c in range(xv.size))) for i in range(side[0].shape[0])]
                a2 = [max(0.0, sum(side[1][i, c] * a1[c] for c in range(len(a1)))) for i in range(side[1].shape[0])]
                for i in range(out.size):
                    out[i] = sum(side[2][i, c] * a2[c] for c in range(len(a2)))
            want[n] += sum(qv[i] * kv[i] for i in range(qv.size))
    np.testing.assert_allclose(opr.predict_blocks_qk(x, blk, qw, kw), want, rtol=1e-12, atol=1e-13)


def test_predictor_pair_matches_torch_modules():
    x, blk, qw, kw = _pair_case(1)
    xt = torch.tensor(x).reshape(-1, blk, x.shape[1]).mean(dim=1)

    def side(w):
        net = torch.nn.Sequential(torch.nn.Linear(w[0].shape[1], w[0].shape[0], bias=False), torch.nn.ReLU(),
                                  torch.nn.Linear(w[1].shape[1], w[1].shape[0], bias=False), torch.nn.ReLU(),
                                  torch.nn.Linear(w[2].shape[1], w[2].shape[0], bias=False)).double()
        for lin, wi in zip([net[0], net[2], net[4]], w):
            lin.weight.data = torch.tensor(wi)
        return net(xt)

    blocks = side(qw) @ side(kw).T
    want = torch.tril(blocks).sum(dim=0).detach().numpy()
    np.testing.assert_allclose(opr.predict_blocks_qk(x, blk, qw, kw), want, rtol=1e-12, atol=1e-13)
    full = blocks.sum(dim=0).detach().numpy()
    np.testing.assert_allclose(opr.predict_blocks_qk(x, blk, qw, kw, causal=False), full, rtol=1e-12, atol=1e-13)


def test_predictor_pair_rank_one_closed_form():
    # d = 1 and identical representative embeddings in every block: every query block has
    # the same scalar q and every key block the same k, so key block n scores q k (nb - n)
    rng = np.random.default_rng(2)
    blk, h, nb = 4, 12, 9
    row = rng.standard_normal(h)
    x = np.tile(row, (nb * blk, 1))
    qw = (np.abs(rng.standard_normal((5, h))), np.abs(rng.standard_normal((4, 5))), rng.standard_normal((1, 4)))
    kw = (np.abs(rng.standard_normal((5, h))), np.abs(rng.standard_normal((4, 5))), rng.standard_normal((1, 4)))
    q = opr.predictor_pair_side(row[None, :], *qw)[0, 0]
    k = opr.predictor_pair_side(row[None, :], *kw)[0, 0]
    np.testing.assert_allclose(opr.predict_blocks_qk(x, blk, qw, kw), q * k * (nb - np.arange(nb)), rtol=1e-12)
