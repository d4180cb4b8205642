"""Pins for oracle.lm_loss (no GPU): closed forms, the textbook cross-entropy of a
library, finite differences, and the ignore rule."""
import numpy as np
import torch

from oracle import lm_loss as olm


def _case(seed, S=40, h=16, V=50, ignore=()):
    rng = np.random.default_rng(seed)
    hid = rng.standard_normal((S, h))
    w = rng.standard_normal((V, h)) * 0.3
    lab = rng.integers(0, V, S)
    for t in ignore:
        lab[t] = -100
    return hid, w, lab


def test_zero_embedding_gives_log_vocab_and_zero_gradient():
    # all logits 0: every token's loss is log V exactly and (softmax - onehot) . 0 = 0
    hid, w, lab = _case(0)
    loss, dh = olm.lm_loss(hid, np.zeros_like(w), lab)
    assert abs(loss - np.log(w.shape[0])) < 1e-14
    assert np.abs(dh).max() == 0


def test_matches_torch_cross_entropy_and_autograd():
    hid, w, lab = _case(1, ignore=(3, 17))
    ht = torch.tensor(hid, requires_grad=True)
    wt = torch.tensor(w)
    lt = torch.tensor(lab)
    ref = torch.nn.functional.cross_entropy(ht @ wt.T, lt, ignore_index=-100, reduction="mean")
    ref.backward()
    loss, dh = olm.lm_loss(hid, w, lab)
    assert abs(loss - ref.item()) < 1e-12
    np.testing.assert_allclose(dh, ht.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_finite_differences():
    hid, w, lab = _case(2, S=6, h=5, V=7, ignore=(1,))
    _, dh = olm.lm_loss(hid, w, lab)
    eps = 1e-6
    for t in range(hid.shape[0]):
        for c in range(hid.shape[1]):
            hp, hm = hid.copy(), hid.copy()
            hp[t, c] += eps
            hm[t, c] -= eps
            fd = (olm.lm_loss(hp, w, lab)[0] - olm.lm_loss(hm, w, lab)[0]) / (2 * eps)
            assert abs(fd - dh[t, c]) < 1e-7, (t, c, fd, dh[t, c])


def test_ignored_tokens_contribute_nothing():
    hid, w, lab = _case(3, ignore=(0, 5, 9))
    keep = lab >= 0
    loss_all, dh_all = olm.lm_loss(hid, w, lab)
    loss_sub, dh_sub = olm.lm_loss(hid[keep], w, lab[keep])
    assert abs(loss_all - loss_sub) < 1e-13
    np.testing.assert_allclose(dh_all[keep], dh_sub, rtol=1e-12, atol=1e-15)
    assert np.abs(dh_all[~keep]).max() == 0


def test_row_subset_equals_full():
    hid, w, lab = _case(4, ignore=(2,))
    _, dh = olm.lm_loss(hid, w, lab)
    rows = np.array([0, 2, 7, 39])
    _, dh_r = olm.lm_loss(hid, w, lab, rows=rows)
    np.testing.assert_array_equal(dh_r, dh[rows])


def test_gradient_rows_sum_rule():
    # (softmax - onehot) sums to 0 over the vocabulary, so with W's rows all equal to one
    # vector u every dhidden row is 0
    hid, w, lab = _case(5)
    u = np.random.default_rng(6).standard_normal(w.shape[1])
    _, dh = olm.lm_loss(hid, np.tile(u, (w.shape[0], 1)), lab)
    assert np.abs(dh).max() < 1e-15
