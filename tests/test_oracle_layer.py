"""Pins for oracle.layer (no GPU).

* keep-all / sparse forward and all gradients against HuggingFace's
  ``LlamaDecoderLayer`` in float64 with torch autograd (a textbook Llama layer that
  shares nothing with the oracle), LoRA attached as W x + s B (A x);
* finite differences of the oracle's own forward against its hand-derived backward;
* keep-none identity, B = 0 => dA = 0, segmented == unsegmented;
* the rotary angle convention against HF's rotary embedding.
"""
import numpy as np
import pytest
import torch

from oracle import layer as oly
from oracle.movement import retained_rows



@pytest.fixture(autouse=True)
def _float64_default():
    old = torch.get_default_dtype()
    torch.set_default_dtype(torch.float64)
    yield
    torch.set_default_dtype(old)


def _weights(seed, h=32, H=2, D=16, F=48, r=4, b_std=0.1, gain_noise=True, scale=2.0, eps=1e-5):
    rng = np.random.default_rng(seed)
    n = lambda *s, std=0.2: rng.standard_normal(s) * std  # noqa: E731
    g1 = 1 + (n(h, std=0.1) if gain_noise else 0)
    g2 = 1 + (n(h, std=0.1) if gain_noise else 0)
    return oly.Weights(wq=n(H * D, h), wk=n(H * D, h), wv=n(H * D, h), wo=n(h, H * D),
                       wg=n(F, h), wu=n(F, h), wd=n(h, F), g1=np.asarray(g1), g2=np.asarray(g2),
                       aq=n(r, h), bq=n(H * D, r, std=b_std), av=n(r, h), bv=n(H * D, r, std=b_std),
                       heads=H, head_dim=D, eps=eps, theta=10000.0, lora_scale=scale)


class _LoRALinear(torch.nn.Module):
    def __init__(self, w, a, b, s):
        super().__init__()
        self.w = torch.tensor(w)
        self.a = torch.nn.Parameter(torch.tensor(a))
        self.b = torch.nn.Parameter(torch.tensor(b))
        self.s = s

    def forward(self, x):
        return torch.nn.functional.linear(x, self.w) + self.s * torch.nn.functional.linear(
            torch.nn.functional.linear(x, self.a), self.b)


def _hf_layer(W: oly.Weights):
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaDecoderLayer
    h = W.wq.shape[1]
    cfg = LlamaConfig(hidden_size=h, num_attention_heads=W.heads, num_key_value_heads=W.heads,
                      head_dim=W.head_dim, intermediate_size=W.wg.shape[0], rms_norm_eps=W.eps,
                      rope_theta=W.theta, attention_bias=False, mlp_bias=False, attention_dropout=0.0)
    cfg._attn_implementation = "eager"
    layer = LlamaDecoderLayer(cfg, 0).double().eval()
    with torch.no_grad():
        layer.self_attn.k_proj.weight.copy_(torch.tensor(W.wk))
        layer.self_attn.o_proj.weight.copy_(torch.tensor(W.wo))
        layer.mlp.gate_proj.weight.copy_(torch.tensor(W.wg))
        layer.mlp.up_proj.weight.copy_(torch.tensor(W.wu))
        layer.mlp.down_proj.weight.copy_(torch.tensor(W.wd))
        layer.input_layernorm.weight.copy_(torch.tensor(W.g1))
        layer.post_attention_layernorm.weight.copy_(torch.tensor(W.g2))
    layer.self_attn.q_proj = _LoRALinear(W.wq, W.aq, W.bq, W.lora_scale)
    layer.self_attn.v_proj = _LoRALinear(W.wv, W.av, W.bv, W.lora_scale)
    for p in layer.parameters():
        if p is not layer.self_attn.q_proj.a and p is not layer.self_attn.q_proj.b \
                and p is not layer.self_attn.v_proj.a and p is not layer.self_attn.v_proj.b:
            p.requires_grad_(False)
    return layer, cfg


def _hf_run(W, x_r, pos, G_r):
    """HF layer on the retained rows at their original positions; returns out, dx, LoRA grads."""
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    layer, cfg = _hf_layer(W)
    n = x_r.shape[0]
    x = torch.tensor(x_r)[None].requires_grad_(True)
    pid = torch.tensor(pos)[None]
    # float64 rotary tables for the given positions (HF applies them with rotate-half)
    D = W.head_dim
    inv = 1.0 / (W.theta ** (torch.arange(0, D, 2, dtype=torch.float64) / D))
    ang = pid[0].double()[:, None] * inv[None, :]
    emb = torch.cat([ang, ang], dim=-1)
    cos, sin = emb.cos()[None], emb.sin()[None]
    # HF's own rotary module, for the convention check (fp32 angles inside HF)
    rot = LlamaRotaryEmbedding(cfg)
    hc, hs = rot(x, pid)
    assert torch.allclose(hc.double(), cos, atol=5e-6) and torch.allclose(hs.double(), sin, atol=5e-6)
    mask = torch.full((n, n), float("-inf")).triu(1)[None, None]
    out = layer(x, attention_mask=mask, position_ids=pid, position_embeddings=(cos, sin))
    out = out[0] if isinstance(out, tuple) else out
    (out[0] * torch.tensor(G_r)).sum().backward()
    qa = layer.self_attn.q_proj
    va = layer.self_attn.v_proj
    return (out[0].detach().numpy(), x.grad[0].numpy(),
            dict(daq=qa.a.grad.numpy(), dbq=qa.b.grad.numpy(), dav=va.a.grad.numpy(), dbv=va.b.grad.numpy()))


def _case(seed, S=24, h=32):
    rng = np.random.default_rng(100 + seed)
    return rng.standard_normal((S, h)), rng.standard_normal((S, h))


# HF's Llama layer computes the RMSNorm variance and the attention softmax in fp32
# even for float64 inputs, so the comparison tolerance is at the fp32 level; a large
# eps case makes the eps placement visible at that tolerance.
RT, AT = 2e-5, 2e-6


@pytest.mark.parametrize("seed,eps", [(0, 1e-5), (1, 0.25)])
def test_keep_all_matches_hf_llama_layer(seed, eps):
    W = _weights(seed, eps=eps)
    X, G = _case(seed)
    S, blk = X.shape[0], 4
    idx = np.arange(S // blk, dtype=np.int32)
    Xo, ctx = oly.sparse_layer_fwd(X, idx, S // blk, blk, W, rnd=False)
    dX, grads = oly.sparse_layer_bwd(ctx, G, W)
    out_hf, dx_hf, g_hf = _hf_run(W, X, np.arange(S), G)
    np.testing.assert_allclose(Xo, out_hf, rtol=RT, atol=AT)
    np.testing.assert_allclose(dX, dx_hf, rtol=RT, atol=AT)
    for key in g_hf:
        np.testing.assert_allclose(grads[key], g_hf[key], rtol=RT, atol=AT * 10)


def test_sparse_rows_match_hf_on_retained_subsequence():
    W = _weights(3)
    X, G = _case(3, S=32)
    blk = 4
    idx = np.array([0, 2, 3, 6, -1, -1, -1, -1], np.int32)
    Xo, ctx = oly.sparse_layer_fwd(X, idx, 4, blk, W, rnd=False)
    dX, grads = oly.sparse_layer_bwd(ctx, G, W)
    rows = retained_rows(idx, 4, blk)
    out_hf, dx_hf, g_hf = _hf_run(W, X[rows], rows, G[rows])
    np.testing.assert_allclose(Xo[rows], out_hf, rtol=RT, atol=AT)
    np.testing.assert_allclose(dX[rows], dx_hf, rtol=RT, atol=AT)
    other = np.setdiff1d(np.arange(32), rows)
    np.testing.assert_array_equal(Xo[other], X[other])
    np.testing.assert_array_equal(dX[other], G[other])
    for key in g_hf:
        np.testing.assert_allclose(grads[key], g_hf[key], rtol=RT, atol=AT * 10)


def test_keep_none_is_identity():
    W = _weights(4)
    X, G = _case(4)
    idx = np.full(6, -1, np.int32)
    Xo, ctx = oly.sparse_layer_fwd(X, idx, 0, 4, W)
    dX, grads = oly.sparse_layer_bwd(ctx, G, W)
    np.testing.assert_array_equal(Xo, X)
    np.testing.assert_array_equal(dX, G)
    assert all((v == 0).all() for v in grads.values())


def test_finite_differences():
    W = _weights(5, h=16, H=2, D=8, F=24, r=3)
    X, G = _case(5, S=16, h=16)
    pos = np.arange(3, 19)            # non-zero positions exercise the rotary angles
    out, ctx = oly.layer_fwd(X, pos, W, rnd=False)
    dx, grads = oly.layer_bwd(ctx, G, W)
    rng = np.random.default_rng(55)

    def loss(Xv, Wv):
        return float((oly.layer_fwd(Xv, pos, Wv, rnd=False)[0] * G).sum())

    eps = 1e-6
    dirx = rng.standard_normal(X.shape)
    num = (loss(X + eps * dirx, W) - loss(X - eps * dirx, W)) / (2 * eps)
    assert abs(num - (dx * dirx).sum()) < 1e-6 * max(1.0, abs(num))
    for key, attr in (("daq", "aq"), ("dbq", "bq"), ("dav", "av"), ("dbv", "bv")):
        d = rng.standard_normal(getattr(W, attr).shape)
        Wp = oly.Weights(**{**W.__dict__, attr: getattr(W, attr) + eps * d})
        Wm = oly.Weights(**{**W.__dict__, attr: getattr(W, attr) - eps * d})
        num = (loss(X, Wp) - loss(X, Wm)) / (2 * eps)
        assert abs(num - (grads[key] * d).sum()) < 1e-6 * max(1.0, abs(num)), key


def test_lora_b_zero_gives_zero_a_gradient():
    W = _weights(6, b_std=0.0)
    X, G = _case(6)
    out, ctx = oly.layer_fwd(X, np.arange(X.shape[0]), W, rnd=True)
    _, grads = oly.layer_bwd(ctx, G, W)
    assert (grads["daq"] == 0).all() and (grads["dav"] == 0).all()
    assert np.abs(grads["dbq"]).max() > 0 and np.abs(grads["dbv"]).max() > 0


@pytest.mark.parametrize("seg", [5, 8, 23])
def test_segmented_equals_unsegmented(seg):
    W = _weights(7)
    X, G = _case(7, S=24)
    out, ctx = oly.layer_fwd(X, np.arange(24), W, rnd=False)
    dx0, g0 = oly.layer_bwd(ctx, G, W, None)
    dx1, g1 = oly.layer_bwd(ctx, G, W, seg)
    np.testing.assert_allclose(dx1, dx0, rtol=1e-11, atol=1e-12)
    for key in g0:
        np.testing.assert_allclose(g1[key], g0[key], rtol=1e-11, atol=1e-12)


def test_rounded_mode_stays_close_to_exact():
    # bf16 storage rounding perturbs the layer at the bf16 epsilon level only.
    W = _weights(8)
    X, G = _case(8)
    pos = np.arange(X.shape[0])
    o0, c0 = oly.layer_fwd(X, pos, W, rnd=False)
    o1, c1 = oly.layer_fwd(X, pos, W, rnd=True)
    rel = np.abs(o1 - o0).max() / np.sqrt((o0 ** 2).mean())
    assert 0 < rel < 3e-2
    d0, _ = oly.layer_bwd(c0, G, W)
    d1, _ = oly.layer_bwd(c1, G, W)
    assert np.abs(d1 - d0).max() / np.sqrt((d0 ** 2).mean()) < 3e-2


# ------------------------------------------------------------------ MLP-block keep mask
def test_mlp_mask_all_kept_is_bit_identical_to_no_mask():
    W = _weights(9)
    X, G = _case(9, S=32)
    idx = np.array([0, 2, 3, 5, 7, -1, -1, -1], np.int32)
    Xa, ca = oly.sparse_layer_fwd(X, idx, 5, 4, W, rnd=True)
    dXa, ga = oly.sparse_layer_bwd(ca, G, W, 8)
    Xb, cb = oly.sparse_layer_fwd(X, idx, 5, 4, W, rnd=True, mlp_keep_blocks=np.ones(5, bool))
    dXb, gb = oly.sparse_layer_bwd(cb, G, W, 8)
    assert np.array_equal(Xa, Xb) and np.array_equal(dXa, dXb)
    assert all(np.array_equal(ga[k], gb[k]) for k in ga)


def _hf_run_mlp_mask(W, x_r, pos, G_r, keep_rows):
    """HF layer whose MLP output is multiplied by the 0/1 row mask: out = h + m * MLP(norm(h))."""
    from transformers.models.llama import modeling_llama as ml
    orig = ml.LlamaMLP.forward
    mask = torch.tensor(keep_rows.astype(np.float64))[None, :, None]
    ml.LlamaMLP.forward = lambda self, x: orig(self, x) * mask
    try:
        return _hf_run(W, x_r, pos, G_r)
    finally:
        ml.LlamaMLP.forward = orig


def test_mlp_mask_matches_hf_layer_with_masked_mlp_branch():
    W = _weights(10)
    X, G = _case(10, S=32)
    idx = np.array([1, 2, 4, 6, 7, -1, -1, -1], np.int32)
    keep_blocks = np.array([True, False, True, False, False])
    Xo, ctx = oly.sparse_layer_fwd(X, idx, 5, 4, W, rnd=False, mlp_keep_blocks=keep_blocks)
    dX, grads = oly.sparse_layer_bwd(ctx, G, W)
    rows = retained_rows(idx, 5, 4)
    out_hf, dx_hf, g_hf = _hf_run_mlp_mask(W, X[rows], rows, G[rows], np.repeat(keep_blocks, 4))
    np.testing.assert_allclose(Xo[rows], out_hf, rtol=RT, atol=AT)
    np.testing.assert_allclose(dX[rows], dx_hf, rtol=RT, atol=AT)
    for key in g_hf:
        np.testing.assert_allclose(grads[key], g_hf[key], rtol=RT, atol=AT * 10)
    # MLP-eliminated rows output exactly h = x + attention output
    h = ctx["h"]
    dropped = ~np.repeat(keep_blocks, 4)
    np.testing.assert_array_equal(Xo[rows][dropped], h[dropped])


def test_mlp_mask_finite_differences():
    W = _weights(11, h=16, H=2, D=8, F=24, r=3)
    X, G = _case(11, S=16, h=16)
    pos = np.arange(2, 18)
    keep = np.arange(16) % 3 != 0
    out, ctx = oly.layer_fwd(X, pos, W, rnd=False, mlp_keep=keep)
    dx, grads = oly.layer_bwd(ctx, G, W, 5)
    rng = np.random.default_rng(66)
    loss = lambda Xv: float((oly.layer_fwd(Xv, pos, W, rnd=False, mlp_keep=keep)[0] * G).sum())  # noqa: E731
    eps = 1e-6
    d = rng.standard_normal(X.shape)
    num = (loss(X + eps * d) - loss(X - eps * d)) / (2 * eps)
    assert abs(num - (dx * d).sum()) < 1e-6 * max(1.0, abs(num))
    # and the mask matters: all kept gives a different gradient
    _, c2 = oly.layer_fwd(X, pos, W, rnd=False)
    dx2, _ = oly.layer_bwd(c2, G, W, 5)
    assert np.abs(dx2 - dx).max() > 1e-3
