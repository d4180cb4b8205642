"""Retained-token Llama decoder layer, forward and backward (oracle).

What the pages fix:
* Jenga notes §4.1 / Jenga summary §4.1 (Fig. 5): per layer, the retained tokens
  run through the attention block and the MLP block; eliminated tokens skip both.
* §4.4 / §4.4.1 (Fig. 9): retained rows are read from the original input and the
  sub-block outputs are added in place into those rows (residual add); eliminated
  rows keep their input, so their gradient is the identity.
* §4.4.2 (Fig. 10): segment-based peak cutting -- the sequence is cut into
  segments, each segment's activations are rebuilt, its gradient computed and its
  activations dropped; gradients are aggregated across segments.
* Experimental setup: Llama-2 models (RMSNorm, rotary positions, SiLU-gated MLP),
  LoRA fine-tuning, mixed bf16/fp32.

Readings (the pages are silent on these):
* RoPE uses the tokens' ORIGINAL positions; attention is causal among retained
  tokens only (eliminated tokens are neither queries nor keys).  Because the kept
  block list ascends, causality in compact order equals causality in original order.
* RMSNorm eps 1e-5, learned gains applied after normalisation; RoPE theta 10000 with
  the rotate-half convention (pairs d and d + D/2); LoRA on q_proj and v_proj,
  delta W = scale * B @ A, no dropout, no biases.
* One index set per layer serves both sub-blocks, unless an MLP keep mask is given
  (Jenga summary §4.2.4, extend to the MLP block): then the MLP sub-block runs only on the
  retained rows whose mask entry is set, and on the others the layer output is h (the
  attention sub-block's output), so their MLP branch contributes nothing to the forward
  and its gradient is zero in the backward.  The mask is per retained row (per retained
  block in ``sparse_layer_fwd``); which blocks to keep is decided elsewhere (the GPU's
  criterion and selection are passed in, like the attention block list).
* bf16 storage rounding (``rnd=True``) at: xn (normed attention input), q and k after
  RoPE, v, the attention output o, h (after the attention residual add), hn (normed
  MLP input), a = SiLU(g) * u, the layer output, and the input gradient dX.  All other
  arithmetic is float64.  LoRA intermediates t = xn A^T and LoRA gradients stay
  unrounded.  ``rnd=False`` gives the exact float64 layer.
* Segmented backward: consecutive segments of ``segment_tokens`` retained rows (last
  one short), processed last segment first; key/value gradients accumulate across
  query segments, so a key segment is complete once every later query segment has
  been processed.  Equal to the unsegmented backward up to float64 summation order.

Shapes: x [n, h]; weights [out, in]; q, k, v, o [n, H, D]; LoRA A [r, h], B [H*D, r].
"""
from dataclasses import dataclass

import numpy as np

from .bf16 import from_bits, round_bf16
from .movement import retained_rows


@dataclass
class Weights:
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wo: np.ndarray
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray
    g1: np.ndarray
    g2: np.ndarray
    aq: np.ndarray
    bq: np.ndarray
    av: np.ndarray
    bv: np.ndarray
    heads: int
    head_dim: int
    eps: float = 1e-5
    theta: float = 10000.0
    lora_scale: float = 1.0

    @classmethod
    def from_bits(cls, p, shape):
        """Build float64 weights from bf16 bit patterns (``synth.LayerParams``)."""
        return cls(wq=from_bits(p.wq), wk=from_bits(p.wk), wv=from_bits(p.wv), wo=from_bits(p.wo),
                   wg=from_bits(p.wg), wu=from_bits(p.wu), wd=from_bits(p.wd),
                   g1=from_bits(p.attn_norm), g2=from_bits(p.mlp_norm),
                   aq=from_bits(p.aq), bq=from_bits(p.bq), av=from_bits(p.av), bv=from_bits(p.bv),
                   heads=shape.heads, head_dim=shape.head_dim, eps=shape.rms_eps,
                   theta=shape.rope_theta, lora_scale=shape.lora_scale)


def _r(x, rnd):
    return round_bf16(x) if rnd else x


# ------------------------------------------------------------------ building blocks


def rms_norm(x, g, eps):
    """y = x / sqrt(mean(x^2) + eps) * g (per row); returns y and the row factor."""
    rstd = 1.0 / np.sqrt((x * x).mean(axis=1) + eps)
    return x * rstd[:, None] * g[None, :], rstd


def rms_norm_bwd(dy, x, g, rstd):
    """Gradient of ``rms_norm`` w.r.t. x (derived by hand):
    dx_j = r g_j dy_j - x_j r^3 / N * sum_i dy_i g_i x_i."""
    N = x.shape[1]
    dyg = dy * g[None, :]
    dot = (dyg * x).sum(axis=1)
    return dyg * rstd[:, None] - x * (rstd ** 3 * dot / N)[:, None]


def rope_cos_sin(pos, D, theta):
    """cos/sin of angle pos * theta^(-2i/D), i = 0 .. D/2-1; shape [n, D/2]."""
    inv = theta ** (-np.arange(0, D, 2, dtype=np.float64) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate-half rotary embedding of x [n, H, D]."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy, cos, sin):
    """Transpose of ``rope`` (rotation by the negative angle)."""
    half = dy.shape[-1] // 2
    d1, d2 = dy[..., :half], dy[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def sigmoid(z):
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def silu(z):
    return z * sigmoid(z)


def silu_grad(z):
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def head_attention_fwd(args):
    """Causal softmax attention of ONE head: args = (qh, kh, vh [n, D], chunk).

    o_i = softmax_j(q_i . k_j / sqrt(D)) v over keys j <= i.  Returns o [n, D] and the
    row log-sum-exp [n] of the scaled logits; rows go in chunks only to bound memory."""
    qh, kh, vh, chunk = args
    n, D = qh.shape
    scale = 1.0 / np.sqrt(D)
    o = np.zeros_like(qh)
    lse = np.zeros(n)
    jj = np.arange(n)
    for i0 in range(0, n, chunk):
        i1 = min(n, i0 + chunk)
        s = (qh[i0:i1] @ kh[:i1].T) * scale
        # keys j < i0 are visible to every row of the chunk; only the diagonal block is masked
        s[:, i0:] = np.where(jj[None, i0:i1] <= np.arange(i0, i1)[:, None], s[:, i0:], -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[i0:i1] = (p / l) @ vh[:i1]
        lse[i0:i1] = (m + np.log(l))[:, 0]
    return o, lse


def _heads(t):
    return [np.ascontiguousarray(t[:, h]) for h in range(t.shape[1])]


def attention_fwd(q, k, v, chunk=1024, pmap=map):
    """Causal softmax attention per head (softmax(q k^T / sqrt(D)) v, keys j <= i).

    Returns o [n, H, D] and the row log-sum-exp [H, n] of the scaled logits.  ``pmap``
    maps ``head_attention_fwd`` over the heads (independent of one another)."""
    n, H, D = q.shape
    o = np.zeros_like(q)
    lse = np.zeros((H, n))
    tasks = [(qh, kh, vh, chunk) for qh, kh, vh in zip(_heads(q), _heads(k), _heads(v))]
    for h, (oh, lh) in enumerate(pmap(head_attention_fwd, tasks)):
        o[:, h] = oh
        lse[h] = lh
    return o, lse


def head_attention_bwd(args):
    """Backward of ``head_attention_fwd`` for ONE head: args = (qh, kh, vh, doh [n, D],
    segments, chunk).  The query rows go segment by segment in the order given (each
    segment (r0, r1) in row chunks); every segment's contribution is added to the key /
    value gradients of keys [0, r1).  Per chunk, the textbook softmax-attention backward:
    P = softmax(q k^T / sqrt(D)) (causal), dP = dO V^T, dS = P * (dP - rowsum(P * dP)),
    dQ = dS K / sqrt(D), dK += dS^T Q / sqrt(D), dV += P^T dO.  Returns dq, dk, dv [n, D]."""
    qh, kh, vh, doh, segments, chunk = args
    n, D = qh.shape
    scale = 1.0 / np.sqrt(D)
    dq = np.zeros((n, D))
    dk = np.zeros((n, D))
    dv = np.zeros((n, D))
    jj = np.arange(n)
    for (r0, r1) in segments:
        for i0 in range(r0, r1, chunk):
            i1 = min(r1, i0 + chunk)
            s = (qh[i0:i1] @ kh[:i1].T) * scale
            s[:, i0:] = np.where(jj[None, i0:i1] <= np.arange(i0, i1)[:, None], s[:, i0:], -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            p /= p.sum(axis=1, keepdims=True)
            dp = doh[i0:i1] @ vh[:i1].T
            delta = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - delta)
            dq[i0:i1] = (ds @ kh[:i1]) * scale
            dk[:i1] += (ds.T @ qh[i0:i1]) * scale
            dv[:i1] += p.T @ doh[i0:i1]
    return dq, dk, dv


def attention_bwd(q, k, v, do, segments, chunk=1024, pmap=map):
    """``head_attention_bwd`` for every head (mapped with ``pmap``): dq, dk, dv [n, H, D]."""
    dq = np.zeros_like(q)
    dk = np.zeros_like(q)
    dv = np.zeros_like(q)
    tasks = [(qh, kh, vh, dh, segments, chunk) for qh, kh, vh, dh in zip(_heads(q), _heads(k), _heads(v), _heads(do))]
    for h, (a, b, c) in enumerate(pmap(head_attention_bwd, tasks)):
        dq[:, h], dk[:, h], dv[:, h] = a, b, c
    return dq, dk, dv


# ------------------------------------------------------------------ layer


def project_qk(x, pos, W: Weights, rnd=True, with_v=False):
    """The attention input projections of rows x [n, h] at original positions ``pos``:
    xn = RMSNorm(x) (rounded), q = RoPE(xn Wq^T + s (xn Aq^T) Bq^T), k = RoPE(xn Wk^T)
    (rounded after RoPE), and with ``with_v`` also v = xn Wv^T + s (xn Av^T) Bv^T (rounded).
    Returns dict(xn, rstd1, tq, tv, q, k[, v], cos, sin); q, k, v are [n, H, D]."""
    x = np.asarray(x, np.float64)
    n, hdim = x.shape
    H, D, s = W.heads, W.head_dim, W.lora_scale
    xn, rstd1 = rms_norm(x, W.g1, W.eps)
    xn = _r(xn, rnd)
    tq = xn @ W.aq.T
    tv = xn @ W.av.T
    q_lin = (xn @ W.wq.T + s * (tq @ W.bq.T)).reshape(n, H, D)
    k_lin = (xn @ W.wk.T).reshape(n, H, D)
    cos, sin = rope_cos_sin(pos, D, W.theta)
    out = dict(xn=xn, rstd1=rstd1, tq=tq, tv=tv, q=_r(rope(q_lin, cos, sin), rnd), k=_r(rope(k_lin, cos, sin), rnd),
               cos=cos, sin=sin)
    if with_v:
        out["v"] = _r((xn @ W.wv.T + s * (tv @ W.bv.T)).reshape(n, H, D), rnd)
    return out


def layer_fwd(x, pos, W: Weights, rnd=True, pmap=map, mlp_keep=None):
    """Llama decoder layer on the retained rows x [n, h] at original positions ``pos``.

    Returns (out [n, h], ctx) where ctx holds what the backward needs.  ``pmap`` maps the
    per-head attention (see ``attention_fwd``).  ``mlp_keep`` (bool [n], optional): rows
    whose MLP sub-block runs; the others output h (module docstring)."""
    x = np.asarray(x, np.float64)
    n, hdim = x.shape
    H, D = W.heads, W.head_dim
    pr = project_qk(x, pos, W, rnd, with_v=True)
    xn, rstd1, tq, tv, q, k, v, cos, sin = (pr[key] for key in ("xn", "rstd1", "tq", "tv", "q", "k", "v", "cos",
                                                                 "sin"))
    o, lse = attention_fwd(q, k, v, pmap=pmap)
    o = _r(o, rnd)
    h = _r(x + o.reshape(n, H * D) @ W.wo.T, rnd)
    hn, rstd2 = rms_norm(h, W.g2, W.eps)
    hn = _r(hn, rnd)
    gt = hn @ W.wg.T
    ut = hn @ W.wu.T
    a = _r(silu(gt) * ut, rnd)
    out = _r(h + a @ W.wd.T, rnd)
    if mlp_keep is not None:
        mlp_keep = np.asarray(mlp_keep, bool)
        out = np.where(mlp_keep[:, None], out, h)
    ctx = dict(x=x, pos=np.asarray(pos), xn=xn, rstd1=rstd1, tq=tq, tv=tv, q=q, k=k, v=v, o=o,
               lse=lse, h=h, hn=hn, rstd2=rstd2, gt=gt, ut=ut, a=a, cos=cos, sin=sin, rnd=rnd, mlp_keep=mlp_keep)
    return out, ctx


def _segments(n, seg):
    if seg is None or seg <= 0 or seg >= n:
        return [(0, n)] if n else []
    return [(s0, min(n, s0 + seg)) for s0 in range(0, n, seg)]


def layer_bwd(ctx, G, W: Weights, segment_tokens=None, pmap=map):
    """Backward of ``layer_fwd`` for loss = sum(out * G) (so dOut = G).

    Frozen base weights get no gradient.  Returns (dx [n, h], grads) with grads the
    LoRA gradients daq [r, h], dbq [H*D, r], dav, dbv.  ``segment_tokens`` splits the
    retained rows into consecutive segments processed last-first (module docstring):
    the MLP block and the o projection are row-local, so every segment's attention-output
    gradient is formed first; the attention backward then runs per head over the query
    segments, last first, accumulating the key / value gradients; the projection backward
    (row-local once a segment's key / value gradients are complete) follows per segment,
    last first, adding each segment's LoRA gradient contribution in that order."""
    G = np.asarray(G, np.float64)
    x, xn, h, hn = ctx["x"], ctx["xn"], ctx["h"], ctx["hn"]
    q, k, v = ctx["q"], ctx["k"], ctx["v"]
    cos, sin = ctx["cos"], ctx["sin"]
    n, hdim = x.shape
    H, D, s = W.heads, W.head_dim, W.lora_scale
    dx = np.zeros((n, hdim))
    grads = dict(daq=np.zeros_like(W.aq), dbq=np.zeros_like(W.bq),
                 dav=np.zeros_like(W.av), dbv=np.zeros_like(W.bv))
    segs = list(reversed(_segments(n, segment_tokens)))
    dh_all = np.zeros((n, hdim))
    do_all = np.zeros((n, H, D))
    for (s0, s1) in segs:
        sl = slice(s0, s1)
        # --- MLP block: out = h + (silu(hn Wg^T) * (hn Wu^T)) Wd^T (rows the MLP keeps)
        Gs = G[sl]
        keep = ctx.get("mlp_keep")
        Gm = Gs if keep is None else Gs * keep[sl][:, None]
        da = Gm @ W.wd
        gt, ut = ctx["gt"][sl], ctx["ut"][sl]
        dut = da * silu(gt)
        dgt = da * ut * silu_grad(gt)
        dhn = dgt @ W.wg + dut @ W.wu
        dh_all[sl] = Gs + rms_norm_bwd(dhn, h[sl], W.g2, ctx["rstd2"][sl])
        # --- attention block: h = x + o Wo^T
        do_all[sl] = (dh_all[sl] @ W.wo).reshape(s1 - s0, H, D)
    dq, dk, dv_h = attention_bwd(q, k, v, do_all, segs, pmap=pmap)
    for (s0, s1) in segs:
        sl = slice(s0, s1)
        dq_lin = rope_bwd(dq[sl], cos[sl], sin[sl]).reshape(s1 - s0, H * D)
        dk_lin = rope_bwd(dk[sl], cos[sl], sin[sl]).reshape(s1 - s0, H * D)
        dv = dv_h[sl].reshape(s1 - s0, H * D)
        dtq = s * (dq_lin @ W.bq)                      # [ns, r]
        dtv = s * (dv @ W.bv)
        grads["dbq"] += s * (dq_lin.T @ ctx["tq"][sl])
        grads["dbv"] += s * (dv.T @ ctx["tv"][sl])
        grads["daq"] += dtq.T @ xn[sl]
        grads["dav"] += dtv.T @ xn[sl]
        dxn = dq_lin @ W.wq + dk_lin @ W.wk + dv @ W.wv + dtq @ W.aq + dtv @ W.av
        dx[sl] = dh_all[sl] + rms_norm_bwd(dxn, x[sl], W.g1, ctx["rstd1"][sl])
    return _r(dx, ctx["rnd"]), grads


# ------------------------------------------------------------------ whole sequence


def sparse_layer_fwd(X, idx, n_kept, blk, W: Weights, rnd=True, pmap=map, mlp_keep_blocks=None):
    """Layer on the kept blocks of X [S, h]; eliminated rows pass through unchanged.
    ``mlp_keep_blocks`` (bool per retained block, in kept-list order, optional): the blocks
    whose MLP sub-block runs (``layer_fwd``'s mlp_keep, expanded to rows)."""
    X = np.asarray(X, np.float64)
    rows = retained_rows(idx, n_kept, blk)
    Xo = X.copy()
    if rows.size == 0:
        return Xo, None
    keep = None
    if mlp_keep_blocks is not None:
        keep = np.repeat(np.asarray(mlp_keep_blocks, bool)[: int(n_kept)], blk)
    out, ctx = layer_fwd(X[rows], rows, W, rnd, pmap=pmap, mlp_keep=keep)
    Xo[rows] = out
    ctx["rows"] = rows
    return Xo, ctx


def sparse_layer_bwd(ctx, G, W: Weights, segment_tokens=None, pmap=map):
    """dX = G on eliminated rows; the layer backward on retained rows."""
    G = np.asarray(G, np.float64)
    dX = G.copy()
    if ctx is None:
        z = dict(daq=np.zeros_like(W.aq), dbq=np.zeros_like(W.bq),
                 dav=np.zeros_like(W.av), dbv=np.zeros_like(W.bv))
        return dX, z
    rows = ctx["rows"]
    dx, grads = layer_bwd(ctx, G[rows], W, segment_tokens, pmap=pmap)
    dX[rows] = dx
    return dX, grads
