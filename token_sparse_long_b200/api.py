"""Python binding of the jenga C ABI: same names, torch tensors in, argument
marshalling only.  Every step of the path runs in libjenga.so kernels; PyTorch
supplies device memory (outputs, workspaces) and the current CUDA stream.
"""
import ctypes

import torch

from . import _lib
from ._lib import BF16, F32, LayerWeights, Lora, LoraGrads, check, load

SCORE_MODES = {"softmax_mass": _lib.SCORE_SOFTMAX_MASS, "paper_blockmax": _lib.SCORE_PAPER_BLOCKMAX}
SELECT_MODES = {"mean_ge": _lib.SELECT_MEAN_GE, "topk_frac": _lib.SELECT_TOPK_FRAC, "abs_ge": _lib.SELECT_ABS_GE,
                "topk": _lib.SELECT_TOPK}


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("jenga: tensors must be CUDA tensors (the library has no CPU path)")


# ------------------------------------------------------------------ status
def jenga_check_device_status(stream=None):
    lib = load()
    det = (ctypes.c_uint32 * 2)()
    st = lib.jenga_check_device_status(_stream(stream), det)
    if st != 0:
        raise _lib.JengaError(st, _lib.last_error())


def jenga_set_wait_budget_ns(ns):
    check(load().jenga_set_wait_budget_ns(int(ns)))


def jenga_version():
    return load().jenga_version().decode()


def jenga_profile_enable(on=True):
    check(load().jenga_profile_enable(1 if on else 0))


def jenga_profile_report():
    """Per-kernel launch counts and milliseconds recorded since jenga_profile_enable."""
    import json
    lib = load()
    buf = ctypes.create_string_buffer(1 << 16)
    lib.jenga_profile_report(buf, 1 << 16)
    return json.loads(buf.value.decode())


# ------------------------------------------------------------------ scoring / selection / movement
def jenga_score_blocks(q, k, heads, head_dim, blk, causal=True, mode="softmax_mass", out=None, ws=None,
                       stream=None):
    """q, k: [B, S, >= heads*head_dim] (or [S, ...]) fp32/bf16 CUDA tensors, last dim contiguous."""
    _need_cuda(q, k)
    q3 = q if q.dim() == 3 else q.unsqueeze(0)
    k3 = k if k.dim() == 3 else k.unsqueeze(0)
    B, S = q3.shape[0], q3.shape[1]
    assert q3.stride(-1) == 1 and k3.stride(-1) == 1 and q3.stride(0) == S * q3.stride(1)
    nb = S // blk
    lib = load()
    need = lib.jenga_score_workspace_bytes(B, S, heads, head_dim, blk)
    if ws is None:
        ws = _ws(need, q.device)
    if out is None:
        out = torch.empty(B, nb, dtype=torch.float32, device=q.device)
    check(lib.jenga_score_blocks(_p(q3), q3.stride(1), _p(k3), k3.stride(1), B, S, heads, head_dim, blk,
                                 1 if causal else 0, _dt(q3), SCORE_MODES[mode], _p(out), _p(ws), ws.numel(),
                                 _stream(stream)))
    return out if q.dim() == 3 else out[0]


def jenga_select(scores, mode, param=0.0, out=None, ws=None, stream=None):
    """scores [B, nb] fp32 -> (idx int32 [B, nb], n_kept int32 [B], mask uint8 [B, nb]).
    out: optional preallocated (idx, n_kept, mask)."""
    _need_cuda(scores)
    s2 = scores if scores.dim() == 2 else scores.unsqueeze(0)
    s2 = s2.contiguous()
    B, nb = s2.shape
    lib = load()
    if out is not None:
        idx, nk, mask = out
    else:
        idx = torch.empty(B, nb, dtype=torch.int32, device=scores.device)
        nk = torch.empty(B, dtype=torch.int32, device=scores.device)
        mask = torch.empty(B, nb, dtype=torch.uint8, device=scores.device)
    need = lib.jenga_select_workspace_bytes(B, nb)
    if ws is None or ws.numel() < need:
        ws = _ws(need, scores.device)
    check(lib.jenga_select(_p(s2), B, nb, SELECT_MODES[mode], float(param), _p(idx), _p(nk), _p(mask), _p(ws),
                           ws.numel(), _stream(stream)))
    if scores.dim() == 1:
        return idx[0], nk, mask[0]
    return idx, nk, mask


def jenga_gather(x, idx, n_kept, blk, n_cap, out=None, stream=None):
    """x [B, S, h] or [S, h]; returns out [B, n_cap, h] (rows past n_kept*blk untouched)."""
    _need_cuda(x, idx, n_kept)
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    B, S, h = x3.shape
    if out is None:
        out = torch.empty(B, n_cap, h, dtype=x.dtype, device=x.device)
    o3 = out if out.dim() == 3 else out.unsqueeze(0)
    check(load().jenga_gather(_p(x3), x3.stride(1), B, S, h, blk, _p(idx), _p(n_kept), _dt(x3), _p(o3), o3.stride(1),
                              n_cap, _stream(stream)))
    return out if x.dim() == 3 else o3[0]


def jenga_scatter_add(x, y, idx, n_kept, blk, alpha=1.0, stream=None):
    """In place: x[row(i)] = round(x + alpha * y[i]) on retained rows."""
    _need_cuda(x, y, idx, n_kept)
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    y3 = y if y.dim() == 3 else y.unsqueeze(0)
    B, S, h = x3.shape
    check(load().jenga_scatter_add(_p(x3), x3.stride(1), _p(y3), y3.stride(1), B, S, h, blk, _p(idx), _p(n_kept),
                                   float(alpha), _dt(x3), y3.shape[1], _stream(stream)))
    return x


def jenga_scale_rows(x, rows, factor, stream=None):
    _need_cuda(x, rows)
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    B, S, h = x3.shape
    r2 = rows if rows.dim() == 2 else rows.unsqueeze(0)
    check(load().jenga_scale_rows(_p(x3), x3.stride(1), B, S, h, _p(r2), r2.shape[1], float(factor), _dt(x3),
                                  _stream(stream)))
    return x


# ------------------------------------------------------------------ layer
class LayerHandle:
    """Device tensors of one layer (frozen bf16 weights, LoRA, packed re-layout) and the
    ctypes structs that point at them."""

    def __init__(self, wq, wk, wv, wo, wg, wu, wd, attn_norm, mlp_norm, aq, bq, av, bv, heads, head_dim,
                 rms_eps=1e-5, rope_theta=10000.0, lora_scale=1.0, stream=None):
        ts = dict(wq=wq, wk=wk, wv=wv, wo=wo, wg=wg, wu=wu, wd=wd, attn_norm=attn_norm, mlp_norm=mlp_norm,
                  aq=aq, bq=bq, av=av, bv=bv)
        for k, t in ts.items():
            if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
                raise ValueError(f"{k}: contiguous bf16 CUDA tensor required")
        self.t = ts
        self.hidden = wq.shape[1]
        self.heads, self.head_dim, self.ffn = heads, head_dim, wg.shape[0]
        self.w = LayerWeights(self.hidden, heads, head_dim, self.ffn, rms_eps, rope_theta,
                              _p(attn_norm), _p(mlp_norm), _p(wq), _p(wk), _p(wv), _p(wo), _p(wg), _p(wu), _p(wd))
        self.lora = Lora(aq.shape[0], lora_scale, _p(aq), _p(bq), _p(av), _p(bv))
        lib = load()
        n = lib.jenga_layer_pack_bytes(ctypes.byref(self.w), ctypes.byref(self.lora))
        if n == 0:
            raise ValueError("jenga_layer_pack_bytes rejected the layer shape: " + _lib.last_error())
        self.packed = _ws(n, wq.device)
        check(lib.jenga_layer_pack(ctypes.byref(self.w), ctypes.byref(self.lora), _p(self.packed),
                                   self.packed.numel(), _stream(stream)))

    def saved_bytes(self, blk, n_kept_max, B=1):
        return load().jenga_layer_saved_bytes(ctypes.byref(self.w), B, blk, n_kept_max)

    def fwd_ws_bytes(self, blk, n_kept_max, B=1):
        return load().jenga_layer_fwd_workspace_bytes(ctypes.byref(self.w), B, blk, n_kept_max)

    def bwd_ws_bytes(self, blk, n_kept_max, segment_tokens, B=1):
        return load().jenga_layer_bwd_workspace_bytes(ctypes.byref(self.w), B, blk, n_kept_max, segment_tokens)

    def qk_ws_bytes(self, S, B=1):
        return load().jenga_layer_score_qk_workspace_bytes(ctypes.byref(self.w), B, S)


def jenga_layer_score_qk(layer: LayerHandle, x, out=None, ws=None, stream=None):
    """q and k of all S tokens for scoring: x [S, h] bf16 -> [S, 2*H*D] bf16 (q | k)."""
    _need_cuda(x)
    S = x.shape[-2]
    HD = layer.heads * layer.head_dim
    if out is None:
        out = torch.empty(S, 2 * HD, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = _ws(layer.qk_ws_bytes(S), x.device)
    check(load().jenga_layer_score_qk(ctypes.byref(layer.w), ctypes.byref(layer.lora), _p(layer.packed), _p(x), 1, S,
                                      _p(out), _p(ws), ws.numel(), _stream(stream)))
    return out


def jenga_sparse_layer_fwd(layer: LayerHandle, x, idx, n_kept, blk, n_kept_max, saved=None, ws=None, stream=None,
                           qk=None):
    """In place on x [S, h] bf16.  Returns the saved-context buffer for the backward.

    qk: optional [S, 2 H D] bf16 q | k of all rows from jenga_layer_score_qk on the same x;
    the retained rows' q and k are then taken from it (bit-identical) instead of projected.
    qk must have been computed from this x, after any change to x (e.g. jenga_scale_rows),
    and with this layer's weights and LoRA: a stale qk silently gives wrong q and k."""
    _need_cuda(x, idx, n_kept)
    S = x.shape[-2]
    if saved is None:
        saved = _ws(layer.saved_bytes(blk, n_kept_max), x.device)
    if ws is None:
        ws = _ws(layer.fwd_ws_bytes(blk, n_kept_max), x.device)
    if qk is None:
        check(load().jenga_sparse_layer_fwd(ctypes.byref(layer.w), ctypes.byref(layer.lora), _p(layer.packed), _p(x), 1,
                                            S, blk, _p(idx), _p(n_kept), int(n_kept_max), _p(saved), saved.numel(),
                                            _p(ws), ws.numel(), _stream(stream)))
    else:
        _need_cuda(qk)
        HD = layer.heads * layer.head_dim
        if qk.dtype != torch.bfloat16 or qk.device != x.device:
            raise ValueError("qk must be a bf16 tensor on x's device")
        if qk.dim() != 2 or qk.shape[0] < S or qk.shape[1] < 2 * HD or qk.stride(1) != 1:
            raise ValueError(f"qk must be [>= {S}, >= {2 * HD}] with a contiguous last dimension, got "
                             f"{tuple(qk.shape)} strides {qk.stride()}")
        check(load().jenga_sparse_layer_fwd_qk(ctypes.byref(layer.w), ctypes.byref(layer.lora), _p(layer.packed), _p(x),
                                               1, S, blk, _p(idx), _p(n_kept), int(n_kept_max), _p(qk), qk.stride(0),
                                               _p(saved), saved.numel(), _p(ws), ws.numel(), _stream(stream)))
    return saved


def jenga_sparse_layer_fwd_mlp(layer: LayerHandle, x, idx, n_kept, blk, n_kept_max, mlp_mode, mlp_param, saved=None,
                               ws=None, stream=None, qk=None, mlp_pos=None, n_mlp=None, mlp_scores=None):
    """jenga_sparse_layer_fwd with MLP-block elimination: the MLP sub-block keeps the retained
    blocks that jenga_select(mlp_mode, mlp_param) picks on their SiLU(gate) * up mass.
    Returns (saved, mlp_scores fp32 [n_kept_max], mlp_pos int32 [n_kept_max], n_mlp int32 [1])."""
    _need_cuda(x, idx, n_kept)
    S = x.shape[-2]
    if saved is None:
        saved = _ws(layer.saved_bytes(blk, n_kept_max), x.device)
    if ws is None:
        ws = _ws(layer.fwd_ws_bytes(blk, n_kept_max), x.device)
    if mlp_pos is None:
        mlp_pos = torch.empty(max(int(n_kept_max), 1), dtype=torch.int32, device=x.device)
    if n_mlp is None:
        n_mlp = torch.empty(1, dtype=torch.int32, device=x.device)
    if mlp_scores is None:
        mlp_scores = torch.empty(max(int(n_kept_max), 1), dtype=torch.float32, device=x.device)
    ld_qk = 0
    if qk is not None:
        _need_cuda(qk)
        HD = layer.heads * layer.head_dim
        if qk.dtype != torch.bfloat16 or qk.device != x.device or qk.dim() != 2 or qk.shape[0] < S \
                or qk.shape[1] < 2 * HD or qk.stride(1) != 1:
            raise ValueError("qk must be a bf16 [>= S, >= 2 H D] tensor on x's device, last dimension contiguous")
        ld_qk = qk.stride(0)
    check(load().jenga_sparse_layer_fwd_mlp(ctypes.byref(layer.w), ctypes.byref(layer.lora), _p(layer.packed), _p(x), 1,
                                            S, blk, _p(idx), _p(n_kept), int(n_kept_max), _p(qk), ld_qk,
                                            SELECT_MODES[mlp_mode], float(mlp_param), _p(mlp_scores), _p(mlp_pos),
                                            _p(n_mlp), _p(saved), saved.numel(), _p(ws), ws.numel(), _stream(stream)))
    return saved, mlp_scores, mlp_pos, n_mlp


def new_lora_grads(layer: LayerHandle):
    dev = layer.t["aq"].device
    return {k: torch.zeros(layer.t[k[1:]].shape, dtype=torch.float32, device=dev) for k in ("daq", "dbq", "dav", "dbv")}


def jenga_sparse_layer_bwd(layer: LayerHandle, dx, idx, n_kept, blk, n_kept_max, saved, grads, segment_tokens=4096,
                           ws=None, stream=None):
    """dx [S, h] bf16 holds G on entry and dL/dx on return; grads (dict of fp32) accumulate."""
    _need_cuda(dx, idx, n_kept, saved)
    S = dx.shape[-2]
    if ws is None:
        ws = _ws(layer.bwd_ws_bytes(blk, n_kept_max, segment_tokens), dx.device)
    g = LoraGrads(_p(grads["daq"]), _p(grads["dbq"]), _p(grads["dav"]), _p(grads["dbv"]))
    check(load().jenga_sparse_layer_bwd(ctypes.byref(layer.w), ctypes.byref(layer.lora), _p(layer.packed), _p(dx), 1, S,
                                        blk, _p(idx), _p(n_kept), int(n_kept_max), _p(saved), saved.numel(),
                                        ctypes.byref(g), int(segment_tokens), _p(ws), ws.numel(), _stream(stream)))
    return dx


# ------------------------------------------------------------------ predictor
def jenga_predict_blocks(x, blk, w1, b1, w2, b2, out=None, ws=None, stream=None):
    """x [S, h] bf16; w1 [m, h] bf16, b1 [m] fp32, w2 [m] bf16, b2 [1] fp32 -> scores [nb] fp32."""
    _need_cuda(x, w1, b1, w2, b2)
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    B, S, h = x3.shape
    nb = S // blk
    lib = load()
    if ws is None:
        ws = _ws(lib.jenga_predict_workspace_bytes(B, S, h, blk), x.device)
    if out is None:
        out = torch.empty(B, nb, dtype=torch.float32, device=x.device)
    check(lib.jenga_predict_blocks(_p(x3), B, S, h, blk, _p(w1), _p(b1), _p(w2), _p(b2), w1.shape[0], _p(out), _p(ws),
                                   ws.numel(), _stream(stream)))
    return out if x.dim() == 3 else out[0]


def jenga_mlp_block_scores(a, blk, n_kept=None, out=None, stream=None):
    """a [n_cap * blk, F] bf16 (compact retained rows) -> scores [n_cap] fp32 (-inf past n_kept)."""
    _need_cuda(a)
    n_cap = a.shape[0] // blk
    if out is None:
        out = torch.empty(n_cap, dtype=torch.float32, device=a.device)
    check(load().jenga_mlp_block_scores(_p(a), a.stride(0), a.shape[1], blk, _p(n_kept) if n_kept is not None else None,
                                        n_cap, _p(out), _stream(stream)))
    return out


def jenga_compose_block_indices(outer, pos, n_pos, out=None, stream=None):
    """out[i] = outer[pos[i]] for i < n_pos, -1 after (int32 device tensors)."""
    _need_cuda(outer, pos, n_pos)
    if out is None:
        out = torch.empty(pos.numel(), dtype=torch.int32, device=pos.device)
    check(load().jenga_compose_block_indices(_p(outer), outer.numel(), _p(pos), _p(n_pos), pos.numel(), _p(out),
                                             _stream(stream)))
    return out


def jenga_predict_blocks_qk(x, blk, q_w, k_w, causal=True, out=None, ws=None, stream=None):
    """x [S, h] or [B, S, h] bf16; q_w, k_w: (W1 [r1, h], W2 [r2, r1], W3 [d, r2]) bf16 ->
    scores [nb] (or [B, nb]) fp32: column sums of the query-key score-block products."""
    _need_cuda(x, *q_w, *k_w)
    x3 = x if x.dim() == 3 else x.unsqueeze(0)
    B, S, h = x3.shape
    r1, r2, d = q_w[0].shape[0], q_w[1].shape[0], q_w[2].shape[0]
    lib = load()
    if ws is None:
        ws = _ws(lib.jenga_predict_qk_workspace_bytes(B, S, h, blk, d), x.device)
    if out is None:
        out = torch.empty(B, S // blk, dtype=torch.float32, device=x.device)
    check(lib.jenga_predict_blocks_qk(_p(x3), B, S, h, blk, *[_p(t) for t in q_w], *[_p(t) for t in k_w], r1, r2, d,
                                      1 if causal else 0, _p(out), _p(ws), ws.numel(), _stream(stream)))
    return out if x.dim() == 3 else out[0]


def jenga_lm_loss_segmented(hidden, w, labels, segment_tokens=4096, dhidden=None, loss=None, ws=None, stream=None):
    """hidden [S, h] bf16, w [V, h] bf16, labels [S] int32 -> (loss fp32 [1], dhidden [S, h] bf16).

    Mean causal-LM cross-entropy over the tokens whose label is in [0, V) and its gradient
    with respect to hidden, computed segment_tokens rows at a time."""
    _need_cuda(hidden, w, labels)
    S, h = hidden.shape
    V = w.shape[0]
    lib = load()
    if ws is None:
        ws = _ws(lib.jenga_lm_loss_workspace_bytes(S, h, V, segment_tokens), hidden.device)
    if dhidden is None:
        dhidden = torch.empty(S, h, dtype=torch.bfloat16, device=hidden.device)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float32, device=hidden.device)
    check(lib.jenga_lm_loss_segmented(_p(hidden), _p(w), _p(labels), S, h, V, segment_tokens, _p(loss), _p(dhidden),
                                      _p(ws), ws.numel(), _stream(stream)))
    return loss, dhidden


def jenga_test_gemm(a, b, out_f32=True, bn=256, stream=None):
    """C = A B^T through the tcgen05 GEMM (test hook)."""
    M, K = a.shape
    N = b.shape[0]
    c = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device=a.device)
    check(load().jenga_test_gemm(_p(a), a.stride(0), _p(b), b.stride(0), M, N, K, _p(c), c.stride(0),
                                 1 if out_f32 else 0, bn, _stream(stream)))
    return c


def jenga_test_wait_timeout(stream=None):
    """Launch the wait-bound test hook (see include/jenga.h); read the result with
    jenga_check_device_status."""
    check(load().jenga_test_wait_timeout(_stream(stream)))


def jenga_test_exp2(x, stream=None):
    """(2^x by the FMA-pipe exponential, 2^x by ex2.approx) for fp32 device x (test hook)."""
    x = x.contiguous()
    y_fma = torch.empty_like(x)
    y_mufu = torch.empty_like(x)
    check(load().jenga_test_exp2(_p(x), _p(y_fma), _p(y_mufu), x.numel(), _stream(stream)))
    return y_fma, y_mufu
