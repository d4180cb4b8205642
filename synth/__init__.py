"""Seeded synthetic inputs for the token-sparse layer path.

This module only draws random numbers and converts storage formats (fp32 <-> bf16
bit patterns).  It holds none of the method's arithmetic: no scoring, selection,
normalisation, projection or attention.  Both the CUDA path (through the tests and
``bench.py``) and the CPU oracle (through the tests) take their inputs from here,
so the two sides see bit-identical data.

Workloads (shapes of the Jenga paper's fine-tuning setups: Llama-2 7B / 13B layer
shapes, sequence lengths 4K-32K, token blocks of 64 or 128 tokens, mixed bf16/fp32):

* ``score_fp32``  - S=512, 4 heads x 64, hidden 256, block 32; Q, K, X ~ N(0,1) fp32,
  8 uniformly chosen key rows scaled x4 (salient tokens).
* ``llama7b_s4k`` - one Llama-2-7B-shaped layer, S=4096, block 64, 5% salient rows x3.
* ``llama7b_s16k`` - same layer at S=16384, 5% salient rows x3 in 8 contiguous spans.
* ``llama7b_x4_s32k`` - four stacked 7B-shaped layers, S=32768, block 128, 4% salient
  rows x3 redrawn per layer.
* ``llama13b_pred_s32k`` - one 13B-shaped layer, S=32768, block 128, block-score
  predictor MLP 5120->128->1.

Draw order (numpy ``Generator(PCG64(seed))``, fp32 normals): layer weights in the
order Wq, Wk, Wv, Wo, Wg, Wu, Wd (layer by layer), then X, then the salient
positions (layer by layer), then G, then LoRA A_q, A_v (then B_q, B_v when a
nonzero B std is asked for), then predictor weights.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------------------
# storage-format helpers (bit conversion only)
# --------------------------------------------------------------------------------------


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); return the uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u                      # finite values cannot overflow 32 bits here
    r >>= 16
    out = r.astype(np.uint16)
    nan = np.isnan(a)           # keep NaN a NaN
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Expand uint16 bf16 bit patterns to fp32 values (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


# --------------------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerShape:
    hidden: int
    heads: int
    head_dim: int
    ffn: int
    lora_rank: int = 16
    lora_alpha: float = 16.0
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0

    @property
    def lora_scale(self) -> float:
        return self.lora_alpha / self.lora_rank


LLAMA2_7B = LayerShape(hidden=4096, heads=32, head_dim=128, ffn=11008)
LLAMA2_13B = LayerShape(hidden=5120, heads=40, head_dim=128, ffn=13824)


@dataclass(frozen=True)
class Workload:
    name: str
    S: int
    blk: int
    shape: LayerShape | None = None
    n_layers: int = 1
    keep: tuple = (0.5,)           # per-layer keep fraction (top-k) ; None = mean threshold
    salient_frac: float = 0.05
    salient_scale: float = 3.0
    salient_spans: int = 0           # 0 = scattered rows
    segment_tokens: int = 4096
    predictor_hidden: int = 0        # >0: block-score predictor MLP width
    batch: int = 1


WORKLOADS = {
    "score_fp32": Workload(name="score_fp32", S=512, blk=32, shape=None, keep=(None,),
                           salient_frac=0.0, salient_scale=4.0),
    "llama7b_s4k": Workload(name="llama7b_s4k", S=4096, blk=64, shape=LLAMA2_7B, keep=(0.5,)),
    "llama7b_s16k": Workload(name="llama7b_s16k", S=16384, blk=64, shape=LLAMA2_7B,
                             keep=(0.25, 0.5, 0.75, 1.0), salient_spans=8),
    "llama7b_x4_s32k": Workload(name="llama7b_x4_s32k", S=32768, blk=128, shape=LLAMA2_7B,
                                n_layers=4, keep=(0.8, 0.6, 0.5, 0.4), salient_frac=0.04),
    "llama13b_pred_s32k": Workload(name="llama13b_pred_s32k", S=32768, blk=128, shape=LLAMA2_13B,
                                   keep=(0.5,), salient_frac=0.0, predictor_hidden=128),
}


# --------------------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------------------


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return f32_to_bf16_bits(a)


def salient_positions(rng: np.random.Generator, S: int, count: int, spans: int = 0) -> np.ndarray:
    """Sorted token positions of the salient tokens.

    ``spans == 0``: ``count`` distinct positions drawn uniformly.  ``spans > 0``: the
    count is split into ``spans`` contiguous runs of length floor/ceil(count/spans)
    at random non-overlapping offsets (sorted uniform gaps).
    """
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    if spans <= 0:
        return np.sort(rng.choice(S, size=count, replace=False)).astype(np.int64)
    base, extra = divmod(count, spans)
    lens = [base + (1 if i < extra else 0) for i in range(spans)]
    free = S - count
    gaps = np.sort(rng.integers(0, free + 1, size=spans))
    pos = []
    consumed = 0
    for i, L in enumerate(lens):
        start = int(gaps[i]) + consumed
        pos.extend(range(start, start + L))
        consumed += L
    return np.asarray(pos, dtype=np.int64)


@dataclass
class LayerParams:
    """bf16 bit patterns (uint16) of one layer's frozen weights ([out, in], PyTorch Linear)."""
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wo: np.ndarray
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray
    attn_norm: np.ndarray
    mlp_norm: np.ndarray
    aq: np.ndarray = None   # LoRA A [r, h]
    bq: np.ndarray = None   # LoRA B [h, r]
    av: np.ndarray = None
    bv: np.ndarray = None


def gen_layer_weights(rng, shape: LayerShape, std: float = 0.02) -> LayerParams:
    h, f = shape.hidden, shape.ffn
    hd = shape.heads * shape.head_dim
    one = f32_to_bf16_bits(np.ones(h, dtype=np.float32))
    return LayerParams(
        wq=_normal_bf16(rng, (hd, h), std), wk=_normal_bf16(rng, (hd, h), std),
        wv=_normal_bf16(rng, (hd, h), std), wo=_normal_bf16(rng, (h, hd), std),
        wg=_normal_bf16(rng, (f, h), std), wu=_normal_bf16(rng, (f, h), std),
        wd=_normal_bf16(rng, (h, f), std), attn_norm=one.copy(), mlp_norm=one.copy())


def gen_lora(rng, shape: LayerShape, p: LayerParams, a_std=0.02, b_std=0.0):
    r, h = shape.lora_rank, shape.hidden
    hd = shape.heads * shape.head_dim
    p.aq = _normal_bf16(rng, (r, h), a_std)
    p.av = _normal_bf16(rng, (r, h), a_std)
    if b_std > 0:
        p.bq = _normal_bf16(rng, (hd, r), b_std)
        p.bv = _normal_bf16(rng, (hd, r), b_std)
    else:
        p.bq = np.zeros((hd, r), dtype=np.uint16)
        p.bv = np.zeros((hd, r), dtype=np.uint16)


@dataclass
class LayerCase:
    shape: LayerShape
    S: int
    blk: int
    layers: list                  # list[LayerParams]
    x: np.ndarray                 # bf16 bits [S, h]
    g: np.ndarray                 # bf16 bits [S, h] (upstream gradient, loss = sum(out * G))
    salient: list = field(default_factory=list)   # per layer sorted positions
    salient_scale: float = 3.0
    keep: tuple = (0.5,)
    segment_tokens: int = 4096
    predictor: dict | None = None


def gen_layer_case(seed: int, S: int, blk: int, shape: LayerShape, n_layers: int = 1,
                   keep=(0.5,), salient_frac=0.05, salient_scale=3.0, salient_spans=0,
                   lora_b_std=0.0, predictor_hidden=0, segment_tokens=4096,
                   weight_std=0.02) -> LayerCase:
    """Draw one layer-stack workload in the fixed documented order.

    Salient rows of X are multiplied by ``salient_scale`` for the first layer; the
    positions for later layers are returned in ``salient`` (the scaling is applied to
    that layer's input by the caller).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    layers = [gen_layer_weights(rng, shape, weight_std) for _ in range(n_layers)]
    x32 = rng.standard_normal(size=(S, shape.hidden), dtype=np.float32)
    count = round_half_up(salient_frac * S)
    sal = [salient_positions(rng, S, count, salient_spans) for _ in range(n_layers)]
    if count:
        x32[sal[0]] *= np.float32(salient_scale)
    x = f32_to_bf16_bits(x32)
    del x32
    g = _normal_bf16(rng, (S, shape.hidden), 1.0)
    for p in layers:
        gen_lora(rng, shape, p, 0.02, lora_b_std)
    pred = None
    if predictor_hidden:
        pred = dict(w1=_normal_bf16(rng, (predictor_hidden, shape.hidden), weight_std),
                    b1=np.zeros(predictor_hidden, dtype=np.float32),
                    w2=_normal_bf16(rng, (1, predictor_hidden), weight_std),
                    b2=np.zeros(1, dtype=np.float32))
    return LayerCase(shape=shape, S=S, blk=blk, layers=layers, x=x, g=g, salient=sal,
                     salient_scale=salient_scale, keep=tuple(keep), segment_tokens=segment_tokens,
                     predictor=pred)


def gen_workload(name: str, seed: int = 0, **overrides) -> LayerCase:
    w = WORKLOADS[name]
    kw = dict(S=w.S, blk=w.blk, shape=w.shape, n_layers=w.n_layers, keep=w.keep,
              salient_frac=w.salient_frac, salient_scale=w.salient_scale,
              salient_spans=w.salient_spans, predictor_hidden=w.predictor_hidden,
              segment_tokens=w.segment_tokens)
    kw.update(overrides)
    return gen_layer_case(seed, **kw)


@dataclass
class ScoreCase:
    S: int
    H: int
    D: int
    hidden: int
    blk: int
    q: np.ndarray    # fp32 [S, H*D]
    k: np.ndarray    # fp32 [S, H*D]
    x: np.ndarray    # fp32 [S, hidden]
    salient: np.ndarray


def gen_score_case(seed: int = 0, S: int = 512, H: int = 4, D: int = 64, hidden: int = 256,
                   blk: int = 32, n_salient: int = 8, salient_scale: float = 4.0) -> ScoreCase:
    """fp32 scoring workload: Q, K, X ~ N(0,1) (drawn in that order), then ``n_salient``
    distinct key rows chosen uniformly and scaled by ``salient_scale``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal(size=(S, H * D), dtype=np.float32)
    k = rng.standard_normal(size=(S, H * D), dtype=np.float32)
    x = rng.standard_normal(size=(S, hidden), dtype=np.float32)
    sal = np.sort(rng.choice(S, size=n_salient, replace=False)) if n_salient else np.zeros(0, np.int64)
    k[sal] *= np.float32(salient_scale)
    return ScoreCase(S=S, H=H, D=D, hidden=hidden, blk=blk, q=q, k=k, x=x, salient=sal)


def gen_scores(seed: int, B: int, nb: int, dist: str = "normal") -> np.ndarray:
    """fp32 block-score vectors [B, nb] for selection tests (normal, or with ties)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if dist == "ties":
        return rng.integers(0, 5, size=(B, nb)).astype(np.float32)
    return rng.standard_normal(size=(B, nb), dtype=np.float32)
