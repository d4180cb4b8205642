#!/usr/bin/env python3
"""Token-sparse layer benchmark: fwd+bwd tokens/s at S=32K.

Workload (default ``llama7b_x4_s32k``): four stacked Llama-2-7B-shaped layers (hidden
4096, 32 heads x 128, SwiGLU FFN 11008), bf16 storage / fp32 accumulation, S=32768,
batch 1, token blocks of 128, per-layer top-k keep fractions 80/60/50/40 %, 4% salient
rows x3 redrawn per layer, LoRA rank 16 on q/v, segment-wise backward over 4096
retained tokens.  One step = for each layer: q/k projection of all S tokens, single-pass
block scoring, top-k selection, retained-token forward (in place); then the backward
of the four layers in reverse (upstream gradient G, loss = sum(out * G)).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead on a
bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "token-sparse layer fwd+bwd tokens/s at S=32K; score/select/gather % roofline"
REF_TOKENS = 512         # oracle sample per reference-arm step (tokens through the whole stack)
BASELINE_TOKENS = 1024   # oracle sample of the cpu_baseline leg


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="jenga", choices=["jenga", "reference"])
    ap.add_argument("--workload", default="llama7b_x4_s32k")
    ap.add_argument("--no-dense", action="store_true", help="skip the keep-all comparison")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-movement", action="store_true", help="skip the standalone gather/scatter/select timing")
    ap.add_argument("--no-lm-loss", action="store_true", help="skip the segmented LM-head loss timing")
    ap.add_argument("--cpu-baseline-one-thread", action="store_true",
                    help="the cpu_baseline leg on one host thread: the CPU oracle over the two small workloads, "
                         "in full, then exit")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------- work model
def causal_pairs(n):
    return n * (n + 1) / 2.0


def work_model(case, ks, seg, scoring="exact"):
    """Algorithmic work per step for each kernel name: (kind, amount) with kind
    'flop' or 'byte'.  GEMM: 2 M N K.  Attention fwd: 2 matmuls per causal pair
    (4 D H pairs); backward: 5 matmul-equivalents per pair (10 D H pairs), shared
    3 : 4 between the dQ and dK/dV kernels in proportion to the matmuls each runs.
    Scoring ('exact'): q, k of all rows, then one QK^T product per causal pair (2 D H pairs,
    single pass); the forward then takes the retained rows' q, k from the scoring and
    projects only v.  Scoring 'predictor': one read of X for the block means (the MLP is
    negligible), and the forward projects q, k and v."""
    sh = case.shape
    S, h, H, D, F = case.S, sh.hidden, sh.heads, sh.head_dim, sh.ffn
    HD = H * D
    w = {}

    def add(name, kind, v):
        k0, v0 = w.get(name, (kind, 0.0))
        w[name] = (kind, v0 + v)

    for k in ks:
        n = k * case.blk
        if scoring == "exact":
            add("gemm_lora_t_all", "flop", 2.0 * S * 32 * h)
            add("gemm_qk_rope_all", "flop", 2.0 * S * 2 * HD * h)
            add("score_fused_tc", "flop", 2.0 * D * H * causal_pairs(S))
            add("gemm_v", "flop", 2.0 * n * HD * h)
            add("gather_qk_rows", "byte", 2.0 * n * 2 * HD * 2)
        else:
            add("pred_block_mean", "byte", 2.0 * S * h)
            add("gemm_qkv_rope", "flop", 2.0 * n * 3 * HD * h)
        add("gemm_lora_t", "flop", 2.0 * n * 32 * h)
        add("attn_fwd_tc", "flop", 4.0 * D * H * causal_pairs(n))
        add("gemm_o_scatter", "flop", 2.0 * n * h * HD)
        add("gemm_gateup_swiglu", "flop", 2.0 * n * 2 * F * h)
        add("gemm_down_scatter", "flop", 2.0 * n * h * F)
        add("gemm_da_swiglu_bwd", "flop", 2.0 * n * F * h)
        add("gemm_dhn", "flop", 2.0 * n * h * 2 * F)
        add("gemm_do", "flop", 2.0 * n * HD * h)
        add("attn_bwd_dq_tc", "flop", 10.0 * D * H * causal_pairs(n) * 3 / 7)
        add("attn_bwd_dkdv_tc", "flop", 10.0 * D * H * causal_pairs(n) * 4 / 7)
        add("gemm_dt", "flop", 2.0 * n * 32 * 3 * HD)
        add("gemm_dxn", "flop", 2.0 * n * h * 3 * HD)
        add("rmsnorm_rows", "byte", 2.0 * (S * h * 2) + 3.0 * n * h * 2 * 2)
        add("select_small", "byte", 9.0 * (S // case.blk))
    return w


# DRAM bytes per unit of work of a kernel, from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum; the capture and its command are in profiles/).  attn_bwd_dkdv_tc:
# its traffic is dominated by the fp32 dK / dV accumulators (read and written back by the
# L2's reduce-adds) and the K / V reads, both proportional to the keys [0, segment end) a
# launch covers, so the unit is a key row; captured on one 7B-shaped layer at S = 16384, keep
# 50 % (the launch of the backward segment over keys 0 .. 8191: 470.9 MB read + 213.5 MB written).
TRAFFIC_PER_UNIT = {"attn_bwd_dkdv_tc": ("key row", (470.904832e6 + 213.455360e6) / 8192)}


def traffic_units(name, case, ks, seg):
    """Units (as in TRAFFIC_PER_UNIT) a step's launches of kernel `name` process, summed."""
    if name == "attn_bwd_dkdv_tc":
        tot = 0
        for k in ks:
            n = k * case.blk
            tot += sum(min(s0 + seg, n) for s0 in range(0, n, seg))
        return tot
    return None


def step_flops(case, ks, scoring="exact"):
    return sum(v for k, v in work_model(case, ks, 4096, scoring).values() if k == "flop")


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except Exception:
                pass
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * (mx or 1)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- oracle timing
def oracle_weights(case):
    """The oracle's float64 copies of every layer's weights (built once, outside the timing)."""
    from oracle import layer as oly
    return [oly.Weights.from_bits(p, case.shape) for p in case.layers]


def oracle_sample(case, n_tok, keep, Ws):
    """Time the CPU oracle on a bounded sample of the workload: the first n_tok tokens of the
    sequence through every layer of the stack, as the GPU step runs them -- per layer the
    salient-row scaling (layers >= 1), the oracle's q / k of the sample's rows, block scores,
    top-k selection at the layer's keep fraction and the retained-token forward; then the
    backward of every layer in reverse with the upstream gradient's first n_tok rows (the same
    diagonal on dX after layers >= 1).  Ws: oracle_weights(case).  Returns (seconds, algorithmic
    flops of the sample)."""
    from oracle import layer as oly
    from oracle import scores as osc
    from oracle import select as osel
    from oracle.bf16 import from_bits, round_bf16
    sh = case.shape
    blk = min(case.blk, n_tok)
    nb = n_tok // blk
    X = from_bits(case.x[:n_tok])
    G = from_bits(case.g[:n_tok])
    HD = sh.heads * sh.head_dim
    P = 4 * sh.hidden * HD + 3 * sh.hidden * sh.ffn
    flops = 0.0
    t0 = time.perf_counter()
    ctxs = []
    for l, W in enumerate(Ws):
        sal = case.salient[l][case.salient[l] < n_tok] if l > 0 else []
        if len(sal):
            X[sal] = round_bf16(X[sal] * case.salient_scale)
        pr = oly.project_qk(X, np.arange(n_tok), W, rnd=True)
        sc = osc.block_scores_softmax_mass(pr["q"], pr["k"], blk)
        k = max(1, osel.topk_count(keep[l], nb))
        idx, n, _ = osel.select_topk(sc, k)
        X, ctx = oly.sparse_layer_fwd(X, idx, n, blk, W, rnd=True)
        ctxs.append((W, ctx, sal))
        nr = n * blk
        flops += (4.0 * sh.hidden * HD * n_tok + 2.0 * sh.head_dim * sh.heads * causal_pairs(n_tok)
                  + 2.0 * P * nr + 4.0 * sh.head_dim * sh.heads * causal_pairs(nr))
    for W, ctx, sal in reversed(ctxs):
        G, _ = oly.sparse_layer_bwd(ctx, G, W, 4096)
        if len(sal):
            G[sal] = round_bf16(G[sal] * case.salient_scale)
        nr = ctx["x"].shape[0] if ctx is not None else 0
        flops += 2.0 * P * nr + 10.0 * sh.head_dim * sh.heads * causal_pairs(nr)
    return time.perf_counter() - t0, flops


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args):
    """The reference arm: the CPU oracle (numpy float64, the machine's host cores), each step a
    bounded sample of the workload (oracle_sample); value = the sample's tokens per second of
    measured time.  The sample is cheaper per token than the full 32K-token step (its causal
    attention and scoring cover n_tok tokens, not S), so the ratio against the GPU arm
    understates the GPU's advantage."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    case = synth.gen_workload(args.workload, seed=0)
    keep = list(w.keep) if len(w.keep) == w.n_layers else [w.keep[0]] * w.n_layers
    Ws = oracle_weights(case)
    for _ in range(args.warmup):
        oracle_sample(case, REF_TOKENS, keep, Ws)
    ts = []
    for _ in range(args.steps):
        dt, _ = oracle_sample(case, REF_TOKENS, keep, Ws)
        ts.append(dt)
    t = sum(ts) / len(ts)
    value = REF_TOKENS / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": gpu_arm_config(case, w, keep, args.gpus),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": "tokens/s", "cores": cpu_cores(),
                             "sample": f"per step: the first {REF_TOKENS} tokens of the sequence through all "
                                       f"{len(case.layers)} layers (oracle q/k, block scores, top-k selection, "
                                       f"retained-token forward, then the backward in reverse); tokens/s = "
                                       f"{REF_TOKENS} / measured step time"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def gpu_arm_config(case, w, keep, world):
    """The `config` object of the JSON line (the same for both arms)."""
    sh = case.shape
    nb = case.S // case.blk
    return {"workload": w.name, "seq_len": case.S, "global_batch": world, "layers": len(case.layers),
            "hidden": sh.hidden, "heads": sh.heads, "ffn": sh.ffn, "block": case.blk, "keep": keep,
            "n_kept_blocks": [synth_k(p, nb) for p in keep], "segment_tokens": case.segment_tokens,
            "parallelism": f"replicas{world}",
            "l2": f"inputs larger than L2 (X {case.S * sh.hidden * 2 / 2 ** 20:.0f} MiB, weights "
                  f"{len(case.layers) * (4 * sh.hidden ** 2 + 3 * sh.hidden * sh.ffn) * 2 / 2 ** 30:.1f} GiB)"}


def synth_k(p, nb):
    from math import ceil
    return max(0, min(nb, ceil(p * nb - 1e-6)))


# ---------------------------------------------------------------------------- GPU arm
def measure_lm_loss(J, torch, dev, S, h, tf_peak, V=32000, seg=4096):
    """Segmented causal-LM loss (vocabulary cross-entropy and its hidden-state gradient) at
    the workload's sequence length and hidden size with the Llama-2 vocabulary (32000),
    4096-token segments: synthetic hidden states N(0,1), output embedding N(0,0.02),
    uniform labels.  Algorithmic work 4 S V h flop (logits and gradient GEMMs); device
    time per call over 3 back-to-back calls, median of 3.  Peak workspace against the
    unsegmented form (segment = S)."""
    g = torch.Generator(device=dev).manual_seed(0)
    hid = torch.randn(S, h, device=dev, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, h, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    lab = torch.randint(0, V, (S,), device=dev, generator=g, dtype=torch.int32)
    lib = J._lib.load()
    ws_b = lib.jenga_lm_loss_workspace_bytes(S, h, V, seg)
    ws_full = lib.jenga_lm_loss_workspace_bytes(S, h, V, S)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    dh = torch.empty(S, h, dtype=torch.bfloat16, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    fn = lambda: J.jenga_lm_loss_segmented(hid, w, lab, segment_tokens=seg, dhidden=dh, loss=loss, ws=ws)
    for _ in range(2):
        fn()
    ts = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(3):
            fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / 3 / 1e3)
    t = sorted(ts)[1]
    J.jenga_check_device_status()
    fl = 4.0 * S * V * h
    out = {"S": S, "h": h, "V": V, "segment_tokens": seg, "ms": t * 1e3, "tokens_per_s": S / t,
           "tflops": fl / t / 1e12, "frac_bf16_sustained": fl / t / 1e12 / tf_peak,
           "workspace_gib": ws_b / 2 ** 30, "workspace_unsegmented_gib": ws_full / 2 ** 30,
           "loss": float(loss.item()), "loss_uniform_reference": float(np.log(V))}
    del hid, w, lab, ws, dh
    torch.cuda.empty_cache()
    return out


def measure_movement(J, torch, dev, X0, case, ks, hbm):
    """Standalone timing of the HBM-bound entry points at the workload's sizes: gather and
    scatter-add of layer 0's retained rows of X (bf16 [S, h]), and threshold selection
    (ABS_GE) over 2^26 fp32 scores.  Algorithmic bytes: gather 2 n h e, scatter-add 3 n h e
    (eliminated rows cost nothing), select 4 nb read + 4 nb (idx, -1 past n_kept) + nb + 4
    written, MLP-block criterion 2 n F read (the retained rows' intermediate activation).  Each
    call moves more than the 126 MB L2; CUDA events around 10 back-to-back calls, median of 5
    such groups after 3 warm-ups."""
    blk, S, h = case.blk, case.S, X0.shape[1]
    nb = S // blk
    k0 = ks[0]
    idx = torch.full((1, nb), -1, dtype=torch.int32, device=dev)
    idx[0, :k0] = torch.arange(0, nb, nb / k0, device=dev).to(torch.int32)[:k0]  # spread over the sequence
    nk = torch.tensor([k0], dtype=torch.int32, device=dev)
    n = k0 * blk
    xg = torch.empty(n, h, dtype=X0.dtype, device=dev)
    x2 = X0.clone()

    def med(fn, reps=10):
        # device time per call: `reps` calls back to back between two events (the host
        # enqueues ahead of the device, so launch latency is not timed), median of 5
        for _ in range(3):
            fn()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3 / reps)
        return sorted(ts)[len(ts) // 2]

    out = {}
    t = med(lambda: J.jenga_gather(X0, idx, nk, blk, n, out=xg))
    by = 2.0 * n * h * X0.element_size()
    out["gather"] = {"rows": n, "bytes": by, "us": t * 1e6, "gbs": by / t / 1e9, "frac_hbm": by / t / 1e9 / hbm}
    t = med(lambda: J.jenga_scatter_add(x2, xg, idx, nk, blk, 1.0))
    by = 3.0 * n * h * X0.element_size()
    out["scatter_add"] = {"rows": n, "bytes": by, "us": t * 1e6, "gbs": by / t / 1e9, "frac_hbm": by / t / 1e9 / hbm}
    del xg, x2
    # MLP-block criterion over the retained blocks' intermediate activation [n, F]
    F = case.shape.ffn
    act = torch.randn(n, F, device=dev, generator=torch.Generator(device=dev).manual_seed(1)).to(torch.bfloat16)
    msc = torch.empty(k0, dtype=torch.float32, device=dev)
    t = med(lambda: J.jenga_mlp_block_scores(act, blk, nk, out=msc))
    by = 2.0 * n * F + 4.0 * k0
    out["mlp_block_scores"] = {"rows": n, "ffn": F, "bytes": by, "us": t * 1e6, "gbs": by / t / 1e9,
                               "frac_hbm": by / t / 1e9 / hbm}
    del act
    nsel = 1 << 26
    g = torch.Generator(device=dev).manual_seed(0)
    sc = torch.rand(1, nsel, device=dev, generator=g)
    sel_out = (torch.empty(1, nsel, dtype=torch.int32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
               torch.empty(1, nsel, dtype=torch.uint8, device=dev))
    t = med(lambda: J.jenga_select(sc, "abs_ge", 0.5, out=sel_out))
    kept = int(sel_out[1].item())
    by = 4.0 * nsel + 4.0 * nsel + nsel + 4  # scores in; idx (kept, then -1 fill), mask, n_kept out
    out["select_abs_ge"] = {"scores": nsel, "kept": kept, "bytes": by, "us": t * 1e6, "gbs": by / t / 1e9,
                            "frac_hbm": by / t / 1e9 / hbm}
    out["hbm_peak_gbs"] = hbm
    return out


def max_over_ranks(x, device):
    """The per-rank value's maximum over the process group (the timing rule for N ranks:
    the slowest replica sets the step time); x itself with no group or one rank."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(S, world, ms):
    """Whole-job throughput of `world` independent replicas of an S-token step that took
    ms milliseconds on the slowest rank."""
    return S * world / (ms / 1e3)


def cpu_baseline_one_thread():
    """The cpu_baseline leg's one-thread figure: the CPU oracle on one host thread, each small
    workload in full: ``score_fp32`` (S 512, 4 heads x 64, blocks of 32: fp32 block scores,
    mean-threshold selection, gather, scatter-add of 2 x the gathered rows) and ``llama7b_s4k``
    (one 7B-shaped layer at S 4096, blocks of 64, keep 50 %: q/k of all rows, block scores,
    top-k selection, retained-token forward and backward).  Inputs and oracle weights are
    built before the clock starts."""
    from threadpoolctl import threadpool_limits
    from oracle import movement as omv
    from oracle import scores as osc
    from oracle import select as osel
    out = {}
    with threadpool_limits(1):
        c = synth.gen_score_case(0)
        q = c.q.reshape(c.S, c.H, c.D).astype(np.float64)
        k = c.k.reshape(c.S, c.H, c.D).astype(np.float64)
        x = c.x.astype(np.float64)
        t0 = time.perf_counter()
        sc = osc.block_scores_softmax_mass(q, k, c.blk)
        (idx, n, _), _ = osel.select_mean_ge(sc)
        xg = omv.gather(x, idx, n, c.blk)
        omv.scatter_add(x, xg, idx, n, c.blk, 2.0, "f32")
        dt = time.perf_counter() - t0
        out["score_fp32"] = {"seconds": dt, "tokens_per_s": c.S / dt, "kept_blocks": int(n)}
        w = synth.WORKLOADS["llama7b_s4k"]
        case = synth.gen_workload("llama7b_s4k", seed=0)
        Ws = oracle_weights(case)
        dt, flops = oracle_sample(case, case.S, list(w.keep), Ws)
        out["llama7b_s4k"] = {"seconds": dt, "tokens_per_s": case.S / dt, "gflop": flops / 1e9}
    print(json.dumps({"cpu_baseline_one_thread": out, "kind": "oracle", "cores": 1}), flush=True)


def main():
    args = parse()
    if args.cpu_baseline_one_thread:
        cpu_baseline_one_thread()
        return
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=torch.device("cuda", local))

    import token_sparse_long_b200 as J

    def bits_to_torch(u16, device):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).to(device)

    def layer_handle(p, shape):
        t = {k: bits_to_torch(getattr(p, k), dev) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "attn_norm",
                                                             "mlp_norm", "aq", "bq", "av", "bv")}
        return J.LayerHandle(**t, heads=shape.heads, head_dim=shape.head_dim, rms_eps=shape.rms_eps,
                             rope_theta=shape.rope_theta, lora_scale=shape.lora_scale)

    J._lib.load()
    w = synth.WORKLOADS[args.workload]
    case = synth.gen_workload(args.workload, seed=0)
    sh = case.shape
    S, blk, nb, HD = case.S, case.blk, case.S // case.blk, sh.heads * sh.head_dim
    keep = list(w.keep) if len(w.keep) == w.n_layers else [w.keep[0]] * w.n_layers
    ks = [synth_k(p, nb) for p in keep]
    dev = torch.device("cuda", local)

    layers = [layer_handle(p, sh) for p in case.layers]
    X0 = bits_to_torch(case.x, dev)
    G0 = bits_to_torch(case.g, dev)
    sal = [torch.from_numpy(s.astype(np.int32)).to(dev) for s in case.salient]
    X = torch.empty_like(X0)
    dX = torch.empty_like(G0)
    seg = case.segment_tokens
    pred = None  # (w1, b1, w2, b2) on the device when the workload scores blocks with the predictor
    if case.predictor is not None:
        pr = case.predictor
        pred = (bits_to_torch(pr["w1"], dev), torch.from_numpy(pr["b1"]).to(dev),
                bits_to_torch(pr["w2"], dev).reshape(-1), torch.from_numpy(pr["b2"]).to(dev))

    def buffers(kmaxes):
        b = {}
        b["qk"] = torch.empty(S, 2 * HD, dtype=torch.bfloat16, device=dev)
        b["qk_ws"] = torch.empty(layers[0].qk_ws_bytes(S), dtype=torch.uint8, device=dev)
        lib = J._lib.load()
        b["sc_ws"] = torch.empty(lib.jenga_score_workspace_bytes(1, S, sh.heads, sh.head_dim, blk),
                                 dtype=torch.uint8, device=dev)
        b["scores"] = [torch.empty(1, nb, dtype=torch.float32, device=dev) for _ in kmaxes]
        b["sel"] = [(torch.empty(1, nb, dtype=torch.int32, device=dev), torch.empty(1, dtype=torch.int32, device=dev),
                     torch.empty(1, nb, dtype=torch.uint8, device=dev)) for _ in kmaxes]
        b["saved"] = [torch.empty(L.saved_bytes(blk, k), dtype=torch.uint8, device=dev) for L, k in zip(layers, kmaxes)]
        b["fws"] = torch.empty(max(L.fwd_ws_bytes(blk, k) for L, k in zip(layers, kmaxes)), dtype=torch.uint8,
                               device=dev)
        b["bws"] = torch.empty(max(L.bwd_ws_bytes(blk, k, seg) for L, k in zip(layers, kmaxes)), dtype=torch.uint8,
                               device=dev)
        b["grads"] = [J.new_lora_grads(L) for L in layers]
        if pred is not None:
            b["pred_ws"] = torch.empty(lib.jenga_predict_workspace_bytes(1, S, sh.hidden, blk), dtype=torch.uint8,
                                       device=dev)
        return b

    def step(b, kmaxes, sparse=True):
        for l, L in enumerate(layers):
            if l > 0 and len(case.salient[l]):
                J.jenga_scale_rows(X, sal[l], case.salient_scale)
            idx, nk, mask = b["sel"][l]
            if sparse and pred is not None:  # block scores from the predictor MLP (a10)
                J.jenga_predict_blocks(X, blk, *pred, out=b["scores"][l], ws=b["pred_ws"])
                J.jenga_select(b["scores"][l], "topk_frac", keep[l], out=(idx, nk, mask))
            elif sparse:
                J.jenga_layer_score_qk(L, X, out=b["qk"], ws=b["qk_ws"])
                J.jenga_score_blocks(b["qk"][:, :HD], b["qk"][:, HD:], sh.heads, sh.head_dim, blk, out=b["scores"][l],
                                     ws=b["sc_ws"])
                J.jenga_select(b["scores"][l], "topk_frac", keep[l], out=(idx, nk, mask))
            # with exact scoring the retained rows' q and k come from the scoring's q | k
            J.jenga_sparse_layer_fwd(L, X, idx, nk, blk, kmaxes[l], saved=b["saved"][l], ws=b["fws"],
                                     qk=b["qk"] if (sparse and pred is None) else None)
        for l in reversed(range(len(layers))):
            idx, nk, _ = b["sel"][l]
            J.jenga_sparse_layer_bwd(layers[l], dX, idx, nk, blk, kmaxes[l], b["saved"][l], b["grads"][l],
                                     segment_tokens=seg, ws=b["bws"])
            if l > 0 and len(case.salient[l]):
                J.jenga_scale_rows(dX, sal[l], case.salient_scale)

    def zero_grads(b):
        for g in b["grads"]:
            for t in g.values():
                t.zero_()

    def device_step(b, kmaxes, sparse=True):
        X.copy_(X0)
        dX.copy_(G0)
        zero_grads(b)
        step(b, kmaxes, sparse)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, K, Wu):
        for _ in range(Wu):
            fn()
        torch.cuda.synchronize()
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(K):
            fn()
        e.record()
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(s.elapsed_time(e) / K, dev)

    # ---------------- sparse step (headline)
    torch.cuda.reset_peak_memory_stats(dev)
    b = buffers(ks)
    J.jenga_check_device_status()
    for _ in range(args.warmup):
        device_step(b, ks)
    torch.cuda.synchronize()
    J.jenga_check_device_status()
    clocks = ClockSampler(local)
    clocks.start()
    J.jenga_profile_enable(True)
    ms = timed(lambda: device_step(b, ks), args.steps, 0)
    prof = J.jenga_profile_report()
    J.jenga_profile_enable(False)
    clk = clocks.stop()
    J.jenga_check_device_status()
    peak_sparse = torch.cuda.max_memory_allocated(dev) / 2 ** 30
    n_kept = [int(b["sel"][l][1].item()) for l in range(len(layers))]

    # ---------------- roofline of the dominant kernel (live per-launch events, timed region)
    hbm, tf_burst, tf_sus, peak_src = load_peaks()
    scoring = "predictor" if pred is not None else "exact"
    wm = work_model(case, ks, seg, scoring)
    top = max(prof.items(), key=lambda kv: kv[1]["ms"])
    tname, tstat = top
    launches = sum(v["launches"] for v in prof.values())
    roof = None
    if tname in wm:
        kind, amount = wm[tname]
        sec = tstat["ms"] / 1e3 / args.steps
        if kind == "flop":
            ach = amount / sec / 1e12
            traffic = None
            if tname in TRAFFIC_PER_UNIT:
                units = traffic_units(tname, case, ks, seg)
                traffic = TRAFFIC_PER_UNIT[tname][1] * units / (tstat["launches"] / args.steps)
            roof = {"kernel": tname, "bound": "tensor", "achieved": ach, "peak": tf_sus, "unit": "TFLOP/s",
                    "frac": ach / tf_sus, "traffic": traffic, "peak_source": f"{peak_src} bf16 sustained",
                    "launches_per_step": tstat["launches"] / args.steps, "share": tstat["ms"] / sum(
                        v["ms"] for v in prof.values())}
        else:
            ach = amount / sec / 1e9
            roof = {"kernel": tname, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                    "frac": ach / hbm, "traffic": None, "peak_source": f"{peak_src} HBM copy"}
    kernels = {}
    for k, v in sorted(prof.items(), key=lambda kv: -kv[1]["ms"]):
        e = {"ms_per_step": v["ms"] / args.steps, "launches_per_step": v["launches"] / args.steps}
        if k in wm:
            kind, amount = wm[k]
            sec = v["ms"] / 1e3 / args.steps
            if kind == "flop":
                e["tflops"] = amount / sec / 1e12
                e["frac_bf16_sustained"] = e["tflops"] / tf_sus
            else:
                e["gbs"] = amount / sec / 1e9
        kernels[k] = e

    # ---------------- predictor path: agreement of predicted and exact block scores (layer 0
    # input; outside the timed region) and the predictor kernels' HBM roofline
    predictor = None
    if pred is not None:
        import scipy.stats
        L0 = layers[0]
        pws = torch.empty(J._lib.load().jenga_predict_workspace_bytes(1, S, sh.hidden, blk), dtype=torch.uint8,
                          device=dev)
        p_sc = J.jenga_predict_blocks(X0, blk, *pred, ws=pws)
        J.jenga_layer_score_qk(L0, X0, out=b["qk"], ws=b["qk_ws"])
        e_sc = J.jenga_score_blocks(b["qk"][:, :HD], b["qk"][:, HD:], sh.heads, sh.head_dim, blk, ws=b["sc_ws"])
        ps, es = p_sc.reshape(-1).double().cpu().numpy(), e_sc.reshape(-1).double().cpu().numpy()
        kk = ks[0]

        def topk_set(v):  # (score desc, index asc), the selection's tie-break
            return set(np.lexsort((np.arange(v.size), -v))[:kk].tolist())

        for _ in range(3):
            J.jenga_predict_blocks(X0, blk, *pred, out=p_sc, ws=pws)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for _ in range(10):
            J.jenga_predict_blocks(X0, blk, *pred, out=p_sc, ws=pws)
        ev1.record()
        torch.cuda.synchronize()
        us = ev0.elapsed_time(ev1) * 100.0  # per call, 10 back to back
        by = S * sh.hidden * X0.element_size()
        # the pages' Q/K predictor pair (Eq. 3) on the same input: ranks 128, 128, output 16
        gq = torch.Generator(device=dev).manual_seed(1)
        pw = lambda: tuple((torch.randn(*shp, device=dev, generator=gq) * sd).to(torch.bfloat16)
                           for shp, sd in (((128, sh.hidden), 0.02), ((128, 128), 0.1), ((16, 128), 0.1)))
        qw_, kw_ = pw(), pw()
        pq = J.jenga_predict_blocks_qk(X0, blk, qw_, kw_)
        for _ in range(3):
            J.jenga_predict_blocks_qk(X0, blk, qw_, kw_, out=pq)
        ev0.record()
        for _ in range(10):
            J.jenga_predict_blocks_qk(X0, blk, qw_, kw_, out=pq)
        ev1.record()
        torch.cuda.synchronize()
        us_pair = ev0.elapsed_time(ev1) * 100.0
        pqs = pq.reshape(-1).double().cpu().numpy()
        predictor_pair = {"us_per_call": us_pair, "gbs": by / us_pair / 1e3, "frac_hbm": by / us_pair / 1e3 / hbm,
                          "ranks": [128, 128, 16],
                          "rank_agreement": {"spearman": float(scipy.stats.spearmanr(pqs, es).statistic),
                                             "topk_overlap": len(topk_set(pqs) & topk_set(es)) / kk}}
        predictor = {"rank_agreement": {"spearman": float(scipy.stats.spearmanr(ps, es).statistic),
                                        "kendall_tau_b": float(scipy.stats.kendalltau(ps, es).statistic),
                                        "topk_overlap": len(topk_set(ps) & topk_set(es)) / kk, "k": kk, "nb": nb},
                     "us_per_call": us, "bytes": by, "gbs": by / us / 1e3, "frac_hbm": by / us / 1e3 / hbm,
                     "pair_qk": predictor_pair,
                     "note": "random-init predictor weights: agreement with exact scores is not expected"}

    # ---------------- dense comparison (keep-all, no scoring)
    dense = None
    if not args.no_dense:
        del b
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        kd = [nb] * len(layers)
        bd = buffers(kd)
        for l in range(len(layers)):
            idx, nk, _ = bd["sel"][l]
            idx.copy_(torch.arange(nb, dtype=torch.int32, device=dev)[None])
            nk.fill_(nb)
        ms_d = timed(lambda: device_step(bd, kd, sparse=False), max(1, min(2, args.steps)), 1)
        dense = {"tokens_per_s": S * world / (ms_d / 1e3), "ms_per_step": ms_d,
                 "peak_mem_gib": torch.cuda.max_memory_allocated(dev) / 2 ** 30,
                 "note": "keep-all retained-token layers without scoring (same kernels)"}
        del bd
        torch.cuda.empty_cache()

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        b = buffers(ks)
        hX = torch.empty(X0.shape, dtype=X0.dtype, pin_memory=True)
        hX.copy_(X0.cpu())
        hG = torch.empty(G0.shape, dtype=G0.dtype, pin_memory=True)
        hG.copy_(G0.cpu())
        hgrads = [{k: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for k, t in g.items()} for g in b["grads"]]

        def e2e_step():
            X.copy_(hX, non_blocking=True)
            dX.copy_(hG, non_blocking=True)
            zero_grads(b)
            step(b, ks)
            for hg, g in zip(hgrads, b["grads"]):
                for k in g:
                    hg[k].copy_(g[k], non_blocking=True)

        ms_e = timed(e2e_step, args.steps, 1)
        h2d = hX.numel() * 2 + hG.numel() * 2
        d2h = sum(t.numel() * 4 for g in hgrads for t in g.values())
        e2e = {"value": S * world / (ms_e / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e}
        del b

    # ---------------- standalone token movement and selection (HBM-bound kernels)
    movement = None
    if not args.no_movement:
        movement = measure_movement(J, torch, dev, X0, case, ks, hbm)

    # ---------------- paper-form block-max score (Eq. 2) on layer 0's q | k of all S rows
    paper = None
    if not args.no_movement and pred is None:
        bq = buffers(ks)
        J.jenga_layer_score_qk(layers[0], X0, out=bq["qk"], ws=bq["qk_ws"])
        qk = bq["qk"]
        fn = lambda: J.jenga_score_blocks(qk[:, :HD], qk[:, HD:], sh.heads, sh.head_dim, blk, mode="paper_blockmax",
                                          out=bq["scores"][0], ws=bq["sc_ws"])
        for _ in range(2):
            fn()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for _ in range(3):
            fn()
        ev1.record()
        torch.cuda.synchronize()
        J.jenga_check_device_status()
        t = ev0.elapsed_time(ev1) / 3 / 1e3
        fl = 2.0 * sh.head_dim * sh.heads * causal_pairs(S)
        paper = {"ms": t * 1e3, "tflops": fl / t / 1e12, "frac_bf16_sustained": fl / t / 1e12 / tf_sus,
                 "work": "one QK^T product per causal (query, key) pair and head (2 D H flop per pair)"}
        del bq
        torch.cuda.empty_cache()

    # ---------------- segmented LM-head loss (segment-based peak cutting)
    lm_loss = None
    if not args.no_lm_loss:
        lm_loss = measure_lm_loss(J, torch, dev, S, sh.hidden, tf_sus)

    # ---------------- CPU baseline (oracle, rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Ws = oracle_weights(case)
        dt, fl = oracle_sample(case, BASELINE_TOKENS, keep, Ws)
        del Ws
        full = step_flops(case, ks, scoring)
        cpu = {"value": BASELINE_TOKENS / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"the first {BASELINE_TOKENS} tokens through all {len(layers)} layers (oracle q/k, block "
                         f"scores, top-k selection, retained-token forward, backward in reverse): {dt:.1f} s, "
                         f"{fl / 1e9:.0f} GFLOP; tokens/s = {BASELINE_TOKENS} / time (cheaper per token than the "
                         f"full {S}-token step)",
               "flop_scaled_full_step_tokens_per_s": S / (full / (fl / dt))}

    if rank == 0:
        line = {"metric": METRIC, "value": replica_tokens_per_s(S, world, ms), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": gpu_arm_config(case, w, keep, world),
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "movement": movement,
                "clocks": clk, "peak_mem_gib": peak_sparse, "dense": dense,
                **({"predictor": predictor} if predictor is not None else {}), "lm_loss": lm_loss,
                "paper_blockmax_score": paper, "step_tflop": step_flops(case, ks, scoring) / 1e12, "kernels": kernels}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
