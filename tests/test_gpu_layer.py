"""GPU parity of the retained-token layer (a1..a9) against the CPU oracle.

The oracle runs on the GPU's kept-block list and the same seeded inputs, so a
selection difference cannot cascade.  Bars:
* the layer output and the input gradient (bf16): max |gpu - oracle| / rms(oracle)
  <= 3e-2, with one bf16 ulp of the stored value forgiven (that final rounding may land
  on either neighbour);
* the same measured on the sub-block contributions alone (out - x, dX - G), which a
  real fault moves by O(1): <= 3e-2 both ways;
* LoRA gradients (fp32): max |gpu - oracle| / rms(oracle) <= 3e-2;
* eliminated rows exactly unchanged (x) and exactly the identity gradient (G)."""
import numpy as np
import pytest
import torch

import synth
from oracle import select as osel
from tests.layer_harness import (SMALL, check_layer_against_oracle, check_qk_all, check_scores, check_topk_selection,
                                 oracle_layer, oracle_qk_all, oracle_scores_from_qk, rel_max, rel_max_ulp,
                                 run_layer_gpu, small_case, torch_to_f64)
from oracle import scores as osc

pytestmark = pytest.mark.gpu
TOL = 3e-2


@pytest.fixture(scope="module")
def J():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import token_sparse_long_b200 as J
    J._lib.load()
    return J


def _check(case, gpu, seg=None):
    Xo, dX, grads, X, G = oracle_layer(case, gpu, seg=seg)
    e = check_layer_against_oracle(case.S, case.blk, gpu["idx"], gpu["n_kept"], gpu["out"], gpu["dx"],
                                   gpu["grads"], Xo, dX, grads, X, G)
    return e.get("out"), e.get("dx")


@pytest.mark.parametrize("keep,seg,lora_b", [(0.5, 4096, 0.02), (0.25, 128, 0.02), (1.0, 256, 0.0),
                                             (0.75, 4096, 0.0)])
def test_small_layer(J, keep, seg, lora_b):
    case = small_case(seed=5, S=1024, blk=64, lora_b_std=lora_b)
    gpu = run_layer_gpu(case, keep=keep, seg=seg)
    ref_sc = oracle_scores_from_qk(torch_to_f64(gpu["qk"]), SMALL.heads, SMALL.head_dim, case.blk)
    assert np.all(np.abs(gpu["scores"] - ref_sc) / ref_sc < 2e-2)
    oi, on, _ = osel.select_topk(gpu["scores"], osel.topk_count(keep, case.S // case.blk))
    assert on == gpu["n_kept"] and np.array_equal(oi, gpu["idx"])
    _check(case, gpu)


def test_mean_threshold_layer_device_count(J):
    # data-dependent n_kept (mean threshold): grids sized for all blocks, kernels read
    # the count on the device
    case = small_case(seed=6, S=512, blk=128)
    gpu = run_layer_gpu(case, keep=0.0, seg=256, mode="mean_ge")
    (oi, on, _), _ = osel.select_mean_ge(gpu["scores"])
    assert on == gpu["n_kept"] and np.array_equal(oi, gpu["idx"])
    _check(case, gpu)


def test_keep_none(J):
    case = small_case(seed=7, S=512, blk=64)
    gpu = run_layer_gpu(case, keep=0.0, seg=4096)
    assert gpu["n_kept"] == 0
    X = gpu["x_in"]
    assert np.array_equal(gpu["out"], X)
    assert all(np.abs(v).max() == 0 for v in gpu["grads"].values())


def test_segmented_equals_unsegmented(J):
    case = small_case(seed=8, S=1024, blk=64)
    a = run_layer_gpu(case, keep=0.75, seg=4096)
    b = run_layer_gpu(case, keep=0.75, seg=128, handle=a["handle"])
    assert np.array_equal(a["out"], b["out"])
    # same quantity, different fp32 summation order of the key/value gradients
    assert rel_max_ulp(b["dx"], a["dx"]) < TOL
    for k in a["grads"]:
        assert rel_max(b["grads"][k], a["grads"][k]) < 1e-2
    _check(case, b)


def test_llama7b_shape_s4k_layer(J):
    """One 7B-shaped layer at S=4096, block 64, keep 50% (the single-layer workload): the
    q | k of all rows (a1) against the oracle's, the block scores against the oracle's
    scores from the oracle's own q and k, bit-exact selection on the GPU's scores, and the
    layer forward / backward."""
    case = synth.gen_workload("llama7b_s4k", seed=0, lora_b_std=0.02)
    gpu = run_layer_gpu(case, keep=0.5, seg=4096)
    q_o, k_o = oracle_qk_all(case)
    check_qk_all(gpu["qk"], q_o, k_o)
    o_sc = osc.block_scores_softmax_mass(q_o, k_o, case.blk)
    check_scores(gpu["scores"], o_sc)
    check_topk_selection(gpu["scores"], gpu["idx"], gpu["n_kept"], 32, o_sc)
    assert gpu["n_kept"] == 32
    _check(case, gpu)


@pytest.mark.parametrize("S,blk", [(1024, 64), (2048, 128)])
def test_small_layer_qk_all_rows_and_scores(J, S, blk):
    """a1 on the small layer: the q | k of ALL rows (retained and eliminated) against the
    oracle's, and the scores from them against the oracle's scores from its own q, k."""
    case = small_case(seed=11, S=S, blk=blk)
    gpu = run_layer_gpu(case, keep=0.5, seg=4096)
    q_o, k_o = oracle_qk_all(case)
    check_qk_all(gpu["qk"], q_o, k_o)
    o_sc = osc.block_scores_softmax_mass(q_o, k_o, case.blk)
    check_scores(gpu["scores"], o_sc)
    check_topk_selection(gpu["scores"], gpu["idx"], gpu["n_kept"], osel.topk_count(0.5, S // blk), o_sc)


@pytest.mark.parametrize("shape_name", ["small", "llama7b_s4k"])
def test_forward_reusing_scoring_qk_is_bit_identical(J, shape_name):
    """The forward may take the retained rows' q and k from the scoring's q | k of all rows
    (same x, same kernels): outputs, saved context and gradients are bit-identical."""
    from tests.layer_harness import bits_to_torch, layer_handle
    case = small_case(seed=9, S=1024, blk=64) if shape_name == "small" else synth.gen_workload("llama7b_s4k", seed=1,
                                                                                               lora_b_std=0.02)
    sh = case.shape
    L = layer_handle(case.layers[0], sh)
    HD = sh.heads * sh.head_dim
    x0 = bits_to_torch(case.x)
    qk = J.jenga_layer_score_qk(L, x0)
    sc = J.jenga_score_blocks(qk[:, :HD], qk[:, HD:], sh.heads, sh.head_dim, case.blk)
    idx, nk, _ = J.jenga_select(sc, "topk_frac", 0.5)
    kmax = osel.topk_count(0.5, case.S // case.blk)
    res = []
    for reuse in (False, True):
        x = x0.clone()
        saved = torch.zeros(L.saved_bytes(case.blk, kmax), dtype=torch.uint8, device="cuda")  # padding compares equal
        J.jenga_sparse_layer_fwd(L, x, idx, nk, case.blk, kmax, saved=saved, qk=qk if reuse else None)
        dx = bits_to_torch(case.g)
        grads = J.new_lora_grads(L)
        J.jenga_sparse_layer_bwd(L, dx, idx, nk, case.blk, kmax, saved, grads, segment_tokens=1024)
        J.jenga_check_device_status()
        res.append((x, saved, dx, grads))
    (xa, sa, da, ga), (xb, sb, db, gb) = res
    assert torch.equal(xa, xb) and torch.equal(sa, sb) and torch.equal(da, db)
    assert all(torch.equal(ga[k], gb[k]) for k in ga)


# ------------------------------------------------------------------ MLP-block elimination (Jenga summary §4.2.4)
def _run_mlp_layer(J, case, keep, mlp_mode, mlp_param, seg, L=None):
    from tests.layer_harness import bits_to_torch, layer_handle
    sh = case.shape
    HD = sh.heads * sh.head_dim
    L = L or layer_handle(case.layers[0], sh)
    x = bits_to_torch(case.x)
    qk = J.jenga_layer_score_qk(L, x)
    sc = J.jenga_score_blocks(qk[:, :HD], qk[:, HD:], sh.heads, sh.head_dim, case.blk)
    idx, nk, _ = J.jenga_select(sc, "topk_frac", keep)
    kmax = osel.topk_count(keep, case.S // case.blk)
    saved = torch.zeros(L.saved_bytes(case.blk, kmax), dtype=torch.uint8, device="cuda")
    if mlp_mode is None:
        J.jenga_sparse_layer_fwd(L, x, idx, nk, case.blk, kmax, saved=saved, qk=qk)
        msc = mpos = nm = None
    else:
        _, msc, mpos, nm = J.jenga_sparse_layer_fwd_mlp(L, x, idx, nk, case.blk, kmax, mlp_mode, mlp_param, saved=saved,
                                                        qk=qk)
    out = x.clone()
    dx = bits_to_torch(case.g)
    grads = J.new_lora_grads(L)
    J.jenga_sparse_layer_bwd(L, dx, idx, nk, case.blk, kmax, saved, grads, segment_tokens=seg)
    J.jenga_check_device_status()
    torch.cuda.synchronize()
    return dict(L=L, idx=idx.cpu().numpy(), n_kept=int(nk.cpu()[0]), kmax=kmax, saved=saved, out=out, dx=dx,
                grads=grads, mlp_scores=None if msc is None else msc.cpu().numpy().astype(np.float64),
                mlp_pos=None if mpos is None else mpos.cpu().numpy(), n_mlp=None if nm is None else int(nm.cpu()[0]))


def test_mlp_elimination_keep_all_is_bit_identical(J):
    """The MLP keeping every retained block reproduces the plain layer bit for bit."""
    case = small_case(seed=12, S=1024, blk=64)
    a = _run_mlp_layer(J, case, 0.5, None, 0, 256)
    b = _run_mlp_layer(J, case, 0.5, "topk_frac", 1.0, 256, L=a["L"])
    assert b["n_mlp"] == a["kmax"]
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["saved"], b["saved"]) and torch.equal(a["dx"], b["dx"])
    assert all(torch.equal(a["grads"][k], b["grads"][k]) for k in a["grads"])


@pytest.mark.parametrize("S,blk,keep,mlp_keep,seg", [(1024, 64, 0.75, 0.5, 256), (2048, 128, 0.5, 0.25, 4096),
                                                     (1024, 64, 1.0, 0.4, 4096)])
def test_mlp_elimination_against_oracle(J, S, blk, keep, mlp_keep, seg):
    """MLP-block elimination inside the layer: the criterion (SiLU(g) * u L1 mass per retained
    block) against the oracle's on the oracle's own activation (2e-2), the oracle's top-k on the
    GPU's criterion bit-exact, and the layer forward / backward against the oracle run with the
    GPU's attention list and MLP keep mask (3e-2 bars); MLP-eliminated rows output exactly h."""
    from oracle import layer as oly
    from oracle import mlp_blocks as omb
    from oracle.bf16 import from_bits
    case = small_case(seed=13, S=S, blk=blk)
    g = _run_mlp_layer(J, case, keep, "topk_frac", mlp_keep, seg)
    nk, kmax = g["n_kept"], g["kmax"]
    kmlp = osel.topk_count(mlp_keep, kmax)
    oi, on, om = osel.select_topk(g["mlp_scores"], kmlp)
    assert on == g["n_mlp"] == kmlp and np.array_equal(oi, g["mlp_pos"]), "MLP selection not bit-exact"
    W = oly.Weights.from_bits(case.layers[0], case.shape)
    X = from_bits(case.x)
    G = from_bits(case.g)
    keep_blocks = om[:nk].astype(bool)
    Xo, ctx = oly.sparse_layer_fwd(X, g["idx"], nk, blk, W, rnd=True, mlp_keep_blocks=keep_blocks)
    o_sc = omb.mlp_block_scores(ctx["a"], blk)
    rel = np.abs(g["mlp_scores"][:nk] - o_sc) / np.abs(o_sc)
    assert rel.max() < 2e-2, rel.max()
    dX, grads = oly.sparse_layer_bwd(ctx, G, W, seg)
    out, dx = torch_to_f64(g["out"]), torch_to_f64(g["dx"])
    gg = {k: v.cpu().numpy().astype(np.float64) for k, v in g["grads"].items()}
    check_layer_against_oracle(S, blk, g["idx"], nk, out, dx, gg, Xo, dX, grads, X, G)
    # rows the MLP eliminated carry h exactly (the oracle's h, compared at the bf16 bar, and
    # the GPU's own saved h bit for bit)
    from tests.layer_harness import split_saved
    parts = split_saved(g["saved"], kmax * blk, case.shape.hidden, case.shape.heads)
    rows = np.concatenate([np.arange(b * blk, (b + 1) * blk) for b in g["idx"][:nk]])
    drop = ~np.repeat(keep_blocks, blk)
    h_gpu = torch_to_f64(parts["h"])[: nk * blk]
    assert np.array_equal(out[rows][drop], h_gpu[drop])
    assert drop.any() and (~drop).any()


def test_pack_reports_weight_outside_fp16_range(J):
    """The backward's weight copies are fp16: a frozen weight beyond fp16's largest finite
    value (65504) is reported through the device status (JENGA_EINVAL) at pack time, and the
    status word is cleared by the read."""
    from token_sparse_long_b200 import LayerHandle
    from tests.layer_harness import bits_to_torch
    case = small_case(seed=3)
    sh, p = case.shape, case.layers[0]
    t = {k: bits_to_torch(getattr(p, k)) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "attn_norm",
                                                    "mlp_norm", "aq", "bq", "av", "bv")}
    J.jenga_check_device_status()
    LayerHandle(**t, heads=sh.heads, head_dim=sh.head_dim, rms_eps=sh.rms_eps, rope_theta=sh.rope_theta,
                lora_scale=sh.lora_scale)
    torch.cuda.synchronize()
    J.jenga_check_device_status()  # in range: no error
    t["wo"][1, 2] = 1.0e5
    LayerHandle(**t, heads=sh.heads, head_dim=sh.head_dim, rms_eps=sh.rms_eps, rope_theta=sh.rope_theta,
                lora_scale=sh.lora_scale)
    torch.cuda.synchronize()
    with pytest.raises(J._lib.JengaError) as ei:
        J.jenga_check_device_status()
    assert ei.value.status == 1  # JENGA_EINVAL
    J.jenga_check_device_status()  # cleared by the read


def test_step_is_deterministic(J):
    """Scoring (with its dynamically dealt work items), selection, forward and the segmented
    backward use fixed reduction orders: two runs on the same inputs give identical bits."""
    case = small_case(seed=5, S=1024, blk=64)
    a = run_layer_gpu(case, keep=0.5, seg=256)
    b = run_layer_gpu(case, keep=0.5, seg=256, handle=a["handle"])
    assert np.array_equal(a["scores"], b["scores"])
    assert np.array_equal(a["idx"], b["idx"]) and a["n_kept"] == b["n_kept"]
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["dx"], b["dx"])
    for k in a["grads"]:
        assert np.array_equal(a["grads"][k], b["grads"][k]), k
    # the scoring alone with many CTAs taking work items from the shared counter
    g = torch.Generator(device="cuda").manual_seed(7)
    q = (torch.randn(8192, 32 * 128, device="cuda", generator=g) * 0.3).to(torch.bfloat16)
    k = (torch.randn(8192, 32 * 128, device="cuda", generator=g) * 0.3).to(torch.bfloat16)
    s1 = J.jenga_score_blocks(q, k, 32, 128, 128)
    s2 = J.jenga_score_blocks(q, k, 32, 128, 128)
    J.jenga_check_device_status()
    assert torch.equal(s1, s2)
