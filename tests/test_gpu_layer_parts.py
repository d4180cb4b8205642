"""Per-step GPU parity of the layer forward: each saved intermediate (gathered x,
q/k/v after RoPE, LoRA t, attention output and its log-sum-exp, h, the MLP pre-activations)
against the oracle's value of the same step, so that a fault is pinned to the step that
makes it."""
import numpy as np
import pytest
import torch

from oracle import layer as oly
from oracle.bf16 import from_bits
from tests.layer_harness import (bits_to_torch, deinterleave_gu, layer_handle, rel_delta_ulp, rel_max, rel_max_ulp,
                                 small_case, split_saved, torch_to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def J():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import token_sparse_long_b200 as J
    J._lib.load()
    return J


@pytest.mark.parametrize("keep_blocks", [[0, 1, 2, 3, 4, 5, 6, 7], [1, 3, 4, 6], [0, 2, 5]])
def test_forward_intermediates(J, keep_blocks):
    case = small_case(seed=11, S=512, blk=64, lora_b_std=0.02)
    sh = case.shape
    L = layer_handle(case.layers[0], sh)
    nb = case.S // case.blk
    idx_np = np.full(nb, -1, np.int32)
    idx_np[: len(keep_blocks)] = keep_blocks
    idx = torch.from_numpy(idx_np).cuda()
    nk = torch.tensor([len(keep_blocks)], dtype=torch.int32, device="cuda")
    x = bits_to_torch(case.x)
    kmax = len(keep_blocks)
    saved = J.jenga_sparse_layer_fwd(L, x, idx, nk, case.blk, kmax)
    J.jenga_check_device_status()
    nc = kmax * case.blk
    parts = split_saved(saved, nc, sh.hidden, sh.heads, F=sh.ffn)
    W = oly.Weights.from_bits(case.layers[0], sh)
    rows = (np.asarray(keep_blocks)[:, None] * case.blk + np.arange(case.blk)[None]).reshape(-1)
    X = from_bits(case.x)
    out, ctx = oly.layer_fwd(X[rows], rows, W, rnd=True)
    HD = sh.heads * sh.head_dim
    errs = {}
    assert np.array_equal(torch_to_f64(parts["xr"]), X[rows])
    errs["rstd1"] = rel_max(parts["rstd1"].cpu().numpy(), ctx["rstd1"])
    errs["t"] = rel_max(torch_to_f64(parts["t"])[:, :16], ctx["tq"])
    qkv = torch_to_f64(parts["qkv"])
    # bf16-stored tensors: one ulp of the stored value forgiven (see test_gpu_layer)
    errs["q"] = rel_max_ulp(qkv[:, :HD], ctx["q"].reshape(nc, HD))
    errs["k"] = rel_max_ulp(qkv[:, HD:2 * HD], ctx["k"].reshape(nc, HD))
    errs["v"] = rel_max_ulp(qkv[:, 2 * HD:], ctx["v"].reshape(nc, HD))
    errs["lse"] = rel_max(-parts["lse"].cpu().numpy() * np.log(2.0), ctx["lse"])  # saved negated, log2 units
    errs["o"] = rel_max_ulp(torch_to_f64(parts["o"]), ctx["o"].reshape(nc, HD))
    errs["h"] = rel_delta_ulp(torch_to_f64(parts["h"]), ctx["h"], X[rows])
    errs["out"] = rel_delta_ulp(torch_to_f64(x)[rows], out, X[rows])
    # the saved (gate, up) pre-activations (fp16); the oracle forms them from its own hn,
    # which differs from the GPU's by the bf16 roundings of h, so they take the common bar
    g16, u16 = deinterleave_gu(parts["gu"].cpu().double().numpy(), sh.ffn)
    errs["g"] = rel_max(g16, ctx["gt"])
    errs["u"] = rel_max(u16, ctx["ut"])
    assert (parts["mlp_mask"][:kmax].cpu().numpy() == 1).all()
    print(errs)
    for k, v in errs.items():
        assert v < 3e-2, (k, errs)
