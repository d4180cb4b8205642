"""Host-side checks of the C ABI (no GPU): the library loads, exports every symbol that
include/jenga.h declares, sizes its workspaces, and rejects bad arguments before any
launch."""
import ctypes
import os
import re

import pytest

from token_sparse_long_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    with open(os.path.join(ROOT, "include", "jenga.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"JENGA_API\s+[\w\s\*]+?\b(jenga_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from token_sparse_long_b200 import build
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    syms = header_symbols()
    assert len(syms) >= 24
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(_lib.exported_symbols())


def test_status_strings_and_version(lib):
    assert lib.jenga_status_string(0) == b"ok"
    assert lib.jenga_status_string(5) == b"workspace too small"
    assert b"sm_100a" in lib.jenga_version()


def test_workspace_sizes(lib):
    assert lib.jenga_score_workspace_bytes(1, 32768, 32, 128, 128) >= 2 * 32 * 32768 * 4
    assert lib.jenga_select_workspace_bytes(1, 256) == 0
    assert lib.jenga_select_workspace_bytes(1, 1 << 26) > 0
    w = _lib.LayerWeights(4096, 32, 128, 11008, 1e-5, 10000.0, *([1] * 9))
    lo = _lib.Lora(16, 1.0, 1, 1, 1, 1)
    saved = lib.jenga_layer_saved_bytes(ctypes.byref(w), 1, 128, 205)
    n = 205 * 128
    assert saved >= n * 4096 * 2 * 6  # xr, q, k, v, o, h in bf16
    assert lib.jenga_layer_pack_bytes(ctypes.byref(w), ctypes.byref(lo)) > 4096 * 4096 * 2 * 12
    assert lib.jenga_layer_bwd_workspace_bytes(ctypes.byref(w), 1, 128, 205, 4096) > 2 * n * 4096 * 4


def test_bad_arguments_rejected_on_host(lib):
    null = ctypes.c_void_p(0)
    assert lib.jenga_select(null, 1, 16, 0, 0.0, null, null, null, null, 0, null) == _lib.EINVAL
    assert lib.jenga_gather(null, 256, 1, 512, 256, 32, null, null, 0, null, 256, 16, null) == _lib.EINVAL
    assert "null" in _lib.last_error()
    p = ctypes.c_void_p(256)
    # S not a multiple of blk
    assert lib.jenga_score_blocks(p, 128, p, 128, 1, 100, 1, 128, 64, 1, 1, 0, p, p, 1 << 20, null) == _lib.EINVAL
    # workspace too small
    assert lib.jenga_score_blocks(p, 128, p, 128, 1, 128, 1, 128, 64, 1, 1, 0, p, p, 16, null) == _lib.EWORKSPACE
    # bad select mode
    assert lib.jenga_select(p, 1, 16, 9, 0.0, p, p, p, null, 0, null) == _lib.EINVAL
    # head_dim other than 128 is rejected by the layer
    w = _lib.LayerWeights(4096, 32, 64, 11008, 1e-5, 10000.0, *([1] * 9))
    lo = _lib.Lora(16, 1.0, 1, 1, 1, 1)
    assert lib.jenga_layer_pack(ctypes.byref(w), ctypes.byref(lo), p, 1 << 30, null) == _lib.EINVAL
    # top-k over very many blocks is not built
    assert lib.jenga_select(p, 1, 1 << 20, 1, 0.5, p, p, null, p, 1 << 20, null) == _lib.EUNSUPPORTED


def test_package_imports_without_gpu():
    import token_sparse_long_b200 as J
    assert callable(J.jenga_score_blocks)
    with pytest.raises(Exception):
        import torch
        J.jenga_select(torch.zeros(4), "mean_ge")   # CPU tensor: refused, no CPU path


def test_lm_loss_and_predictor_pair_host_checks(lib):
    null = ctypes.c_void_p(0)
    p = ctypes.c_void_p(256)
    # segmented LM loss: the workspace holds one segment's logits (fp32) and gradient rows
    # (bf16) plus the transposed embedding, so it grows with the segment, not with S
    seg = lib.jenga_lm_loss_workspace_bytes(32768, 4096, 32000, 4096)
    full = lib.jenga_lm_loss_workspace_bytes(32768, 4096, 32000, 32768)
    assert seg >= 4096 * 32000 * 6 + 4096 * 32000 * 2 and full >= 32768 * 32000 * 6
    assert full > 5 * seg
    assert lib.jenga_lm_loss_workspace_bytes(100, 64, 64, 4096) == lib.jenga_lm_loss_workspace_bytes(100, 64, 64, 100)
    # V not a multiple of 64; null pointers; workspace too small
    assert lib.jenga_lm_loss_segmented(p, p, p, 128, 64, 1000, 64, p, p, p, 1 << 30, null) == _lib.EINVAL
    assert lib.jenga_lm_loss_segmented(null, p, p, 128, 64, 1024, 64, p, p, p, 1 << 30, null) == _lib.EINVAL
    assert lib.jenga_lm_loss_segmented(p, p, p, 128, 64, 1024, 64, p, p, p, 16, null) == _lib.EWORKSPACE
    # Q/K predictor pair: output width above 64 and misaligned inputs are refused
    assert lib.jenga_predict_qk_workspace_bytes(1, 32768, 5120, 128, 16) >= 256 * 5120 * 4 + 2 * 256 * 16 * 4
    assert lib.jenga_predict_blocks_qk(p, 1, 1024, 512, 128, p, p, p, p, p, p, 128, 64, 65, 1, p, p, 1 << 30,
                                       null) == _lib.EINVAL
    q = ctypes.c_void_p(264)
    assert lib.jenga_predict_blocks_qk(q, 1, 1024, 512, 128, p, p, p, p, p, p, 128, 64, 16, 1, p, p, 1 << 30,
                                       null) == _lib.EINVAL
    # MLP-block criterion: F must be a multiple of 8
    assert lib.jenga_mlp_block_scores(p, 1004, 1004, 64, null, 4, p, null) == _lib.EINVAL
    assert lib.jenga_mlp_block_scores(p, 1008, 1008, 64, null, 0, p, null) == 0  # nothing to do


def test_product_path_never_touches_the_oracle():
    # the oracle is test infrastructure: the package (binding, build script, kernels) must
    # neither import it nor reference its files
    pkg = os.path.join(ROOT, "token_sparse_long_b200")
    hits = []
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    for n, line in enumerate(fh, 1):
                        if re.search(r"\b(import\s+oracle|from\s+oracle|oracle/)", line):
                            hits.append(f"{f}:{n}")
    assert not hits, hits
