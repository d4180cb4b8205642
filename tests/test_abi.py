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
