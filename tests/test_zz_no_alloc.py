"""jenga_score_blocks_noalloc: block scoring for callers that cannot give the library
device scratch memory (hosts that own all device memory, or code that cannot afford a
cudaMalloc and the synchronisation it may cause).  The entry point runs on a fixed
array inside the library instead of a caller workspace.

Checked through the C ABI (ctypes), on two calls in a row with different inputs and
shapes, against jenga_score_blocks given an ordinary workspace: same kernels, so the
scores must agree to the tolerance the scoring tests use (here they are identical).
Collected last on purpose; it needs nothing from the other tests."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_sparse_long_b200 import _lib
    return _lib.load()


def _scores_both(lib, q, k, H, D, blk, dtype_code):
    from token_sparse_long_b200 import _lib
    S = q.shape[0]
    nb = S // blk
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = torch.empty(nb, dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.jenga_score_workspace_bytes(1, S, H, D, blk), dtype=torch.uint8, device="cuda")
    _lib.check(lib.jenga_score_blocks(_p(q), q.stride(0), _p(k), k.stride(0), 1, S, H, D, blk, 1, dtype_code, 0,
                                      _p(ref), _p(ws), ws.numel(), stream))
    got = torch.full((nb,), float("nan"), dtype=torch.float32, device="cuda")
    _lib.check(lib.jenga_score_blocks_noalloc(_p(q), q.stride(0), _p(k), k.stride(0), 1, S, H, D, blk, 1, dtype_code,
                                              0, _p(got), stream))
    torch.cuda.synchronize()
    return got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_twice(lib):
    from token_sparse_long_b200 import _lib
    g = torch.Generator(device="cuda").manual_seed(1234)
    # call 1: bf16, 3 heads x 128, S 1024, blocks of 64
    q = (torch.randn(1024, 3 * 128, device="cuda", generator=g, dtype=torch.float32) * 0.3).to(torch.bfloat16)
    k = (torch.randn(1024, 3 * 128, device="cuda", generator=g, dtype=torch.float32) * 0.3).to(torch.bfloat16)
    got, ref = _scores_both(lib, q, k, 3, 128, 64, _lib.BF16)
    assert np.all(np.abs(got - ref) <= 2e-2 * np.abs(ref))
    assert abs(got.sum() - 3 * 1024) < 2e-3 * 3 * 1024
    # and against the CPU oracle on the same bf16 values (the scoring tests' 2e-2 bar)
    from oracle import scores as osc
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64).reshape(1024, 3, 128)
    want = osc.block_scores_softmax_mass(f64(q), f64(k), 64)
    assert np.all(np.abs(got - want) <= 2e-2 * np.abs(want))
    # call 2: different data and shape (fp32, 4 heads x 64, S 512, blocks of 32); the
    # scratch still holds call 1's values and must not leak into this result
    q2 = torch.randn(512, 4 * 64, device="cuda", generator=g, dtype=torch.float32)
    k2 = torch.randn(512, 4 * 64, device="cuda", generator=g, dtype=torch.float32)
    got2, ref2 = _scores_both(lib, q2, k2, 4, 64, 32, _lib.F32)
    assert np.all(np.abs(got2 - ref2) <= 1e-3 * np.abs(ref2))
    from token_sparse_long_b200.api import jenga_check_device_status
    jenga_check_device_status()


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    from token_sparse_long_b200 import _lib
    cap = lib.jenga_score_blocks_noalloc_max_bytes()
    assert cap == 16 << 20
    null = ctypes.c_void_p(0)
    p = ctypes.c_void_p(256)
    # S = 131072 at 32 heads needs far more than 16 MiB of scratch: refused on the host,
    # nothing launched
    st = lib.jenga_score_blocks_noalloc(p, 4096, p, 4096, 1, 131072, 32, 128, 128, 1, _lib.BF16, 0, p, null)
    assert st == _lib.EWORKSPACE
    assert "fixed" in _lib.last_error()
