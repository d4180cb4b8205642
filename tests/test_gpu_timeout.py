"""The device-side wait bound (every pipeline wait in the library gives up after a time
budget, records JENGA_ETIMEOUT in the device error word and returns).

The test makes one wait run out on purpose through the jenga_test_wait_timeout hook: one
warp waits on a barrier that nothing completes, with no copy or tensor-core operation in
flight, under a 1 ms budget.  The host must then read JENGA_ETIMEOUT with the hook's site
and detail, the word must be cleared by that read, and the context must stay usable."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from token_sparse_long_b200 import _lib
    return _lib.load()


def test_wait_budget_expiry_is_reported_and_context_survives(lib):
    from token_sparse_long_b200 import _lib
    import token_sparse_long_b200 as J
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    det = (ctypes.c_uint32 * 2)()
    assert lib.jenga_check_device_status(stream, det) == 0
    _lib.check(lib.jenga_set_wait_budget_ns(1_000_000))
    try:
        _lib.check(lib.jenga_test_wait_timeout(stream))
        st = lib.jenga_check_device_status(stream, det)
        assert st == _lib.ETIMEOUT, _lib.status_name(st)
        assert (det[0], det[1]) == (8, 0xC0FFEE)
        assert "timed out" in _lib.last_error()
        assert lib.jenga_check_device_status(stream, det) == 0  # read-and-clear
    finally:
        _lib.check(lib.jenga_set_wait_budget_ns(2_000_000_000))
    # the context is still usable: a normal library call runs and reports no fault
    x = torch.arange(4 * 64, dtype=torch.float32, device="cuda").reshape(4, 64)
    idx = torch.tensor([1, 3], dtype=torch.int32, device="cuda")
    nk = torch.tensor([2], dtype=torch.int32, device="cuda")
    out = J.jenga_gather(x, idx, nk, 1, 2)
    J.jenga_check_device_status()
    assert torch.equal(out, x[[1, 3]])
