"""float64 -> bf16 rounding for the oracle's storage-rounding points.

The Jenga notes (experimental setup, "A4") state that all measurements use mixed
bf16/fp32 precision.  The oracle therefore rounds to bf16 at the tensor boundaries
where the layer stores bf16 (listed in ``oracle.layer``), and computes in float64
everywhere else.  Rounding is round-to-nearest-even applied directly to the float64
value (one rounding step).  Exact for results in the bf16 normal range and zero.
"""
import numpy as np

_DROP = 45                      # float64 has 52 fraction bits, bf16 keeps 7
_HALF = np.uint64((1 << (_DROP - 1)) - 1)
_MASK = np.uint64(~((1 << _DROP) - 1) & 0xFFFFFFFFFFFFFFFF)


def round_bf16(x):
    """Round float64 values to the nearest bf16 value (ties to even); returns float64."""
    a = np.array(x, dtype=np.float64, copy=True)
    b = a.view(np.uint64)
    lsb = (b >> np.uint64(_DROP)) & np.uint64(1)
    finite = np.isfinite(a)
    r = ((b + _HALF + lsb) & _MASK)
    out = np.where(finite, r, b).view(np.float64)
    return out.reshape(np.shape(x)) if np.ndim(x) else float(out)


def from_bits(u16):
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_f32(x):
    """Round float64 values to fp32 (one rounding); returns float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
