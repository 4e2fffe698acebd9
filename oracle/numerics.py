"""Rounding helpers for the oracle (fp64 in, exact decisions out).

Pinned in tests/test_oracle_numerics.py against torch's own fp32 -> bf16 cast
(an independent round-to-nearest-even implementation) and hand-made ties.
"""
import numpy as np


def round_to_bf16(x):
    """Round float64 values to the nearest bfloat16 value, ties to even, in ONE
    rounding (no detour through fp32, which could round twice).

    bfloat16 keeps 8 significant bits and the fp32 exponent range, so the
    spacing around x = m * 2**e (0.5 <= |m| < 1) is 2**(e - 8) for normal
    values, floored at the subnormal spacing 2**-133.  Values beyond the
    bf16 range are not expected (the caller's data is bounded) and raise.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    _, e = np.frexp(x[nz])
    sp = np.maximum(e - 8, -133)
    q = np.ldexp(x[nz], -sp)          # exact: scaling by a power of two
    out[nz] = np.ldexp(np.rint(q), sp)  # np.rint rounds half to even
    if np.any(np.abs(out) > 3.3895313892515355e38):
        raise OverflowError("value outside the bf16 range")
    return out


def round_to_f32(x):
    """Round float64 values to the nearest float32 (numpy's cast is RNE)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(x, kv_dtype):
    if kv_dtype == "bf16":
        return round_to_bf16(x)
    if kv_dtype == "f32":
        return round_to_f32(x)
    raise ValueError(kv_dtype)
