"""bfloat16 helpers for the oracle (test infrastructure only).

bfloat16 is the upper half of an IEEE binary32. Rounding from float32 is
round-to-nearest, ties-to-even on the discarded 16 bits. The inputs here
are finite; NaN handling is not needed by the oracle.
"""

import numpy as np


def round_f32_to_bf16_bits(x):
    """Round float32 values to bfloat16 (RNE); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b):
    """Widen uint16 bfloat16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16(x):
    """float32 -> nearest bfloat16 value, returned as float32 (exactly representable)."""
    return bf16_bits_to_f32(round_f32_to_bf16_bits(x))
