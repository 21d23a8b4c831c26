"""bfloat16 <-> float32 bit conversions (round to nearest even), NumPy only."""

import numpy as np


def f32_to_bf16_bits(x):
    """float32 array -> uint16 bf16 bit patterns, round-to-nearest-even.

    NaN is mapped to the canonical quiet NaN 0x7FC0.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounded = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b):
    """uint16 bf16 bit patterns -> float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(x):
    """float array -> float32 array holding the nearest bf16 values."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))
