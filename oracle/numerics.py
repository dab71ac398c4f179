"""Storage rounding used by the oracle to mirror the GPU path's stored intermediates.

bf16 is the upper 16 bits of an IEEE-754 binary32.  Rounding a binary32 to bf16
with round-to-nearest, ties-to-even, adds 0x7FFF plus the lowest kept bit to
the 32-bit pattern and truncates the low 16 bits; NaN inputs stay NaN.  The
oracle uses this where the GPU stores a tensor as bf16, and a plain cast to
float32 where it stores fp32.
"""
import numpy as np


def round_bf16(x):
    """Round to the nearest bf16 value (ties to even); returns float32 values."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(f)
    if nan.any():
        out[nan] = np.float32("nan")
    return out


def bf16_bits_to_f32(bits):
    """Widen raw bf16 bit patterns (uint16) to float32 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits(x):
    """bf16 bit patterns of the RNE rounding of x."""
    return (round_bf16(x).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def round_storage(x, storage):
    """Round x to the storage type of the path: 'bf16' or 'fp32'."""
    if storage == "bf16":
        return round_bf16(x).astype(np.float64)
    if storage == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage type {storage!r}")


def round_f32(x):
    """Round to binary32 and return as float64 (for fp32-stored intermediates)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
