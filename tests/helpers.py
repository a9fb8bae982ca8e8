"""Test-only helpers: bf16 bit conversion and small brute-force references."""
import numpy as np


def f32_to_bf16_bits(x):
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f64(h):
    u = np.asarray(h, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def ulp32(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x).astype(np.float64)
