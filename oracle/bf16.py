"""bfloat16 storage format for the oracle (test infrastructure; see the package docstring).

bfloat16 keeps the upper 16 bits of an IEEE binary32 value (1 sign, 8 exponent, 7 fraction bits).
Rounding binary32 -> bfloat16 here is round-to-nearest, ties-to-even, written from that definition:
keep the upper half; round up by one unit in the last kept place when the discarded lower half is
more than half a unit, or exactly half a unit and the kept part is odd. Activations and weights are
bf16 in the pages' workloads ("张量并行与序列并行", §预备：记号与集合通信的代价: activations and weights
default to bf16, two bytes per element).
"""
from __future__ import annotations

import numpy as np


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round binary32 values to bfloat16, returned as uint16 storage bits."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    kept = u >> np.uint64(16)
    dropped = u & np.uint64(0xFFFF)
    half = np.uint64(0x8000)
    odd = (kept & np.uint64(1)) == np.uint64(1)
    up = (dropped > half) | ((dropped == half) & odd)
    out = kept + up.astype(np.uint64)
    # NaN stays NaN: exponent all ones with a non-zero fraction -> a quiet NaN of the same sign.
    exp_all_ones = (u & np.uint64(0x7F800000)) == np.uint64(0x7F800000)
    frac_nonzero = (u & np.uint64(0x007FFFFF)) != np.uint64(0)
    nan = exp_all_ones & frac_nonzero
    out = np.where(nan, kept | np.uint64(0x0040), out)
    return out.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact widening of bfloat16 storage bits to binary32 (the bits become the upper half)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bfloat16 storage bits to float64."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def round_to_bf16_f64(x) -> np.ndarray:
    """Value of a real array after the binary32 -> bfloat16 rounding (the fp64 input is first
    rounded to binary32, as a GPU holding it in fp32 registers would)."""
    return bf16_bits_to_f64(f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32)))
