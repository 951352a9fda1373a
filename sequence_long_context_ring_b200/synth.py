"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds no attention or convolution arithmetic: it only draws i.i.d. normal values from a
fixed seed and rounds them to bfloat16.  Both sides of every parity check read the same
host arrays produced here.

Generator: numpy ``Generator(PCG64)`` seeded with ``default_rng([cfg_id, tensor_id])``;
tensor ids are Q=0, K=1, V=2, dO=3, and for the convolution x=4, h=5.  Values are float32 ``standard_normal`` (drawn in
blocks of at most 64 Mi elements to bound host memory), multiplied by ``scale`` in
float32, then rounded to bf16 by round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import numpy as np

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "do": 3, "x": 4, "h": 5}
_BLOCK = 1 << 26  # elements per float32 draw (256 MiB)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(cfg_id: int, tensor_id: int, shape, scale: float = 1.0) -> np.ndarray:
    """i.i.d. N(0, scale^2) values rounded to bf16, as a uint16 array of ``shape``."""
    n = int(np.prod(shape))
    rng = np.random.default_rng([int(cfg_id), int(tensor_id)])
    out = np.empty(n, dtype=np.uint16)
    s = np.float32(scale)
    for lo in range(0, n, _BLOCK):
        hi = min(n, lo + _BLOCK)
        blk = rng.standard_normal(hi - lo, dtype=np.float32)
        if s != np.float32(1.0):
            blk *= s
        out[lo:hi] = f32_to_bf16_bits(blk)
    return out.reshape(shape)


def tagged_u16(shape) -> np.ndarray:
    """Distinct 16-bit tags (index mod 65521, a prime) for layout tests: bit patterns only."""
    n = int(np.prod(shape))
    return (np.arange(n, dtype=np.int64) % 65521).astype(np.uint16).reshape(shape)
