"""Seeded synthetic inputs shared by the CUDA path, its tests and the benchmark.

This module only draws random numbers and converts them to bf16 bit patterns.
It holds none of the attention arithmetic, so both the fp64 oracle and the GPU
path can be fed the very same bits without sharing any code that computes the
method.

Recipe: Q, K and V are drawn i.i.d. N(0, 1) in float32 from
``numpy.random.default_rng(seed)`` (seeds 0, 1, 2 for Q, K, V unless a caller
says otherwise), then rounded to bf16 with round-to-nearest-even on the bit
pattern.  The oracle upcasts the same bf16 values to float64 exactly.
"""
from __future__ import annotations

import numpy as np

Q_SEED, K_SEED, V_SEED = 0, 1, 2


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + rounding) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def normal_bf16_bits(shape, seed: int) -> np.ndarray:
    """N(0,1) float32 draws from ``default_rng(seed)``, rounded to bf16 bits."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def qkv_bits(heads: int, kv_heads: int, n: int, d: int,
             seeds=(Q_SEED, K_SEED, V_SEED)):
    """Q ``[heads, n, d]`` and K, V ``[kv_heads, n, d]`` as bf16 bit arrays.

    ``heads`` and ``kv_heads`` are the folded batch*head counts: a batch of
    ``b`` sequences with ``H`` query heads is ``heads = b*H`` contiguous slices.
    """
    q = normal_bf16_bits((heads, n, d), seeds[0])
    k = normal_bf16_bits((kv_heads, n, d), seeds[1])
    v = normal_bf16_bits((kv_heads, n, d), seeds[2])
    return q, k, v
