"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and rounds them to the storage type; it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can consume its output without
sharing any of the method's code.

Recipe (one per call):
  rng = numpy.random.default_rng(seed)
  q = rng.standard_normal(shape, float32); k = ...; v = ...      (drawn in that order)
  bf16 storage: each float32 value rounded to bfloat16, round-to-nearest-even.
  fp32 storage: the float32 draw as is.
The oracle upcasts the *stored* values to float64, so a parity check measures kernel error only.
"""

from __future__ import annotations

import numpy as np

BF16 = "bf16"
F32 = "f32"


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    nan = np.isnan(x)
    # add 0x7FFF plus the lowest kept bit, then truncate: round-half-to-even on the dropped 16 bits
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    r = r.astype(np.uint16)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def draw_qkv(shape, seed: int, dtype: str = BF16, scale: float = 1.0):
    """Draw q, k, v ~ N(0, scale^2) in float32 with one seeded generator, in the order q, k, v.

    Returns the three arrays in *storage* form: uint16 bfloat16 bit patterns for ``bf16``,
    float32 for ``f32``.
    """
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        x = rng.standard_normal(shape, dtype=np.float32)
        if scale != 1.0:
            x = (x * np.float32(scale)).astype(np.float32)
        out.append(f32_to_bf16_bits(x) if dtype == BF16 else x)
    return tuple(out)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage form -> float64 values exactly as the kernels see them."""
    return bf16_bits_to_f64(x) if dtype == BF16 else np.asarray(x, dtype=np.float32).astype(np.float64)


def draw_conv(shape, seed: int, dtype: str = BF16):
    """Inputs of the temporal convolution: x ~ N(0, 1) of `shape` [B, T, S, C] in storage form, then
    fp32 weights w [C, 3] ~ N(0, 1/4) and bias [C] ~ N(0, 1/4) (synthetic: the pages give none), all
    from one seeded generator in that order."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape, dtype=np.float32)
    C = shape[-1]
    w = (rng.standard_normal((C, 3), dtype=np.float32) * np.float32(0.5)).astype(np.float32)
    b = (rng.standard_normal((C,), dtype=np.float32) * np.float32(0.5)).astype(np.float32)
    return (f32_to_bf16_bits(x) if dtype == BF16 else x), w, b


def draw_proj(x_shape, n_out: int, seed: int):
    """Inputs of a projection: x ~ N(0, 1) of `x_shape` (last dim = input features C), then the
    weight [n_out, C] ~ N(0, 1/C) (synthetic: the pages give no trained weights), from one seeded
    generator in that order; both as bf16 bit patterns (round to nearest even)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(x_shape, dtype=np.float32)
    C = x_shape[-1]
    w = (rng.standard_normal((n_out, C), dtype=np.float32) * np.float32(1.0 / np.sqrt(C))).astype(np.float32)
    return f32_to_bf16_bits(x), f32_to_bf16_bits(w)
