"""Seeded synthetic inputs shared by the CPU oracle, the GPU tests and the bench.

This module draws random numbers and converts them between number formats.  It
holds none of the method's arithmetic (no patchify, no rotation, no attention):
both sides of every parity check start from the same arrays built here, and
each side then computes on its own.

Recipe (the same for every workload):

* generator: NumPy ``PCG64`` seeded with ``SeedSequence([seed, tensor_id])``;
  ``tensor_id`` is 0/1/2 for Q/K/V and 3 for the latent clip; the default seed
  is 0;
* Q, K, V: standard normal draws in float32, rounded to bfloat16 with
  round-to-nearest-even, laid out ``[B, L, heads, head_dim]`` (token-major,
  the unpermuted output of a ``[B, L, heads*head_dim]`` projection);
* latent clip: standard normal draws in float32, laid out ``[N, C, T, H, W]``.

Large tensors are drawn in fixed-size blocks from one generator, which yields
the same stream as a single draw, so the values do not depend on memory limits.
"""
from __future__ import annotations

import numpy as np

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "latent": 3, "w_embed": 4, "w_qkv": 5}

_BLOCK = 1 << 24  # elements per draw


def rng_for(seed: int, tensor_id: int) -> np.random.Generator:
    """The generator every consumer uses for tensor ``tensor_id`` of ``seed``."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id])))


def normal_f32(shape, seed: int, tensor_id: int, scale: float = 1.0) -> np.ndarray:
    """Standard-normal float32 array of ``shape`` (times ``scale``), drawn blockwise."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    g = rng_for(seed, tensor_id)
    for s in range(0, n, _BLOCK):
        e = min(n, s + _BLOCK)
        g.standard_normal(e - s, dtype=np.float32, out=out[s:e])
    if scale != 1.0:
        out *= np.float32(scale)
    return out.reshape(shape)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bit patterns.

    Inputs are finite.  Works in place-sized blocks so multi-GB arrays stay cheap.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.reshape(-1).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    for s in range(0, u.size, _BLOCK):
        blk = u[s:s + _BLOCK]
        r = blk + (np.uint32(0x7FFF) + ((blk >> np.uint32(16)) & np.uint32(1)))
        out[s:s + _BLOCK] = (r >> np.uint32(16)).astype(np.uint16)
    return out.reshape(x.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 values of bfloat16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 values of bfloat16 bit patterns."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even) without a float32 detour."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    # bfloat16 keeps 8 significant bits; round the float64 significand directly.
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                  # 8 significant bits before the point
    r = np.rint(scaled)                      # round half to even
    y = np.ldexp(r, e - 8).astype(np.float32)  # exact: r has <= 9 bits, 2**8 case renormalises
    return f32_to_bf16_bits(y)


def qkv_bf16(B: int, L: int, heads: int, head_dim: int, seed: int = 0, q_scale: float = 1.0):
    """Seeded bf16 Q, K, V bit patterns, each ``[B, L, heads, head_dim]`` uint16.

    ``q_scale`` multiplies the float32 draws of Q before rounding; values above 1
    sharpen the softmax (a stress variant, not a workload of the pages).
    """
    shape = (B, L, heads, head_dim)
    q = f32_to_bf16_bits(normal_f32(shape, seed, TENSOR_ID["q"], q_scale))
    k = f32_to_bf16_bits(normal_f32(shape, seed, TENSOR_ID["k"]))
    v = f32_to_bf16_bits(normal_f32(shape, seed, TENSOR_ID["v"]))
    return q, k, v


def latent_f32(N: int, C: int, T: int, H: int, W: int, seed: int = 0) -> np.ndarray:
    """Seeded float32 latent clip ``[N, C, T, H, W]``."""
    return normal_f32((N, C, T, H, W), seed, TENSOR_ID["latent"])


def sample_rows(L: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted query-row indices checked at full size: ``count`` distinct rows of ``L``."""
    g = np.random.default_rng(seed)
    if count >= L:
        return np.arange(L, dtype=np.int64)
    return np.sort(g.choice(L, count, replace=False)).astype(np.int64)


def tiny_weights(in_features: int, width: int, seed: int = 0):
    """Random projection weights for the tiny clip: embed ``in_features -> width`` and
    ``width -> 3*width`` (Q, K, V), drawn N(0, 1/fan_in) in float64."""
    we = rng_for(seed, TENSOR_ID["w_embed"]).standard_normal((in_features, width)) / np.sqrt(in_features)
    wq = rng_for(seed, TENSOR_ID["w_qkv"]).standard_normal((width, 3 * width)) / np.sqrt(width)
    return we, wq
