"""Seeded synthetic inputs shared by the oracle-side tests, the GPU parity tests,
the benchmark and the smoke check.

This module holds no arithmetic of the attention or cache method. It only turns a
tuple of integers into reproducible bf16 tensors so that the CPU oracle and the
CUDA path are fed the very same bytes.

Definition (so that any other implementation can regenerate the same bytes):

* Seed:  ``seed = mix(base_seed, config_id, layer, chunk, kind)`` where ``mix``
  folds each value into a SplitMix64 state: ``s = splitmix64(s ^ v)``.
* Stream: element ``i`` of a tensor draws two 64-bit words
  ``a = splitmix64(seed + (2i+1)*G)`` and ``b = splitmix64(seed + (2i+2)*G)``
  with ``G = 0x9E3779B97F4A7C15`` (mod 2**64).
* Uniforms: ``u1 = ((a >> 11) + 1) / 2**53`` in (0, 1], ``u2 = (b >> 11) / 2**53``.
* Normal:  ``z = sqrt(-2 ln u1) * cos(2 pi u2)`` (Box-Muller, fp64).
* Scale:   ``z * scale`` in fp64.
* Rounding: fp64 -> fp32 (IEEE round-to-nearest-even), then fp32 -> bf16
  (round-to-nearest-even on the upper 16 bits).

Tensors are returned as ``numpy.uint16`` arrays of bf16 bit patterns in the
token-major layout ``[tokens][heads][head_dim]`` that a QKV projection emits.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 20261202
GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor kinds
KIND_Q, KIND_K, KIND_V, KIND_KNEW, KIND_VNEW = 1, 2, 3, 4, 5


def _splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser applied elementwise to a uint64 array (wraps mod 2**64)."""
    with np.errstate(over="ignore"):
        z = x + GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def mix_seed(*values: int, base_seed: int = BASE_SEED) -> int:
    s = np.array([base_seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    for v in values:
        s = _splitmix64(s ^ np.uint64(v & 0xFFFFFFFFFFFFFFFF))
    return int(s[0])


def normal_f64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """n standard normals (fp64) from the counter stream of `seed`, starting at element `offset`."""
    i = np.arange(offset, offset + n, dtype=np.uint64)
    s = np.uint64(seed)
    with np.errstate(over="ignore"):
        a = _splitmix64(s + (np.uint64(2) * i + np.uint64(1)) * GOLDEN)
        b = _splitmix64(s + (np.uint64(2) * i + np.uint64(2)) * GOLDEN)
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) / 9007199254740992.0
    u2 = (b >> np.uint64(11)).astype(np.float64) / 9007199254740992.0
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (inputs are finite)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_normal(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    z = normal_f64(seed, n) * scale
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(shape)


def chunk_tensor(kind: int, config_id: int, layer: int, chunk: int, tokens: int, heads: int,
                 head_dim: int, scale: float = 1.0, base_seed: int = BASE_SEED) -> np.ndarray:
    """One [tokens][heads][head_dim] bf16 tensor (uint16 bits) for (config, layer, chunk, kind)."""
    seed = mix_seed(config_id, layer, chunk, kind, base_seed=base_seed)
    return bf16_normal(seed, (tokens, heads, head_dim), scale)


def chunk_qkv(config_id: int, layer: int, chunk: int, tokens: int, heads: int, head_dim: int,
              scale: float = 1.0, base_seed: int = BASE_SEED):
    """(q, k_cur, v_cur) of one chunk as uint16 bf16 bit arrays."""
    return tuple(chunk_tensor(k, config_id, layer, chunk, tokens, heads, head_dim, scale, base_seed)
                 for k in (KIND_Q, KIND_K, KIND_V))


def recache_kv(config_id: int, layer: int, event: int, tokens: int, heads: int, head_dim: int,
               scale: float = 1.0, base_seed: int = BASE_SEED):
    """(k_new, v_new) for a recache event: [tokens][heads][head_dim] bf16 bits each."""
    return tuple(chunk_tensor(k, config_id, layer, 100000 + event, tokens, heads, head_dim, scale, base_seed)
                 for k in (KIND_KNEW, KIND_VNEW))
