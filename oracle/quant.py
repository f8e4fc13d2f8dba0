"""O3 - quantisers for a low-precision KV cache, bit-exact, in IEEE fp32.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The LongLive-2.0 explainer (wmrh.cn, sec. 15.2) stores the history KV cache in
NVFP4 / FP4 to save memory, and sec. 15.3 dequantises it in parallel when it is
used. The pages give no rounding or scaling details; the readings taken here:

FP8 (E4M3, per (token, head) row of D values, one fp32 scale per row)
  1. amax  = max |x|                        (exact)
  2. scale = the smallest power of two s with amax <= 448 * s, but at least
     2^-124;  scale = 1 if amax == 0.
     A power-of-two scale keeps every step exact: x / scale is an exact fp32
     value (no rounding before the E4M3 rounding; only quotients far below
     the smallest E4M3 step can underflow, and they encode as zero either
     way), and every dequantised
     value, E4M3 value * scale, has at most 4 significant bits and lies at or
     above 2^-133, so it is exact in bf16 (the floor 2^-124 guarantees the
     latter and keeps 1 / scale finite). The row maximum lands in (224, 448],
     so E4M3's 3-bit relative precision is kept for every value but the
     lowest binade of the row's range.
  3. inv   = 1 / scale    (exact, a power of two)
  4. code  = E4M3(x * inv)   fp32 product (exact, as above), then round-to-nearest-even
             into E4M3 with saturation to +-448 (no NaN is ever produced)
  dequantised value = E4M3 value * scale (exact in bf16)

NVFP4 (E2M1 values, 16-element blocks along D, E4M3 block scale)
  1. amax = max |x| over the block
  2. sb   = E4M3(amax / 6)  (fp32 division, round-to-nearest-even, saturating)
  3. sb == 0  ->  every code of the block is +0
     else code = E2M1(x / sb)  (fp32 division; round-to-nearest-even into the
     grid {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating at +-6, sign kept for -0)
  4. two codes per byte, element 2i in the low nibble
  dequantised value = E2M1 value * sb

Formats (OCP 8-bit floating point / MX specifications):
  E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
        subnormal (m/8 * 2^-6); S.1111.111 is NaN; largest finite 448.
  E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is
        subnormal (m/2); largest 6.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
FP8_MIN_SCALE_LOG2 = -124      # scale floor: dequantised values stay exact in bf16


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code from the bit definition (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e2m1_value(code: int) -> float:
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * (m / 2.0)
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
_E4M3_POS = {float(E4M3_TABLE[c]): c for c in range(0x7F)}   # +values, codes 0..126
_E2M1_POS = {float(E2M1_TABLE[c]): c for c in range(8)}


def _round_to_grid(a: np.ndarray, min_exp: int, mant_bits: int) -> np.ndarray:
    """Round |y| (fp64 copy of an fp32 value) to the nearest value with
    `mant_bits` fraction bits, ties to even, subnormals below 2^min_exp.
    Scaling by a power of two is exact, and numpy's rint rounds half to even."""
    _, ex = np.frexp(np.where(a > 0, a, 1.0))     # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex.astype(np.float64) - 1.0, min_exp)
    quantum = np.exp2(e - mant_bits)
    return np.rint(a / quantum) * quantum


def e4m3_encode(y) -> np.ndarray:
    """fp32 values -> E4M3 codes (uint8), round-to-nearest-even, saturating."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    a = np.abs(y)
    r = _round_to_grid(a, -6, 3)
    r = np.minimum(r, E4M3_MAX)
    mags = np.vectorize(lambda v: _E4M3_POS[float(v)], otypes=[np.uint8])(r) if r.size else r.astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << np.uint8(7)
    return (mags | sign).astype(np.uint8)


def e2m1_encode(y) -> np.ndarray:
    """fp32 values -> E2M1 codes (uint8 holding 4 bits), round-to-nearest-even, saturating."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    a = np.abs(y)
    r = _round_to_grid(a, 0, 1)
    r = np.minimum(r, E2M1_MAX)
    mags = np.vectorize(lambda v: _E2M1_POS[float(v)], otypes=[np.uint8])(r) if r.size else r.astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << np.uint8(3)
    return (mags | sign).astype(np.uint8)


def fp8_quantize_rows(x_bits: np.ndarray):
    """bf16 rows [..., D] (uint16 bits) -> (codes uint8 [..., D], scales float32 [...])."""
    x = (np.asarray(x_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    amax = np.max(np.abs(x), axis=-1).astype(np.float64)               # exact
    # smallest k with amax <= 448 * 2^k: amax / 448 and its log2 are exact in
    # fp64 whenever the result is an integer (amax = 7 * 2^j for bf16 inputs),
    # and otherwise nowhere near one
    with np.errstate(divide="ignore"):
        k = np.ceil(np.log2(amax / E4M3_MAX))
    k = np.where(amax == 0, 0.0, np.maximum(k, FP8_MIN_SCALE_LOG2))
    scale = np.exp2(k).astype(np.float32)                              # powers of two: exact
    inv = np.exp2(-k).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)                        # fp32 products (exact)
    return e4m3_encode(y), scale


def fp8_dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[codes] * scales.astype(np.float64)[..., None]


def nvfp4_quantize_rows(x_bits: np.ndarray):
    """bf16 rows [..., D] -> (packed codes uint8 [..., D/2], block scales uint8 E4M3 [..., D/16])."""
    x = (np.asarray(x_bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    D = x.shape[-1]
    assert D % 16 == 0
    xb = x.reshape(x.shape[:-1] + (D // 16, 16))
    amax = np.max(np.abs(xb), axis=-1)                                 # [..., D/16]
    sb_code = e4m3_encode((amax / np.float32(E2M1_MAX)).astype(np.float32))
    sb = E4M3_TABLE[sb_code].astype(np.float32)                        # exact in fp32
    safe = np.where(sb == 0, np.float32(1.0), sb).astype(np.float32)
    y = (xb / safe[..., None]).astype(np.float32)                      # fp32 quotients
    codes = e2m1_encode(y)
    codes = np.where((sb == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    codes = codes.reshape(x.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << np.uint8(4))).astype(np.uint8)
    return packed, sb_code


def nvfp4_dequantize_rows(packed: np.ndarray, sb_code: np.ndarray) -> np.ndarray:
    lo = packed & np.uint8(0xF)
    hi = packed >> np.uint8(4)
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))
    vals = E2M1_TABLE[codes]
    D = vals.shape[-1]
    vb = vals.reshape(vals.shape[:-1] + (D // 16, 16)) * E4M3_TABLE[sb_code][..., None]
    return vb.reshape(vals.shape)
