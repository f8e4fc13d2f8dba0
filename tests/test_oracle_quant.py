"""Pins of the quantiser oracle (O3): exhaustive code tables, hand-derived ties
and saturation cases (tests/golden/fp8_fp4_rounding_cases.txt), and
round-to-nearest-even casts of an independent library (ml_dtypes)."""
import os

import ml_dtypes
import numpy as np

from oracle import quant
from seeded_inputs import bf16_normal, mix_seed, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_table_against_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        a, b = quant.E4M3_TABLE[c], lib[c]
        assert (np.isnan(a) and np.isnan(b)) or a == b, c
    assert quant.E4M3_TABLE[0x7E] == 448.0 and quant.E4M3_TABLE[0x01] == 2.0 ** -9


def test_e2m1_table_against_library():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64) \
        if hasattr(ml_dtypes, "float4_e2m1fn") else None
    assert list(quant.E2M1_TABLE[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    if lib is not None:
        np.testing.assert_array_equal(np.abs(quant.E2M1_TABLE), np.abs(lib))


def test_roundtrip_all_codes():
    for c in range(256):
        v = quant.E4M3_TABLE[c]
        if np.isnan(v):
            continue
        assert int(quant.e4m3_encode(np.float32(v))) == c, hex(c)
    for c in range(16):
        assert int(quant.e2m1_encode(np.float32(quant.E2M1_TABLE[c]))) == c


def test_hand_derived_cases():
    with open(os.path.join(GOLDEN, "fp8_fp4_rounding_cases.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            fmt, val, code = line.split()
            x = np.float32(float(val))
            enc = quant.e4m3_encode(x) if fmt == "e4m3" else quant.e2m1_encode(x)
            assert int(enc) == int(code, 16), (fmt, val)


def test_e4m3_rne_matches_library_on_random_values():
    rng = np.random.default_rng(1)
    y = (rng.standard_normal(200000) * np.exp2(rng.integers(-12, 9, 200000))).astype(np.float32)
    y = y[np.abs(y) < 464]           # the library cast turns overflow into NaN; saturation is pinned above
    ours = quant.e4m3_encode(y)
    lib = y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(ours, lib)


def test_e2m1_rne_matches_library_on_random_values():
    rng = np.random.default_rng(2)
    y = (rng.standard_normal(100000) * 2.5).astype(np.float32)
    y = y[np.abs(y) <= 6]
    ours = quant.e2m1_encode(y)
    lib = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & np.uint8(0xF)
    np.testing.assert_array_equal(ours, lib)


def test_fp8_rows_error_bound_and_scale():
    x = bf16_normal(mix_seed(8, 8), (300, 4, 128))
    codes, sc = quant.fp8_quantize_rows(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    amax = np.abs(xf).max(-1)
    # the scale is a power of two with amax / 448 <= scale < 2 * amax / 448
    m, _ = np.frexp(sc.astype(np.float64))
    assert np.all(m == 0.5)
    assert np.all(amax <= 448 * sc) and np.all(448 * sc < 2 * amax)
    deq = quant.fp8_dequantize_rows(codes, sc)
    # E4M3 has 3 fraction bits: relative error <= 2^-4 for normals, absolute <= 2^-10 * scale below
    err = np.abs(deq - xf)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, sc[..., None].astype(np.float64) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-6))
    # the row maximum lands in (224, 448] before rounding, so its code is at least 224
    assert np.all(np.abs(quant.E4M3_TABLE[codes]).max(-1) >= 224)
    # every dequantised value is exact in bf16 (at most 8 significant bits, in range)
    d32 = deq.astype(np.float32)
    assert np.all(d32.astype(np.float64) == deq)
    assert np.all((d32.view(np.uint32) & 0xFFFF) == 0)


def test_fp8_scale_hand_derived_cases():
    """Hand-derived: a row with maximum 448 has scale 1 and keeps its values
    (448 -> 0x7E, -1 -> 0xB8); 450 (exact in bf16) needs scale 2: 450/2 = 225
    rounds to the E4M3 value 224 (0x76), 3/2 = 1.5 (0x3C); a maximum of 1
    gives scale 2^-8 (1/448 lies between 2^-9 and 2^-8), so 1 -> 256 (0x78)
    and 0.5 -> 128 (0x70); a maximum of exactly 7 * 2^-6 = 448 * 2^-12 gives
    scale 2^-12 exactly and the code 448 (0x7E)."""
    vals = [[448.0, -1.0], [450.0, 3.0], [1.0, 0.5], [7 * 2.0 ** -6, 0.0]]
    y = np.array([f32_to_bf16_bits(np.array(v, dtype=np.float32)) for v in vals], dtype=np.uint16)
    codes, sc = quant.fp8_quantize_rows(y)
    assert sc.tolist() == [1.0, 2.0, 2.0 ** -8, 2.0 ** -12]
    assert codes.tolist() == [[0x7E, 0xB8], [0x76, 0x3C], [0x78, 0x70], [0x7E, 0x00]]


def test_fp8_zero_row_and_sign():
    x = np.zeros((2, 1, 16), dtype=np.uint16)
    x[1, 0, 3] = f32_to_bf16_bits(np.array([-2.0], dtype=np.float32))[0]
    codes, sc = quant.fp8_quantize_rows(x)
    assert sc[0, 0] == 1.0 and not codes[0].any()
    # amax 2: scale 2^-7 (2/448 lies between 2^-8 and 2^-7), -2 * 128 = -256 -> 0xF8
    assert codes[1, 0, 3] == 0xF8 and sc[1, 0] == np.float32(2.0 ** -7)


def test_fp8_tiny_rows_use_the_floor_scale():
    """Rows whose maximum is below 448 * 2^-124 take the floor scale 2^-124.
    Hand-derived: a row holding only the smallest positive bf16 subnormal
    2^-133 has x * 2^124 = 2^-9, the smallest E4M3 subnormal (code 0x01);
    its zeros stay code 0x00; at exactly 448 * 2^-124 the maximum gets the
    floor itself and the code 448 (0x7E)."""
    y = np.zeros((3, 16), dtype=np.uint16)
    y[0, 2] = 0x0001                                     # 2^-133
    y[1, 0] = 0x8001                                     # -2^-133
    y[2, 5] = f32_to_bf16_bits(np.array([448.0 * 2.0 ** -124], dtype=np.float32))[0]
    codes, sc = quant.fp8_quantize_rows(y)
    assert sc.view(np.uint32).tolist() == [0x01800000] * 3
    assert codes[0, 2] == 0x01 and codes[1, 0] == 0x81 and codes[2, 5] == 0x7E
    assert int(np.count_nonzero(codes)) == 3


def test_fp8_every_bf16_row_maximum_gives_finite_codes():
    """Every finite bf16 value as the only non-zero element of a row, next to a
    zero: no NaN code (S.1111.111) ever appears, the scale is a finite positive
    power of two, the value comes back within the E4M3 bound (half a step:
    2^-4 relative for normals, 2^-10 * scale for subnormals), and the
    dequantised value is exact in bf16 (except the top of the bf16 range,
    where code x scale reaches 2^128)."""
    p = np.arange(1 << 16, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    x = np.zeros((len(p), 2), dtype=np.uint16)
    x[:, 0] = p
    codes, sc = quant.fp8_quantize_rows(x)
    assert not np.any((codes & 0x7F) == 0x7F)
    assert np.all(np.isfinite(sc)) and np.all(sc > 0)
    assert np.all(np.frexp(sc.astype(np.float64))[0] == 0.5)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = quant.fp8_dequantize_rows(codes, sc)
    err = np.abs(deq - xf)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, sc[:, None].astype(np.float64) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-6))
    fin = np.abs(deq) < 2.0 ** 128
    d32 = deq[fin].astype(np.float32)
    assert np.all(d32.astype(np.float64) == deq[fin]) and np.all((d32.view(np.uint32) & 0xFFFF) == 0)
    assert np.count_nonzero(~fin) <= 16


def test_nvfp4_blocks_error_bound_and_packing():
    x = bf16_normal(mix_seed(9, 9), (200, 3, 64))
    packed, sb = quant.nvfp4_quantize_rows(x)
    assert packed.shape == (200, 3, 32) and sb.shape == (200, 3, 4)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = quant.nvfp4_dequantize_rows(packed, sb)
    blk = xf.reshape(200, 3, 4, 16)
    amax = np.abs(blk).max(-1, keepdims=True)
    # E2M1 step is at most 2 (between 4 and 6): half-step error at block scale amax/6,
    # plus the E4M3 rounding of the scale (<= 2^-4 relative) applied to values <= 6
    err = np.abs(deq.reshape(blk.shape) - blk)
    assert np.all(err <= amax / 6 * (1 + 2 ** -4) * 1.0 + amax * 2 ** -4 + 1e-12)
    # element 2i lives in the low nibble
    codes = quant.e2m1_encode(np.float32(1.0)), quant.e2m1_encode(np.float32(-3.0))
    y = np.zeros((1, 16), dtype=np.uint16)
    y[0, 0] = f32_to_bf16_bits(np.array([6.0], dtype=np.float32))[0]   # sb = E4M3(1) = 1
    y[0, 1] = f32_to_bf16_bits(np.array([-3.0], dtype=np.float32))[0]
    p, s = quant.nvfp4_quantize_rows(y)
    assert s[0, 0] == 0x38 and p[0, 0] == (0x7 | (0xD << 4))
    del codes


def test_nvfp4_tiny_block_is_zero():
    y = np.zeros((1, 16), dtype=np.uint16)
    y[0, 5] = 0x0001          # smallest positive bf16 subnormal: amax/6 rounds to E4M3 zero
    p, s = quant.nvfp4_quantize_rows(y)
    assert s[0, 0] == 0 and not p.any()
