"""The FP8 quantiser kernel finds its power-of-two row scale from the
exponent bits of the row maximum instead of dividing by 448: that rule,
restated in numpy, equals the oracle's scale for every finite bf16 maximum."""
import numpy as np

from oracle import quant


def _fp8_scale_log2_rule(amax: np.ndarray) -> np.ndarray:
    """The FP8 kernel's scale exponent, from the bits of amax (fp32): amax in
    [2^E, 2^(E+1)) gives k = E - 8, or E - 7 when amax > 1.75 * 2^E; below 2^-118
    (biased exponent < 9) and below -124 the floor -124 applies; 0 for amax 0."""
    bits = amax.view(np.uint32)
    eb = (bits >> 23).astype(np.int64)
    thr = ((eb.astype(np.uint32) << 23) | np.uint32(0x600000)).view(np.float32)
    k = eb - 127 - 8 + (amax > thr)
    k = np.where(eb < 9, -124, np.maximum(k, -124))
    return np.where(amax == 0, 0, k)


def test_fp8_scale_exponent_rule_equals_the_oracle_for_every_row_maximum():
    """The FP8 quantiser kernel finds the power-of-two row scale from the
    exponent bits of the row maximum; restated here, it equals the oracle's
    scale for every finite non-negative bf16 value as the maximum."""
    p = np.arange(1 << 15, dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF]
    amax = (p << 16).view(np.float32)
    x = np.zeros((len(p), 2), dtype=np.uint16)
    x[:, 0] = p
    _, sc = quant.fp8_quantize_rows(x)
    np.testing.assert_array_equal(np.exp2(_fp8_scale_log2_rule(amax).astype(np.float64)), sc.astype(np.float64))


# ---------------------------------------------------------------------------
# NVFP4: the quantiser kernel forms both of its quotients (amax / 6 for the
# block scale and x / sb for the codes) as a product with the correctly rounded
# reciprocal plus one correction step with the exact residual (Markstein):
#   q = rn(x * inv), r = rn(x - q * b) (an fma, exact), q' = rn(q + r * inv),
# with the sign of x kept. Restated here with the fp32 roundings emulated
# exactly in fp64, the resulting codes equal the oracle's (IEEE fp32 quotient,
# then E4M3 / E2M1 rounding) for every operand the kernel can meet.

def _rn32_of_exact_sum(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """fp32 rounding (nearest even) of the exact a + b, a and b fp64 arrays."""
    s = a + b
    bb = s - a
    e = (a - (s - bb)) + (b - bb)            # a + b = s + e exactly (TwoSum)
    s32 = s.astype(np.float32)
    lo = np.where(s32.astype(np.float64) > s, np.nextafter(s32, np.float32(-np.inf)), s32)
    hi = np.nextafter(lo, np.float32(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2
    # s itself is the exact sum unless e != 0; only a tie at s needs e's sign
    return np.where((s == mid) & (e != 0), np.where(e > 0, hi, lo), s32).astype(np.float32)


def _div_corrected(x: np.ndarray, b: np.float32, inv: np.float32) -> np.ndarray:
    q = (x * inv).astype(np.float32)                                       # fp32 product
    # x - q*b: q*b is exact in fp64 and within a factor 2 of x (Sterbenz), so the
    # difference is exact too; one rounding to fp32 is the fma's
    r = (x.astype(np.float64) - q.astype(np.float64) * np.float64(b)).astype(np.float32)
    q2 = _rn32_of_exact_sum(q.astype(np.float64), r.astype(np.float64) * np.float64(inv))
    return np.copysign(q2, x).astype(np.float32)


def _finite_bf16(nonneg: bool) -> np.ndarray:
    p = np.arange(1 << (15 if nonneg else 16), dtype=np.uint32)
    p = p[((p >> 7) & 0xFF) != 0xFF]
    return (p << 16).view(np.float32)


def test_nvfp4_block_scale_rule_equals_the_oracle_for_every_block_maximum():
    amax = _finite_bf16(nonneg=True)
    got = quant.e4m3_encode(_div_corrected(amax, np.float32(6.0), np.float32(1.0) / np.float32(6.0)))
    blocks = np.zeros((len(amax), 16), dtype=np.uint16)
    blocks[:, 0] = (amax.view(np.uint32) >> 16).astype(np.uint16)
    _, sb_code = quant.nvfp4_quantize_rows(blocks)
    np.testing.assert_array_equal(got, sb_code[:, 0])


def test_nvfp4_code_rule_equals_the_oracle_for_every_value_and_scale():
    """Every finite bf16 x (both signs) against every positive E4M3 scale whose
    quotient is finite: the E2M1 code of the corrected quotient equals the code
    of the IEEE fp32 quotient. (In a block |x| <= amax and sb ~ amax/6, so the
    kernel's quotients are far inside this range.)"""
    x = _finite_bf16(nonneg=False)
    n_pairs = 0
    for code in range(1, 127):
        sb = np.float32(quant.E4M3_TABLE[code])
        with np.errstate(over="ignore"):
            ref = (x / sb).astype(np.float32)                              # the oracle's quotient
        ok = np.isfinite(ref) & (np.abs(ref) < np.float32(2.0 ** 100))
        xs, ref = x[ok], ref[ok]
        got = _div_corrected(xs, sb, np.float32(1.0) / sb)
        diff = (got != ref) | (np.signbit(got) != np.signbit(ref))
        # the corrected quotient can differ from the IEEE one only where the
        # residual is subnormal: |x| < 2^-103, so |x / sb| < 2^-94 (sb >= 2^-9)
        assert not diff.any() or np.max(np.abs(ref[diff])) < 2.0 ** -94, code
        if diff.any():
            np.testing.assert_array_equal(quant.e2m1_encode(got[diff]), quant.e2m1_encode(ref[diff]))
        n_pairs += len(xs)
    assert n_pairs > 7_000_000
