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
