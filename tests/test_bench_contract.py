"""Host-side checks of bench.py (no GPU): the work and byte counts its roofline
divides by, worked out here from the geometry by hand, the peak denominators,
and that a recorded DRAM-traffic figure belongs to the current kernel sources."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_wan_geometry_and_visible_keys():
    # 3 sink + 9 window cached frames and the own 3-frame chunk, 1560 tokens each
    assert (bench.H, bench.D, bench.T, bench.F, bench.S, bench.W) == (12, 128, 1560, 3, 3, 9)
    assert bench.TQ == 4680
    assert bench.NK == 15 * 1560 == 23400


def test_attention_work_and_minimum_bytes():
    # QK^T and PV: 2 flops per multiply-add each, over visible keys only
    assert bench.ATTN_FLOP == 4 * 4680 * 23400 * 128 * 12 == 672_841_728_000
    # q, k_cur, v_cur, out: 4 x 4680 x 12 x 128 bf16 = 57.5 MB; cached K and V
    # of 12 frames: 2 x 18720 x 12 x 128 bf16 = 115.0 MB
    assert bench.ATTN_MIN_BYTES == 57_507_840 + 115_015_680


def test_append_and_recache_bytes():
    # append of one layer: K and V of the chunk read once and written once
    assert bench.APPEND_BYTES == 2 * 28_753_920
    # recache of 30 layers x 12 frames, K and V, read + write
    assert bench.recache_bytes(30) == 6_900_940_800
    # quantised rows: FP8 128 codes + 4-byte scale; NVFP4 64 bytes of codes + 8 block scales
    assert bench.QUANT_ROW_BYTES == {"fp8": 132, "nvfp4": 72}


def test_peaks_come_from_the_measured_file():
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
        p = json.load(fh)
    burst, sustained, hbm, kind = bench._peaks()
    assert kind == "measured"
    assert (burst, sustained, hbm) == (p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"])


def test_recorded_traffic_matches_the_kernel_sources():
    """A DRAM-traffic figure from ncu is kept only with the hash of the sources it
    was captured from; after a kernel change it must be re-captured or set to None."""
    assert bench.ATTN_TRAFFIC is None or bench.ATTN_TRAFFIC_SRC_SHA == bench._kernel_sha(), \
        "attention kernel sources changed since the traffic capture: re-capture it or set ATTN_TRAFFIC = None"
    if bench.ATTN_TRAFFIC is not None:
        # a launch cannot move less than its minimum bytes by much (L2 hits aside)
        # and wasted re-reads would show as far more
        assert 0.8 * bench.ATTN_MIN_BYTES < bench.ATTN_TRAFFIC < 1.5 * bench.ATTN_MIN_BYTES


def test_tiny_configuration_oracle_run():
    """The CPU baseline also times the whole tiny configuration: 8 chunks whose
    visible keys grow 48, 96, 144, then 192 (sink 3 + window 6 + own 3 frames
    of 16 tokens) for the last five."""
    r = bench.cpu_oracle_config0()
    keys = 48 + 96 + 144 + 5 * 192
    assert r["tflop"] * 1e12 == pytest.approx(4 * 48 * keys * 64 * 2, rel=1e-12)
    assert 0 < r["seconds"] < 30


def test_datasheet_figure_is_the_dense_one():
    # 2.25 PFLOP/s dense bf16; the 4.5 PFLOP/s figure assumes 2:4 sparsity
    assert bench.DATASHEET_BF16_DENSE_TFLOPS == 2250.0
