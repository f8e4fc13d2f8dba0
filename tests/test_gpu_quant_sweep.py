"""GPU sweep of the FP8 and NVFP4 quantisers against the oracle's, bit for bit.

The LongLive-2.0 explainer (wmrh.cn, sec. 15.2) stores the history KV cache in
a 4-bit float format; the FP8 E4M3 row format and the NVFP4 block format used
here, and their rounding and scaling rules, are the readings written out in
oracle/quant.py. The N(0,1) rows of the other cache tests never reach the
encoder's edge branches, so here the K/V rows are crafted:

* every finite bf16 bit pattern (65280 of the 65536), in rows (FP8: 127
  patterns + one setter; NVFP4: 16-value blocks of 15 patterns + one setter)
  whose setter fixes the row or block maximum at one of several values, from
  the smallest subnormal to the largest finite bf16, and once more in a seeded
  shuffled order, so that patterns of very different sizes share a scale;
* all-zero rows and blocks (FP8 scale 1, NVFP4 block scale 0), -0 rows and
  blocks, and mixtures of +0 and -0;
* NVFP4 blocks whose maximum makes the block scale round to zero, exactly at
  the tie and just above it;
* values whose scaled quotient lands exactly on a rounding tie of the E4M3 grid
  (row maximum 448, scale 1) and of the E2M1 grid (several exact block scales);
* NVFP4 blocks with maximum above 6 * 448 = 2688, whose block scale saturates.

Each set goes through ll_kv_append (frame by frame into a cache that holds
them all), then through ll_kv_recache_write (all held frames, another
arrangement), and through the fused call ll_attn_sink_window_append; after each
call the exported cache bytes must equal the oracle cache model's."""
import numpy as np
import pytest

import oracle
from oracle.quant import E4M3_TABLE, E2M1_TABLE

pytestmark = pytest.mark.gpu

D = 128
H = 2


def _bf16(x) -> np.ndarray:
    """fp64 values that are exact in bf16 -> their bf16 bit patterns."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def _finite_patterns() -> np.ndarray:
    p = np.arange(1 << 16, dtype=np.uint32)
    return p[((p >> 7) & 0xFF) != 0xFF].astype(np.uint16)


# row/block maxima that the setter element imposes (all exact in bf16)
_SETTERS = [None, 1.0, 0.5, 7.0, 448.0, 2688.0, 3.0e4, 2.0 ** -133, 2.0 ** -126, 1.0e-20, 1.0e20,
            float(np.uint32(0x7F7F0000).view(np.float32))]


def _rows_with_setter(pats: np.ndarray, group: int, setter) -> np.ndarray:
    """pats cut into groups of `group` values, each group completed by the setter
    (or by the next pattern when setter is None) to group + 1 values; the groups
    are laid out along D."""
    per = group + 1
    n = -(-len(pats) // group)
    out = np.zeros((n, per), dtype=np.uint16)
    padded = np.concatenate([pats, np.zeros(n * group - len(pats), dtype=np.uint16)])
    out[:, :group] = padded.reshape(n, group)
    if setter is None:
        out[:, group] = np.roll(padded, 1)[::group][:n]
    else:
        out[:, group] = f32_to_bf16(setter)
    flat = out.reshape(-1)
    pad = (-len(flat)) % D
    return np.concatenate([flat, np.zeros(pad, dtype=np.uint16)]).reshape(-1, D)


def _special_rows(fmt: str) -> np.ndarray:
    rows = [np.zeros(D, np.uint16),                                # all zero
            np.full(D, 0x8000, np.uint16),                         # all -0
            np.tile(np.array([0x0000, 0x8000], np.uint16), D // 2)]  # +0 / -0 mixed
    # E4M3 ties: midpoints of adjacent codes, in a row whose maximum is 448 (scale 1)
    pos = np.sort(E4M3_TABLE[:0x7F])
    mids = (pos[:-1] + pos[1:]) / 2.0
    vals = np.concatenate([mids, -mids])
    for i in range(0, len(vals), D - 1):
        r = np.full(D, 448.0)
        chunk = vals[i:i + D - 1]
        r[:len(chunk)] = chunk
        rows.append(_bf16(r))
    # E2M1 ties for several exact block scales: block max 6*sb, quotients on the
    # midpoints {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5} of the E2M1 grid
    e2 = np.sort(E2M1_TABLE[:8])
    mids2 = (e2[:-1] + e2[1:]) / 2.0
    for sb in (1.0, 1.125, 0.5, 0.0625, 2.0 ** -9, 448.0, 3.0, 14.0):
        blk = np.concatenate([mids2, -mids2, [6.0], [-6.0]])[:16] * sb
        blk[15] = 6.0 * sb                                        # the block maximum
        rows.append(_bf16(np.tile(blk, D // 16)))
    # NVFP4 blocks whose scale rounds to 0 (max/6 at and below half the smallest
    # E4M3 subnormal, a tie that rounds to even = 0), and just above that tie
    tiny = 6.0 * 2.0 ** -10
    for m in (tiny, tiny / 2, tiny * (1 + 2.0 ** -7), 2.0 ** -133):
        blk = np.linspace(-m, m, 16)
        blk[0] = -m
        rows.append(f32_to_bf16(np.tile(blk, D // 16)))
    # NVFP4 blocks whose scale saturates at 448 (max > 2688): codes saturate at 6
    for m in (2688.0, 2700.0, 4000.0, 1.0e5, float(np.uint32(0x7F7F0000).view(np.float32))):
        blk = np.linspace(-m, m, 16)
        rows.append(f32_to_bf16(np.tile(blk, D // 16)))
    return np.stack(rows)


def f32_to_bf16(x) -> np.ndarray:
    from seeded_inputs import f32_to_bf16_bits
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def crafted_rows(fmt: str) -> np.ndarray:
    """All crafted (token, head) rows of D bf16 patterns for one format."""
    pats = _finite_patterns()
    group = D - 1 if fmt == "fp8" else 15
    rng = np.random.default_rng(1515)
    parts = [_special_rows(fmt)]
    for s in _SETTERS:
        parts.append(_rows_with_setter(pats, group, s))
    for s in (None, 1.0, 3.0e4):
        parts.append(_rows_with_setter(rng.permutation(pats), group, s))
    return np.concatenate(parts)


def _frames(rows: np.ndarray, T: int) -> np.ndarray:
    """rows -> frames [n][T][H][D], zero-padded to whole frames."""
    per = T * H
    pad = (-len(rows)) % per
    r = np.concatenate([rows, np.zeros((pad, D), np.uint16)])
    return r.reshape(-1, T, H, D)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_quantisers_bit_exact_on_crafted_rows(fmt):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    T, F = 256, 1
    rows = crafted_rows(fmt)
    kf = _frames(rows, T)
    vf = _frames(rows[::-1].copy(), T)                 # V sees the rows in the other order
    n = len(kf)
    S, W = 2, n - 2                                    # the cache holds every frame
    model = oracle.CacheModel(1, H, D, T, F, S, W, fmt)
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W, fmt)
    try:
        for f in range(n):
            ll.ll_kv_append(cache, 0, to_dev(kf[f]), to_dev(vf[f]))
            model.append(0, kf[f], vf[f])
        torch.cuda.synchronize()
        _assert_same(ll.ll_kv_cache_export(cache, 0), model.export(0), f"{fmt} append")
        # recache of every held frame, V and K rows swapped and rolled by half a frame
        kn = np.roll(vf.reshape(-1, H, D), T // 2, axis=0)[None]
        vn = np.roll(kf.reshape(-1, H, D), -T // 2, axis=0)[None]
        ll.ll_kv_recache_write(cache, 0, to_dev(kn), to_dev(vn), 0, n)
        model.recache_write(0, kn, vn, 0, n)
        torch.cuda.synchronize()
        _assert_same(ll.ll_kv_cache_export(cache, 0), model.export(0), f"{fmt} recache")
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_fused_append_quantises_bit_exact_on_crafted_rows(fmt):
    """The same rows stored by the fused call's copy warps (their own call of the
    row quantiser), a chunk at a time, on a cache with spare ring slots. The
    attention output of these extreme rows is not checked here."""
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    T, F = 256, 1
    rows = crafted_rows(fmt)
    kf = _frames(rows, T)
    vf = _frames(rows[::-1].copy(), T)
    n = len(kf)
    G, W = 2, n - 2
    model = oracle.CacheModel(1, H, D, T, F, G, W, fmt, shot_sink_frames=0, ring_slots=W + F)
    cache = ll.ll_kv_cache_create_fused(1, H, D, T, F, G, 0, W, fmt)
    q = torch.zeros(F * T, H, D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    try:
        for f in range(n):
            ll.ll_attn_sink_window_append(q, to_dev(kf[f]), to_dev(vf[f]), cache, 0, out)
            model.append(0, kf[f], vf[f])
        torch.cuda.synchronize()
        _assert_same(ll.ll_kv_cache_export(cache, 0), model.export(0), f"{fmt} fused append")
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def _assert_same(got: bytes, want: bytes, what: str):
    assert len(got) == len(want), what
    if got != want:
        a = np.frombuffer(got, np.uint8)
        b = np.frombuffer(want, np.uint8)
        bad = np.nonzero(a != b)[0]
        pytest.fail(f"{what}: {len(bad)} bytes differ, first at {bad[0]} (got {a[bad[0]]:#x}, want {b[bad[0]]:#x})")
