"""Pins of the cache oracle (O2).

* invariant: after any sequence of appends the held context, read in logical
  order, is the first S frames plus the last W non-sink frames, checked against
  a list + bounded-deque simulation that knows nothing about slots or modulo;
* recache equivalence: a prompt switch followed by a recache of the held frames
  leaves the bytes equal to a fresh cache into which the same frames were
  appended with the new K/V;
* constant footprint over a long rollout.
"""
import collections

import numpy as np
import pytest

from oracle import CacheModel
from seeded_inputs import bf16_normal, mix_seed


def _chunk(seed, c, F, T, H, D):
    return (bf16_normal(mix_seed(seed, c, 1), (F * T, H, D)), bf16_normal(mix_seed(seed, c, 2), (F * T, H, D)))


@pytest.mark.parametrize("S,W,F,T", [(3, 9, 3, 2), (3, 6, 3, 1), (0, 4, 2, 2), (2, 0, 2, 1), (3, 2, 3, 2),
                                     (5, 3, 2, 1), (1, 1, 1, 3), (2, 7, 4, 1)])
def test_logical_view_is_sink_plus_last_window(S, W, F, T):
    H, D = 2, 8
    seed = mix_seed(S, W, F, T, 11)
    m = CacheModel(1, H, D, T, F, S, W)
    sink = []
    window = collections.deque(maxlen=W) if W > 0 else None
    for c in range(14):
        k, v = _chunk(seed, c, F, T, H, D)
        m.append(0, k, v)
        for fi in range(F):
            fr = (k[fi * T:(fi + 1) * T], v[fi * T:(fi + 1) * T])
            if len(sink) < S:
                sink.append(fr)
            elif window is not None:
                window.append(fr)
        held = sink + (list(window) if window is not None else [])
        want_k = np.concatenate([h[0] for h in held]) if held else np.zeros((0, H, D), np.uint16)
        want_v = np.concatenate([h[1] for h in held]) if held else np.zeros((0, H, D), np.uint16)
        np.testing.assert_array_equal(m.logical_view(0, 0), want_k)
        np.testing.assert_array_equal(m.logical_view(0, 1), want_v)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("S,W,F,T,switch,first,num", [
    (3, 9, 3, 2, 20, 0, 12),     # sink + window (all held frames)
    (3, 9, 3, 2, 20, 3, 9),      # window only, sink unchanged
    (3, 6, 3, 1, 5, 2, 4),       # a sub-range
    (2, 5, 3, 2, 1, 0, 2),       # early: window not yet full
])
def test_recache_equals_fresh_append(kv_dtype, S, W, F, T, switch, first, num):
    L, H, D = 2, 2, 32
    seed = mix_seed(S, W, F, T, switch, first, num)
    chunks = [[_chunk(mix_seed(seed, l), c, F, T, H, D) for c in range(switch + 4)] for l in range(L)]
    a = CacheModel(L, H, D, T, F, S, W, kv_dtype)
    for c in range(switch):
        for l in range(L):
            a.append(l, *chunks[l][c])
    # the frames held at the switch, by absolute frame number, in logical order
    p = switch * F
    s, w = min(p, S), min(W, max(0, p - S))
    held = list(range(s)) + list(range(p - w, p))
    sel = held[first:first + num]
    k_new = np.stack([bf16_normal(mix_seed(seed, 900, l, 1), (num * T, H, D)) for l in range(L)])
    v_new = np.stack([bf16_normal(mix_seed(seed, 900, l, 2), (num * T, H, D)) for l in range(L)])
    a.recache_write(-1, k_new, v_new, first, num)
    # fresh cache: append the same history with the recached frames replaced
    b = CacheModel(L, H, D, T, F, S, W, kv_dtype)
    for c in range(switch):
        for l in range(L):
            k, v = (x.copy() for x in chunks[l][c])
            for i, fr in enumerate(sel):
                if fr // F == c:
                    t0 = (fr % F) * T
                    k[t0:t0 + T] = k_new[l, i * T:(i + 1) * T]
                    v[t0:t0 + T] = v_new[l, i * T:(i + 1) * T]
            b.append(l, k, v)
    for l in range(L):
        assert a.export(l) == b.export(l)
    # generation continues identically afterwards
    for c in range(switch, switch + 4):
        for l in range(L):
            a.append(l, *chunks[l][c])
            b.append(l, *chunks[l][c])
    for l in range(L):
        assert a.export(l) == b.export(l)


def test_single_layer_recache_touches_only_that_layer():
    L, H, D, T, F, S, W = 3, 1, 16, 2, 3, 3, 6
    m = CacheModel(L, H, D, T, F, S, W)
    for c in range(5):
        for l in range(L):
            m.append(l, *_chunk(mix_seed(l), c, F, T, H, D))
    before = [m.export(l) for l in range(L)]
    k_new = bf16_normal(mix_seed(1, 2, 3), (1, 9 * T, H, D))
    m.recache_write(1, k_new, k_new, 0, 9)
    assert m.export(0) == before[0] and m.export(2) == before[2] and m.export(1) != before[1]


def test_constant_footprint_long_rollout():
    m = CacheModel(1, 1, 16, 2, 3, 3, 9)
    buf = m.data
    n0 = m.export_nbytes()
    for c in range(320):
        k, v = _chunk(7, c, 3, 2, 1, 16)
        m.append(0, k, v)
        assert m.data is buf and m.export_nbytes() == n0
    assert m.held(0) == (3, 9)


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
def test_held_frames_are_the_appended_frames_dequantized(kv_dtype):
    """held_frames maps absolute frame numbers to the values of exactly those
    frames: bf16 frames bit-exact, quantised frames within the format's error
    bound of the appended values (and equal to quantising each frame alone)."""
    from oracle import quant
    from seeded_inputs import bf16_bits_to_f64
    S, W, F, T, H, D = 3, 6, 3, 2, 2, 32
    m = CacheModel(1, H, D, T, F, S, W, kv_dtype)
    frames = {}
    for c in range(7):
        k, v = _chunk(mix_seed(5, 5), c, F, T, H, D)
        m.append(0, k, v)
        for fi in range(F):
            frames[c * F + fi] = k[fi * T:(fi + 1) * T]
    held = m.held_frames(0, 0)
    p = 7 * F
    assert sorted(held) == list(range(S)) + list(range(p - W, p))
    for f, vals in held.items():
        x = frames[f]
        if kv_dtype == "bf16":
            np.testing.assert_array_equal(vals, bf16_bits_to_f64(x))
        elif kv_dtype == "fp8":
            codes, sc = quant.fp8_quantize_rows(np.transpose(x, (1, 0, 2)))
            np.testing.assert_array_equal(vals, np.transpose(quant.fp8_dequantize_rows(codes, sc), (1, 0, 2)))
        else:
            codes, sb = quant.nvfp4_quantize_rows(np.transpose(x, (1, 0, 2)))
            np.testing.assert_array_equal(vals, np.transpose(quant.nvfp4_dequantize_rows(codes, sb), (1, 0, 2)))
