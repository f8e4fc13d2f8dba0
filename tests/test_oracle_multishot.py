"""Pins of the multi-shot oracle (global sink + per-shot sink + window).

* reduction: with no shot sink and a single shot, the visible frames are those
  of the single-shot rule, for every small geometry;
* a hand-derived two-shot example (tests/golden/);
* the cache model's held context, read in logical order, against a
  list + deque simulation that knows nothing about slots or rings;
* two independent definitions agree: the frames the cache model holds, plus
  the own chunk, are the frames multishot_visible_frames names;
* recache equivalence with shots;
* attention over an explicit visible-frame set against a plain Python loop.
"""
import collections
import os
import random

import numpy as np
import pytest

from oracle import CacheModel
from oracle.attention import multishot_visible_frames, visible_key_frames, sink_window_attention
from seeded_inputs import bf16_normal, bf16_bits_to_f64, mix_seed

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "multishot_visible_G1_Ss2_W3_F1.txt")


def test_no_shot_sink_reduces_to_single_shot_rule():
    for G in range(4):
        for W in range(6):
            for F in range(1, 4):
                if G + W < 1:
                    continue
                for c in range(9):
                    assert multishot_visible_frames(c, G, 0, W, F) == visible_key_frames(c, G, W, F)


def test_hand_derived_two_shot_example():
    n = 0
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        c, clear, *frames = (int(x) for x in line.split())
        assert multishot_visible_frames(c, 1, 2, 3, 1, [(5, bool(clear))]) == frames, (c, clear)
        n += 1
    assert n == 15


def _schedule(seed, n_chunks):
    rng = random.Random(seed)
    return sorted({(c, rng.random() < 0.5) for c in range(1, n_chunks) if rng.random() < 0.25},
                  key=lambda x: x[0])


def _chunk(seed, c, F, T, H, D):
    return (bf16_normal(mix_seed(seed, c, 1), (F * T, H, D)), bf16_normal(mix_seed(seed, c, 2), (F * T, H, D)))


GEOMS = [(1, 2, 3, 1, 2), (3, 3, 6, 3, 1), (2, 1, 2, 3, 1), (0, 2, 4, 2, 1), (3, 0, 9, 3, 1), (2, 3, 0, 2, 1),
         (1, 4, 1, 3, 1)]


@pytest.mark.parametrize("G,Ss,W,F,T", GEOMS)
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_cache_model_holds_global_shot_and_window_frames(G, Ss, W, F, T, seed):
    H, D, n = 1, 8, 16
    shots = dict(_schedule(mix_seed(seed, G, Ss, W, F), n))
    m = CacheModel(1, H, D, T, F, G, W, shot_sink_frames=Ss)
    glob, shot = [], []
    window = collections.deque()
    for c in range(n):
        if c in shots:
            m.shot_begin(0, shots[c])
            shot = []
            if shots[c]:
                window.clear()
        # held context before this chunk's append: frame sets and logical order
        held = m.held_frames(0, 0)
        expect = glob + shot + list(window)
        assert list(held.keys()) == expect
        vis = multishot_visible_frames(c, G, Ss, W, F, sorted(shots.items()))
        assert sorted(set(expect) | set(range(c * F, (c + 1) * F))) == vis
        k, v = _chunk(seed, c, F, T, H, D)
        m.append(0, k, v)
        for fi in range(F):
            f = c * F + fi
            if f < G:
                glob.append(f)
            elif len(shot) < Ss:
                shot.append(f)
            elif W > 0:
                window.append(f)
                if len(window) > W:
                    window.popleft()
        lv = m.logical_view(0, 0)
        assert lv.shape[0] == (len(glob) + len(shot) + len(window)) * T


@pytest.mark.parametrize("G,Ss,W,F,T", GEOMS[:4])
def test_logical_view_holds_the_appended_bits(G, Ss, W, F, T):
    """The stored rows, read in logical order, are exactly the bf16 bits of the
    held frames (global, shot sink, window)."""
    H, D, n = 2, 8, 14
    seed = mix_seed(G, Ss, W, F, 77)
    shots = dict(_schedule(seed, n))
    m = CacheModel(1, H, D, T, F, G, W, shot_sink_frames=Ss)
    frames = {}
    for c in range(n):
        if c in shots:
            m.shot_begin(0, shots[c])
        k, v = _chunk(seed, c, F, T, H, D)
        m.append(0, k, v)
        for fi in range(F):
            frames[c * F + fi] = k[fi * T:(fi + 1) * T]
        order = list(m.held_frames(0, 0).keys())
        want = np.concatenate([frames[f] for f in order]) if order else np.zeros((0, H, D), np.uint16)
        np.testing.assert_array_equal(m.logical_view(0, 0), want)


@pytest.mark.parametrize("kv_dtype", ["bf16", "nvfp4"])
def test_recache_with_shots_equals_fresh_append(kv_dtype):
    """Recaching every held frame equals a fresh rollout, with the same shot
    starts, whose appended frames carried the new values."""
    L, H, D, T, F, G, Ss, W = 2, 2, 32, 2, 3, 2, 3, 4
    n_before, shots = 9, {3: False, 6: True}
    seed = mix_seed(5, 5, 5)
    chunks = [[_chunk(mix_seed(seed, l), c, F, T, H, D) for c in range(n_before + 2)] for l in range(L)]
    a = CacheModel(L, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss)
    for c in range(n_before):
        if c in shots:
            a.shot_begin(-1, shots[c])
        for l in range(L):
            a.append(l, *chunks[l][c])
    held = list(a.held_frames(0, 0).keys())
    num = len(held)
    k_new = np.stack([bf16_normal(mix_seed(seed, 900, l, 1), (num * T, H, D)) for l in range(L)])
    v_new = np.stack([bf16_normal(mix_seed(seed, 900, l, 2), (num * T, H, D)) for l in range(L)])
    a.recache_write(-1, k_new, v_new, 0, num)
    b = CacheModel(L, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss)
    for c in range(n_before):
        if c in shots:
            b.shot_begin(-1, shots[c])
        for l in range(L):
            k, v = (x.copy() for x in chunks[l][c])
            for i, fr in enumerate(held):
                if fr // F == c:
                    t0 = (fr % F) * T
                    k[t0:t0 + T] = k_new[l, i * T:(i + 1) * T]
                    v[t0:t0 + T] = v_new[l, i * T:(i + 1) * T]
            b.append(l, k, v)
    for l in range(L):
        assert a.export(l) == b.export(l)


def test_attention_over_explicit_visible_frames_brute_force():
    """sink_window_attention with an explicit visible-frame set against a
    Python loop over (head, row, key)."""
    T, F, H, D, c = 2, 1, 2, 4, 8
    vis = multishot_visible_frames(c, 1, 2, 3, F, [(5, False)])
    n = (c + 1) * F * T
    q = bf16_normal(mix_seed(9, 1), (F * T, H, D))
    k = bf16_normal(mix_seed(9, 2), (n, H, D))
    v = bf16_normal(mix_seed(9, 3), (n, H, D))
    got = sink_window_attention(q, k, v, c, 0, 0, F, T, visible_frames=vis)
    qf, kf, vf = (bf16_bits_to_f64(x) for x in (q, k, v))
    for h in range(H):
        for i in range(F * T):
            keys = [j for j in range(n) if j // T in vis]
            s = [sum(qf[i, h, d] * kf[j, h, d] for d in range(D)) / np.sqrt(D) for j in keys]
            mx = max(s)
            e = [np.exp(x - mx) for x in s]
            z = sum(e)
            want = [sum(e[t] * vf[keys[t], h, d] for t in range(len(keys))) / z for d in range(D)]
            np.testing.assert_allclose(got[i, h], want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("G,Ss,W,F,T", GEOMS)
def test_spare_ring_slots_hold_the_same_frames(G, Ss, W, F, T):
    """A cache whose ring has F spare slots (R = W + F, the layout that lets
    attention and append share one launch) holds exactly the frames of the
    plain layout, with the same bits in logical order; only slots differ. And
    the frames a chunk appends never land in a slot the window covered just
    before that append."""
    H, D, n = 1, 8, 15
    seed = mix_seed(G, Ss, W, F, 91)
    shots = dict(_schedule(seed, n))
    plain = CacheModel(1, H, D, T, F, G, W, shot_sink_frames=Ss)
    spare = CacheModel(1, H, D, T, F, G, W, shot_sink_frames=Ss, ring_slots=W + F)
    for c in range(n):
        for m in (plain, spare):
            if c in shots:
                m.shot_begin(0, shots[c])
        visible_slots = {spare.logical_slot(0, k) for k in range(spare.n_held(0))}
        before = dict(spare.slot_frame[0])
        k, v = _chunk(seed, c, F, T, H, D)
        plain.append(0, k, v)
        spare.append(0, k, v)
        written = {sl for sl, f in spare.slot_frame[0].items() if before.get(sl) != f}
        assert not (written & visible_slots), f"chunk {c} wrote a visible slot"
        assert list(plain.held_frames(0, 0)) == list(spare.held_frames(0, 0))
        np.testing.assert_array_equal(plain.logical_view(0, 0), spare.logical_view(0, 0))
