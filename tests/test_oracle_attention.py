"""Pins of the attention oracle (O1) against things other than itself.

* brute force: Python loops over sets of frames built directly from the
  definitions (sink = first S frames, window = last W non-sink frames before the
  chunk, own chunk), math.exp softmax;
* the textbook case: when the window covers all history the method is plain
  block-causal attention, checked against torch's scaled_dot_product_attention
  in fp64 with a block-causal mask;
* closed forms: zero queries give the mean of the visible V; a single visible
  key gives its V;
* the visible-frame sets of the pages' configuration, derived by hand
  (tests/golden/visible_frames_S3_W9_F3.txt).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import bf16_normal, bf16_bits_to_f64, mix_seed

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hist(seed, chunks, F, T, H, D):
    n = chunks * F * T
    k = bf16_normal(mix_seed(seed, 1), (n, H, D))
    v = bf16_normal(mix_seed(seed, 2), (n, H, D))
    return k, v


def _brute(q_bits, k_bits, v_bits, chunk, S, W, F, T):
    """Python loops; key frames from explicit sets."""
    Tq, H, D = q_bits.shape
    sink = set(range(min(S, chunk * F)))
    window = set(range(max(S, chunk * F - W), chunk * F))
    own = set(range(chunk * F, chunk * F + F))
    frames = sorted(sink | window | own)
    keys = [f * T + t for f in frames for t in range(T)]
    q = bf16_bits_to_f64(q_bits)
    k = bf16_bits_to_f64(k_bits)
    v = bf16_bits_to_f64(v_bits)
    out = np.zeros((Tq, H, D))
    for h in range(H):
        for i in range(Tq):
            logits = [sum(q[i, h, d] * k[j, h, d] for d in range(D)) / math.sqrt(D) for j in keys]
            m = max(logits)
            w = [math.exp(x - m) for x in logits]
            z = sum(w)
            for d in range(D):
                out[i, h, d] = sum(w[a] * v[keys[a], h, d] for a in range(len(keys))) / z
    return out


@pytest.mark.parametrize("S,W,F,T,H,D,chunks", [
    (3, 6, 3, 2, 1, 4, 6),     # config-0 proportions, tiny
    (1, 2, 1, 3, 2, 4, 6),
    (0, 2, 2, 2, 1, 8, 5),     # no sink
    (2, 0, 2, 2, 1, 4, 4),     # no window
    (3, 1, 2, 1, 2, 4, 6),     # window shorter than a chunk
    (4, 3, 3, 2, 1, 4, 5),     # sink longer than a chunk
])
def test_brute_force_tiny(S, W, F, T, H, D, chunks):
    seed = mix_seed(S, W, F, T, H, D)
    k, v = _hist(seed, chunks, F, T, H, D)
    for c in range(chunks):
        q = bf16_normal(mix_seed(seed, 10 + c), (F * T, H, D))
        n = (c + 1) * F * T
        got = oracle.sink_window_attention(q, k[:n], v[:n], c, S, W, F, T)
        want = _brute(q, k[:n], v[:n], c, S, W, F, T)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("S,F,T,H,D,chunks", [(3, 3, 4, 2, 16, 6), (0, 2, 5, 1, 32, 5), (1, 1, 7, 2, 8, 8)])
def test_full_window_is_block_causal_attention(S, F, T, H, D, chunks):
    """With W >= all history the method reduces to block-causal attention (textbook)."""
    W = chunks * F
    seed = mix_seed(77, S, F, T)
    k, v = _hist(seed, chunks, F, T, H, D)
    n = chunks * F * T
    q_all = bf16_normal(mix_seed(seed, 5), (n, H, D))
    # library routine: whole sequence at once, block-causal boolean mask
    tq = torch.from_numpy(bf16_bits_to_f64(q_all)).permute(1, 0, 2)
    tk = torch.from_numpy(bf16_bits_to_f64(k)).permute(1, 0, 2)
    tv = torch.from_numpy(bf16_bits_to_f64(v)).permute(1, 0, 2)
    blk = torch.arange(n) // (F * T)
    mask = blk[None, :] <= blk[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask).permute(1, 0, 2).numpy()
    Tq = F * T
    for c in range(chunks):
        got = oracle.sink_window_attention(q_all[c * Tq:(c + 1) * Tq], k[:(c + 1) * Tq], v[:(c + 1) * Tq],
                                           c, S, W, F, T)
        np.testing.assert_allclose(got, ref[c * Tq:(c + 1) * Tq], rtol=0, atol=1e-12)


def test_no_history_is_plain_attention_within_chunk():
    S, W, F, T, H, D = 0, 0, 3, 5, 2, 16
    seed = mix_seed(91)
    k, v = _hist(seed, 4, F, T, H, D)
    Tq = F * T
    q = bf16_normal(mix_seed(seed, 3), (Tq, H, D))
    c = 3
    got = oracle.sink_window_attention(q, k[:(c + 1) * Tq], v[:(c + 1) * Tq], c, S, W, F, T)
    tq = torch.from_numpy(bf16_bits_to_f64(q)).permute(1, 0, 2)
    tk = torch.from_numpy(bf16_bits_to_f64(k[c * Tq:(c + 1) * Tq])).permute(1, 0, 2)
    tv = torch.from_numpy(bf16_bits_to_f64(v[c * Tq:(c + 1) * Tq])).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def _golden_frames():
    out = {}
    with open(os.path.join(GOLDEN, "visible_frames_S3_W9_F3.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            c, ranges = line.split(":")
            frames = []
            for r in ranges.split():
                a, b = r.split("-")
                frames += list(range(int(a), int(b) + 1))
            out[int(c)] = frames
    return out


def test_visible_frames_match_pages_configuration():
    for c, frames in _golden_frames().items():
        assert oracle.visible_key_frames(c, 3, 9, 3) == frames, c


def test_zero_queries_give_mean_of_visible_values():
    S, W, F, T, H, D = 3, 9, 3, 4, 2, 8
    chunks = 8
    seed = mix_seed(5150)
    k, v = _hist(seed, chunks, F, T, H, D)
    golden = _golden_frames()
    for c in (0, 1, 4, 5, 7):
        n = (c + 1) * F * T
        q = np.zeros((F * T, H, D), dtype=np.uint16)
        got = oracle.sink_window_attention(q, k[:n], v[:n], c, S, W, F, T)
        frames = golden.get(c) or oracle.visible_key_frames(c, S, W, F)
        if c in golden:
            assert frames == golden[c]
        toks = [f * T + t for f in frames for t in range(T)]
        mean = bf16_bits_to_f64(v[toks]).mean(axis=0)
        np.testing.assert_allclose(got, np.broadcast_to(mean, got.shape), rtol=0, atol=1e-13)


def test_single_visible_key_returns_its_value():
    S, W, F, T, H, D = 0, 0, 1, 1, 3, 8
    seed = mix_seed(4242)
    k, v = _hist(seed, 5, F, T, H, D)
    q = bf16_normal(mix_seed(seed, 9), (1, H, D))
    got = oracle.sink_window_attention(q, k[:5], v[:5], 4, S, W, F, T)
    np.testing.assert_array_equal(got, bf16_bits_to_f64(v[4:5]))


def test_steady_state_key_count_is_constant():
    """Memory and work per chunk stop growing once the window is full."""
    S, W, F, T = 3, 9, 3, 1560
    counts = [len(oracle.visible_key_frames(c, S, W, F)) * T for c in range(4, 60)]
    assert set(counts) == {(S + W + F) * T}


def test_sampled_rows_match_full_rows():
    S, W, F, T, H, D = 3, 6, 3, 16, 2, 64
    seed = mix_seed(31337)
    k, v = _hist(seed, 5, F, T, H, D)
    q = bf16_normal(mix_seed(seed, 3), (F * T, H, D))
    full = oracle.sink_window_attention(q, k, v, 4, S, W, F, T)
    rows = np.array([0, 5, 17, 47])
    part = oracle.sink_window_attention(q, k, v, 4, S, W, F, T, rows=rows)
    np.testing.assert_array_equal(part, full[rows])
