"""Full-size parity in the launch configuration the benchmark times: the
30-layer Wan-1.3B-shaped stack (12 heads, head_dim 128, 1560 tokens per frame,
chunk 3, sink 3, window 9), attention then append for every layer of every
chunk over 60 chunks, and a prompt switch before chunk 20 that rewrites the
sink + window of all 30 layers in one ll_kv_recache_write call.

Three layers (first, middle, last) are checked against the fp64 oracle on
sampled query rows at chunks 0, 1, 4 (cache full), 20 (first chunk after the
recache), 21 and 59, and their cache bytes against the cache oracle at the end.
A checked layer carries seeded host inputs in every chunk whose frames are
visible at a check or held at the end; its other chunks, and all chunks of the
other layers, get device-random inputs (their frames are evicted or recached
before anyone looks, which the test asserts). Layers are independent: the
unchecked ones only have to run."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_qkv, recache_kv, bf16_bits_to_f64

L, H, D, T, F, S, W = 30, 12, 128, 1560, 3, 3, 9
TQ = F * T
CHECK_LAYERS = (0, 14, 29)
SWITCH = 20
N_CHUNKS = 60
CHECKS = (0, 1, 4, 20, 21, 59)


def _held(p):
    """Absolute frames held after p appended frames (sink, then window)."""
    s, w = min(p, S), min(W, max(0, p - S))
    return list(range(s)) + list(range(p - w, p))


def _seeded_chunks():
    """Chunks whose inputs are visible at a check or held at the end. Frames
    overwritten by the recache no longer depend on their chunk's input."""
    src = {}                       # frame -> chunk whose input it holds, or None (recached)
    need = set()
    for c in range(N_CHUNKS):
        if c == SWITCH:
            for f in _held(c * F):
                src[f] = None
        if c in CHECKS:
            need.add(c)
            need |= {src[f] for f in _held(c * F) if src[f] is not None}
        for f in range(c * F, (c + 1) * F):
            src[f] = c
    need |= {src[f] for f in _held(N_CHUNKS * F) if src[f] is not None}
    return need, src


def test_seeded_chunk_selection_covers_every_visible_frame():
    """Host-side check of the selection above (CPU suite)."""
    need, _ = _seeded_chunks()
    assert need == {0, 1, 2, 3, 4, 20, 21, 56, 57, 58, 59}


@pytest.mark.gpu
def test_wan_stack_with_prompt_switch():
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, sample_rows
    torch.manual_seed(3)
    need, _ = _seeded_chunks()
    ci = {l: i for i, l in enumerate(CHECK_LAYERS)}
    model = oracle.CacheModel(len(CHECK_LAYERS), H, D, T, F, S, W)
    frame_src = [dict() for _ in CHECK_LAYERS]     # frame -> seeded chunk, "r" (recached) or None
    zeros = np.zeros((TQ, H, D), np.uint16)
    cache = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    try:
        other = [torch.randn(3, TQ, H, D, device="cuda").to(torch.bfloat16) for _ in range(2)]
        outs = {l: torch.empty(TQ, H, D, device="cuda", dtype=torch.bfloat16) for l in CHECK_LAYERS}
        scratch = torch.empty(TQ, H, D, device="cuda", dtype=torch.bfloat16)
        for c in range(N_CHUNKS):
            if c == SWITCH:
                # prompt switch: new K/V for the held frames (sink + window) of all layers
                n_held = S + W
                kn = torch.randn(L, n_held * T, H, D, device="cuda").to(torch.bfloat16)
                vn = torch.randn(L, n_held * T, H, D, device="cuda").to(torch.bfloat16)
                for l in CHECK_LAYERS:
                    k_new, v_new = recache_kv(3, l, 0, n_held * T, H, D)
                    kn[l].copy_(to_dev(k_new))
                    vn[l].copy_(to_dev(v_new))
                    model.recache_write(ci[l], k_new[None], v_new[None], 0, n_held)
                    for f in _held(c * F):
                        frame_src[ci[l]][f] = "r"
                ll.ll_kv_recache_write(cache, -1, kn, vn, 0, n_held)
                del kn, vn
            seeded, dev_in = {}, {}
            for l in CHECK_LAYERS:
                seeded[l] = chunk_qkv(3, l, c, TQ, H, D) if c in need else None
                dev_in[l] = tuple(to_dev(x) for x in seeded[l]) if c in need else other[(l + c) % 2]
            for l in range(L):
                if l in ci:
                    dq, dk, dv = dev_in[l]
                    ll.ll_attn_sink_window(dq, dk, dv, cache, l, outs[l])
                    ll.ll_kv_append(cache, l, dk, dv)
                else:
                    t = other[l % 2]
                    ll.ll_attn_sink_window(t[0], t[1], t[2], cache, l, scratch)
                    ll.ll_kv_append(cache, l, t[1], t[2])
            for l in CHECK_LAYERS:
                if c in CHECKS:
                    q, k, v = seeded[l]
                    held = _held(c * F)
                    assert all(frame_src[ci[l]][f] is not None for f in held), "unseeded frame visible"
                    n = (c + 1) * TQ
                    kh = np.zeros((n, H, D), np.float32)   # untouched pages stay uncommitted
                    vh = np.zeros((n, H, D), np.float32)
                    for f, vals in model.held_frames(ci[l], 0).items():
                        kh[f * T:(f + 1) * T] = vals
                    for f, vals in model.held_frames(ci[l], 1).items():
                        vh[f * T:(f + 1) * T] = vals
                    kh[c * TQ:] = bf16_bits_to_f64(k)
                    vh[c * TQ:] = bf16_bits_to_f64(v)
                    torch.cuda.synchronize()
                    rows = sample_rows(TQ, 96, 1000 + 7 * c + l)
                    ref = oracle.sink_window_attention(q, kh, vh, c, S, W, F, T, rows=rows)
                    assert_attn_close(dev_to_f64(outs[l])[rows], ref, f"layer {l} chunk {c}")
                    del kh, vh
                if seeded[l] is not None:
                    model.append(ci[l], seeded[l][1], seeded[l][2])
                    src = c
                else:
                    model.append(ci[l], zeros, zeros)
                    src = None
                for f in range(c * F, (c + 1) * F):
                    frame_src[ci[l]][f] = src
        torch.cuda.synchronize()
        for l in CHECK_LAYERS:
            assert all(frame_src[ci[l]][f] is not None for f in _held(N_CHUNKS * F))
            assert ll.ll_kv_cache_export(cache, l) == model.export(ci[l]), f"layer {l} cache bytes"
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()
