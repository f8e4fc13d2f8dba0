"""Fused append: ll_attn_sink_window_append on a cache made by
ll_kv_cache_create_fused (F spare ring slots) gives, per chunk, the attention
of the oracle over the visible frames and, after the call, the cache bytes of
the oracle's cache model with the same spare slots (attention then append).

Covered: the three storage formats, several shots with window restarts, W < F,
head_dim 64 and 128, ragged frames, fused and separate calls mixed on one
cache, a captured fused step replayed per chunk, and the error on a cache
without spare slots."""
import random

import numpy as np
import pytest

import oracle
from oracle.attention import multishot_visible_frames
from seeded_inputs import chunk_qkv, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


def _history(model, k, v, c, F, T, H, D):
    n = (c + 1) * F * T
    kh = np.zeros((n, H, D))
    vh = np.zeros((n, H, D))
    for f, vals in model.held_frames(0, 0).items():
        kh[f * T:(f + 1) * T] = vals
    for f, vals in model.held_frames(0, 1).items():
        vh[f * T:(f + 1) * T] = vals
    kh[c * F * T:] = bf16_bits_to_f64(k)
    vh[c * F * T:] = bf16_bits_to_f64(v)
    return kh, vh


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("H,D,T,F,G,Ss,W,n,seed,mixed", [
    (2, 128, 50, 3, 3, 0, 9, 9, 1, False),     # single shot: ragged frames, cache fills then rolls
    (2, 64, 16, 3, 3, 3, 6, 12, 2, False),     # shots with a shot sink (random starts, window restarts)
    (1, 128, 40, 3, 2, 1, 2, 9, 3, True),      # W < F; fused and separate calls mixed
    (3, 128, 129, 1, 1, 2, 3, 14, 4, True),    # one frame per chunk, one-row tail tile
])
def test_fused_rollout_matches_oracle(kv_dtype, H, D, T, F, G, Ss, W, n, seed, mixed):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    Tq = F * T
    rng = random.Random(seed)
    shots = {c: rng.random() < 0.5 for c in range(1, n) if Ss and rng.random() < 0.3}
    model = oracle.CacheModel(1, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss, ring_slots=W + F)
    cache = ll.ll_kv_cache_create_fused(1, H, D, T, F, G, Ss, W, kv_dtype)
    try:
        for c in range(n):
            if c in shots:
                ll.ll_kv_shot_begin(cache, 0, shots[c])
                model.shot_begin(0, shots[c])
            q, k, v = chunk_qkv(200 + seed, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            if mixed and c % 3 == 2:
                ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
                ll.ll_kv_append(cache, 0, dk, dv)
            else:
                ll.ll_attn_sink_window_append(dq, dk, dv, cache, 0, out)
            vis = multishot_visible_frames(c, G, Ss, W, F, sorted(shots.items()))
            kh, vh = _history(model, k, v, c, F, T, H, D)
            torch.cuda.synchronize()
            ref = oracle.sink_window_attention(q, kh, vh, c, 0, 0, F, T, visible_frames=vis)
            assert_attn_close(dev_to_f64(out), ref, f"{kv_dtype} chunk {c}")
            model.append(0, k, v)
            assert ll.ll_kv_cache_export(cache, 0) == model.export(0), f"cache bytes after chunk {c}"
            assert ll.ll_kv_cache_info(cache, 0)[0] == (c + 1) * F
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_fused_wan_shape_sampled_rows():
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, sample_rows
    H, D, T, F, S, W = 12, 128, 1560, 3, 3, 9
    Tq = F * T
    model = oracle.CacheModel(1, H, D, T, F, S, W, ring_slots=W + F)
    cache = ll.ll_kv_cache_create_fused(1, H, D, T, F, S, 0, W)
    try:
        for c in range(7):
            q, k, v = chunk_qkv(210, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window_append(dq, dk, dv, cache, 0, out)
            if c in (1, 4, 6):
                vis = multishot_visible_frames(c, S, 0, W, F)
                kh, vh = _history(model, k, v, c, F, T, H, D)
                torch.cuda.synchronize()
                rows = sample_rows(Tq, 128, 700 + c)
                ref = oracle.sink_window_attention(q, kh, vh, c, 0, 0, F, T, rows=rows, visible_frames=vis)
                assert_attn_close(dev_to_f64(out)[rows], ref, f"chunk {c}")
            model.append(0, k, v)
        assert ll.ll_kv_cache_export(cache, 0) == model.export(0)
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_captured_fused_step_replays():
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    L, H, D, T, F, S, W = 2, 2, 128, 40, 3, 2, 4
    Tq = F * T
    eager = ll.ll_kv_cache_create_fused(L, H, D, T, F, S, 0, W, "fp8")
    graphed = ll.ll_kv_cache_create_fused(L, H, D, T, F, S, 0, W, "fp8")
    try:
        q_in, k_in, v_in = (torch.empty(L, Tq, H, D, device="cuda", dtype=torch.bfloat16) for _ in range(3))
        out_e, out_g = torch.empty_like(q_in), torch.empty_like(q_in)

        def step(cache, out):
            for l in range(L):
                ll.ll_attn_sink_window_append(q_in[l], k_in[l], v_in[l], cache, l, out[l])

        graph = None
        for c in range(8):
            for l in range(L):
                for dst, x in zip((q_in[l], k_in[l], v_in[l]), chunk_qkv(220, l, c, Tq, H, D)):
                    dst.copy_(to_dev(x))
            step(eager, out_e)
            if c == 0:
                step(graphed, out_g)
            else:
                if graph is None:
                    torch.cuda.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph):
                        step(graphed, out_g)
                graph.replay()
            torch.cuda.synchronize()
            assert torch.equal(out_e, out_g), f"chunk {c}"
        for l in range(L):
            assert ll.ll_kv_cache_export(eager, l) == ll.ll_kv_cache_export(graphed, l)
            assert ll.ll_kv_cache_info(graphed, l)[0] == 8 * F
        del graph
    finally:
        eager.close()
        graphed.close()


def test_fused_call_needs_spare_slots():
    import torch
    import kv_cache_attention_ll_b200 as ll
    cache = ll.ll_kv_cache_create(1, 1, 64, 4, 3, 3, 6)
    try:
        x = torch.zeros(12, 1, 64, device="cuda", dtype=torch.bfloat16)
        out = torch.empty_like(x)
        with pytest.raises(ll.LLError) as e:
            ll.ll_attn_sink_window_append(x, x, x, cache, 0, out)
        assert e.value.status == ll.LL_ERR_UNSUPPORTED
        assert ll.ll_kv_cache_info(cache, 0)[0] == 0
    finally:
        cache.close()
