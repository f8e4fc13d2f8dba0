"""GPU parity of multi-shot caches (a global sink every shot sees, a sink per
shot, the window; LongLive-2.0 explainer, wmrh.cn, sec. 16).

* Cache bytes after every append, shot start and recache equal the oracle's
  cache model byte for byte, in all three formats, on random shot schedules
  (with and without window restarts, so the window's ring range wraps).
* Attention of every chunk against the fp64 oracle over the frames that
  multishot_visible_frames names (the frame-classification definition, not
  the ring), within the standard bound.
* ll_kv_cache_held agrees with the model; a captured chunk step that contains
  a shot start replays correctly."""
import random

import numpy as np
import pytest

import oracle
from oracle.attention import multishot_visible_frames
from seeded_inputs import chunk_qkv, bf16_bits_to_f64, recache_kv, mix_seed

pytestmark = pytest.mark.gpu


def _schedule(seed, n_chunks, p=0.3):
    rng = random.Random(seed)
    return {c: rng.random() < 0.5 for c in range(1, n_chunks) if rng.random() < p}


def _history(model, layer, k, v, c, F, T, H, D):
    n = (c + 1) * F * T
    kh = np.zeros((n, H, D))
    vh = np.zeros((n, H, D))
    for f, vals in model.held_frames(layer, 0).items():
        kh[f * T:(f + 1) * T] = vals
    for f, vals in model.held_frames(layer, 1).items():
        vh[f * T:(f + 1) * T] = vals
    kh[c * F * T:] = bf16_bits_to_f64(k)
    vh[c * F * T:] = bf16_bits_to_f64(v)
    return kh, vh


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("H,D,T,F,G,Ss,W,n,seed", [
    (2, 64, 16, 3, 3, 3, 6, 14, 1),      # the reference geometry with a shot sink
    (2, 128, 40, 1, 1, 2, 3, 16, 2),     # one frame per chunk: shot sinks fill across chunks
    (1, 128, 50, 3, 2, 1, 2, 12, 3),     # W < F and a one-frame shot sink
    (2, 64, 129, 2, 0, 2, 3, 12, 4),     # no global sink; ragged 129-token frames
    (1, 64, 16, 3, 2, 2, 0, 8, 5),       # no window at all
])
def test_multishot_rollout_matches_oracle(kv_dtype, H, D, T, F, G, Ss, W, n, seed):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    Tq = F * T
    shots = _schedule(mix_seed(seed, 31), n)
    model = oracle.CacheModel(1, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss)
    cache = ll.ll_kv_cache_create_multishot(1, H, D, T, F, G, Ss, W, kv_dtype)
    try:
        for c in range(n):
            if c in shots:
                ll.ll_kv_shot_begin(cache, 0, shots[c])
                model.shot_begin(0, shots[c])
            assert ll.ll_kv_cache_held(cache, 0) == model.held3(0)
            q, k, v = chunk_qkv(60 + seed, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            vis = multishot_visible_frames(c, G, Ss, W, F, sorted(shots.items()))
            assert sorted(set(model.held_frames(0, 0)) | set(range(c * F, (c + 1) * F))) == vis
            kh, vh = _history(model, 0, k, v, c, F, T, H, D)
            torch.cuda.synchronize()
            ref = oracle.sink_window_attention(q, kh, vh, c, 0, 0, F, T, visible_frames=vis)
            assert_attn_close(dev_to_f64(out), ref, f"{kv_dtype} chunk {c} shots {sorted(shots.items())}")
            model.append(0, k, v)
            assert ll.ll_kv_cache_export(cache, 0) == model.export(0), f"cache bytes after chunk {c}"
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "nvfp4"])
def test_multishot_recache_all_layers_bit_exact(kv_dtype):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    L, H, D, T, F, G, Ss, W = 3, 2, 128, 24, 3, 3, 3, 6
    shots = {4: False, 7: True}
    model = oracle.CacheModel(L, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss)
    cache = ll.ll_kv_cache_create_multishot(L, H, D, T, F, G, Ss, W, kv_dtype)
    try:
        for c in range(10):
            if c in shots:
                ll.ll_kv_shot_begin(cache, -1, shots[c])
                model.shot_begin(-1, shots[c])
            for l in range(L):
                _, k, v = chunk_qkv(70, l, c, F * T, H, D)
                ll.ll_kv_append(cache, l, to_dev(k), to_dev(v))
                model.append(l, k, v)
            if c in (5, 8, 9):
                n_held = model.n_held(0)
                first = 1 if c == 8 else 0
                num = n_held - first
                kn = np.stack([recache_kv(70, l, c, num * T, H, D)[0] for l in range(L)])
                vn = np.stack([recache_kv(70, l, c, num * T, H, D)[1] for l in range(L)])
                ll.ll_kv_recache_write(cache, -1, to_dev(kn), to_dev(vn), first, num)
                model.recache_write(-1, kn, vn, first, num)
                with pytest.raises(ll.LLError):        # one frame more than held
                    ll.ll_kv_recache_write(cache, -1, to_dev(kn), to_dev(vn), first, num + 1)
        torch.cuda.synchronize()
        for l in range(L):
            assert ll.ll_kv_cache_export(cache, l) == model.export(l), f"layer {l}"
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_multishot_wan_shape_sampled_rows():
    """Wan-1.3B single-layer shape, global sink 3, shot sink 3, window 6; a new
    shot at chunk 6 that keeps the window, another at chunk 9 that restarts it."""
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, sample_rows
    H, D, T, F, G, Ss, W = 12, 128, 1560, 3, 3, 3, 6
    Tq = F * T
    shots = {6: False, 9: True}
    checks = {2, 5, 6, 7, 9, 11}
    model = oracle.CacheModel(1, H, D, T, F, G, W, shot_sink_frames=Ss)
    cache = ll.ll_kv_cache_create_multishot(1, H, D, T, F, G, Ss, W)
    try:
        for c in range(12):
            if c in shots:
                ll.ll_kv_shot_begin(cache, 0, shots[c])
                model.shot_begin(0, shots[c])
            q, k, v = chunk_qkv(80, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            if c in checks:
                vis = multishot_visible_frames(c, G, Ss, W, F, sorted(shots.items()))
                kh, vh = _history(model, 0, k, v, c, F, T, H, D)
                torch.cuda.synchronize()
                rows = sample_rows(Tq, 128, 500 + c)
                ref = oracle.sink_window_attention(q, kh, vh, c, 0, 0, F, T, rows=rows, visible_frames=vis)
                assert_attn_close(dev_to_f64(out)[rows], ref, f"chunk {c}")
            model.append(0, k, v)
        assert ll.ll_kv_cache_export(cache, 0) == model.export(0)
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_captured_step_with_shot_start_replays():
    """A graph holding [shot start, attention, append] replayed chunk after
    chunk equals the same calls made eagerly, bit for bit."""
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    H, D, T, F, G, Ss, W = 2, 128, 40, 1, 1, 2, 4
    Tq = F * T
    eager = ll.ll_kv_cache_create_multishot(1, H, D, T, F, G, Ss, W)
    graphed = ll.ll_kv_cache_create_multishot(1, H, D, T, F, G, Ss, W)
    try:
        q_in, k_in, v_in = (torch.empty(Tq, H, D, device="cuda", dtype=torch.bfloat16) for _ in range(3))
        out_e, out_g = torch.empty_like(q_in), torch.empty_like(q_in)

        def step(cache, out, shot):
            if shot:
                ll.ll_kv_shot_begin(cache, 0, False)
            ll.ll_attn_sink_window(q_in, k_in, v_in, cache, 0, out)
            ll.ll_kv_append(cache, 0, k_in, v_in)

        graph = None
        for c in range(10):
            for dst, x in zip((q_in, k_in, v_in), chunk_qkv(90, 0, c, Tq, H, D)):
                dst.copy_(to_dev(x))
            # every chunk from 3 on starts a new shot: each shot is one frame
            shot = c >= 3
            step(eager, out_e, shot)
            if c < 3:
                step(graphed, out_g, False)
            else:
                if graph is None:
                    torch.cuda.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph):
                        step(graphed, out_g, True)
                graph.replay()
            torch.cuda.synchronize()
            assert torch.equal(out_e, out_g), f"chunk {c}"
        assert ll.ll_kv_cache_export(eager, 0) == ll.ll_kv_cache_export(graphed, 0)
        assert ll.ll_kv_cache_held(graphed, 0) == ll.ll_kv_cache_held(eager, 0)
        del graph
    finally:
        eager.close()
        graphed.close()
