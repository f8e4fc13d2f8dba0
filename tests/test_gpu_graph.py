"""Device-side frame counters: one chunk step (attention then append, every
layer) captured once in a CUDA graph and replayed for each later chunk matches
the same calls made eagerly, bit for bit, and the oracle.

The kernels read each layer's frame counter p from device memory and the
append kernel advances it, so a replay sees the p of its own chunk, not the p
at capture time. After a captured append the host no longer knows p:
ll_kv_cache_info then reads the device counter, and a recache of frames the
layer does not hold is refused by the kernel (status word ERR_RANGE, nothing
written) instead of by the host."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_qkv, recache_kv, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_captured_chunk_step_matches_eager_calls(kv_dtype):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    L, H, D, T, F, S, W = 2, 2, 128, 50, 3, 2, 5
    Tq = F * T
    n_chunks, switch = 9, 5
    eager = ll.ll_kv_cache_create(L, H, D, T, F, S, W, kv_dtype)
    graphed = ll.ll_kv_cache_create(L, H, D, T, F, S, W, kv_dtype)
    model = oracle.CacheModel(L, H, D, T, F, S, W, kv_dtype)
    try:
        q_in = [torch.empty(Tq, H, D, device="cuda", dtype=torch.bfloat16) for _ in range(L)]
        k_in = [torch.empty_like(q_in[0]) for _ in range(L)]
        v_in = [torch.empty_like(q_in[0]) for _ in range(L)]
        out_g = [torch.empty_like(q_in[0]) for _ in range(L)]
        out_e = [torch.empty_like(q_in[0]) for _ in range(L)]

        def step(cache, outs):
            for l in range(L):
                ll.ll_attn_sink_window(q_in[l], k_in[l], v_in[l], cache, l, outs[l])
                ll.ll_kv_append(cache, l, k_in[l], v_in[l])

        graph = None
        for c in range(n_chunks):
            host = [chunk_qkv(50, l, c, Tq, H, D) for l in range(L)]
            for l in range(L):
                for dst, x in zip((q_in[l], k_in[l], v_in[l]), host[l]):
                    dst.copy_(to_dev(x))
            if c == switch:
                n_held = S + W
                kn, vn = recache_kv(50, 0, c, n_held * T, H, D)
                kn_all = np.stack([kn] * L)
                vn_all = np.stack([vn] * L)
                for cache in (eager, graphed):
                    ll.ll_kv_recache_write(cache, -1, to_dev(kn_all), to_dev(vn_all), 0, n_held)
                model.recache_write(-1, kn_all, vn_all, 0, n_held)
            step(eager, out_e)
            if c == 0:
                step(graphed, out_g)         # first calls set up the library outside any capture
            else:
                if graph is None:
                    torch.cuda.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph):
                        step(graphed, out_g)  # recorded, not run
                graph.replay()
            torch.cuda.synchronize()
            for l in range(L):
                assert torch.equal(out_g[l], out_e[l]), f"layer {l} chunk {c}: graph differs from eager"
            if c in (1, switch, n_chunks - 1):
                for l in range(L):
                    q, k, v = host[l]
                    n = (c + 1) * Tq
                    kh = np.zeros((n, H, D))
                    vh = np.zeros((n, H, D))
                    for f, vals in model.held_frames(l, 0).items():
                        kh[f * T:(f + 1) * T] = vals
                    for f, vals in model.held_frames(l, 1).items():
                        vh[f * T:(f + 1) * T] = vals
                    kh[c * Tq:] = bf16_bits_to_f64(k)
                    vh[c * Tq:] = bf16_bits_to_f64(v)
                    ref = oracle.sink_window_attention(q, kh, vh, c, S, W, F, T)
                    assert_attn_close(dev_to_f64(out_g[l]), ref, f"graph layer {l} chunk {c}")
            for l in range(L):
                model.append(l, host[l][1], host[l][2])
        for l in range(L):
            assert ll.ll_kv_cache_export(graphed, l) == ll.ll_kv_cache_export(eager, l) == model.export(l)
            # the host lost track of p at the capture; info reads the device counter
            assert ll.ll_kv_cache_info(graphed, l)[0] == n_chunks * F
            assert ll.ll_kv_cache_info(eager, l)[0] == n_chunks * F
        assert ll.ll_debug_status(graphed) == 0 and ll.ll_debug_status(eager) == 0
        del graph
    finally:
        eager.close()
        graphed.close()


def test_recache_range_is_checked_on_device_after_capture():
    import torch
    import kv_cache_attention_ll_b200 as ll
    L, H, D, T, F, S, W = 1, 1, 64, 4, 3, 3, 6
    Tq = F * T
    cache = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    try:
        x = torch.randn(Tq, H, D, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(x)
        buf = torch.randn((S + W) * T, H, D, device="cuda").to(torch.bfloat16)
        ll.ll_attn_sink_window(x, x, x, cache, 0, out)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            ll.ll_kv_append(cache, 0, x, x)
        graph.replay()                      # p: 0 -> 3 frames (the sink), window empty
        assert ll.ll_kv_cache_info(cache, 0)[0] == F
        before = ll.ll_kv_cache_export(cache, 0)
        # frames 0..3 are not all held (only the 3 sink frames are): refused on the device
        ll.ll_kv_recache_write(cache, 0, buf, buf, 0, 4)
        torch.cuda.synchronize()
        assert ll.ll_kv_cache_export(cache, 0) == before
        word = ll.ll_debug_status(cache, clear=True)
        assert word & 0xFF == 2 and (word >> 8) & 0xFF == 2     # ERR_RANGE from the scatter kernel
        assert ll.ll_debug_status(cache) == 0
        # in range: written
        ll.ll_kv_recache_write(cache, 0, buf, buf, 0, 3)
        torch.cuda.synchronize()
        assert ll.ll_kv_cache_export(cache, 0) != before
        assert ll.ll_debug_status(cache) == 0
        # the host still rejects what no layer can hold
        with pytest.raises(ll.LLError):
            ll.ll_kv_recache_write(cache, 0, buf, buf, 0, S + W + 1)
        del graph
    finally:
        cache.close()
