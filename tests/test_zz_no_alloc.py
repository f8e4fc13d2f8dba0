"""The no-allocation entry point ll_attn_sink_window_noalloc.

Some callers cannot call cudaMalloc: code whose device memory belongs to a host
framework's pool that forbids libraries from allocating, or code on a
latency-critical path that cannot afford cudaMalloc's implicit device
synchronisation. For them ll_attn_sink_window_noalloc computes the attention of
a quantised cache layer that the caller holds in its own memory, using a static
device array of the library as its scratch.

Here a regular cache (FP8, then NVFP4) supplies the bytes: each layer is
exported, copied into caller-owned device buffers, and the no-allocation call
must give the same output as ll_attn_sink_window on the cache, on two calls in
a row (the scratch keeps the previous call's contents, which must not leak into
the next). This file is collected last so that a run stopping at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest

from seeded_inputs import chunk_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv_dtype", ["fp8", "nvfp4"])
def test_noalloc_matches_cache_entry_point_on_two_calls(kv_dtype):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    H, D, T, F, S, W = 2, 128, 64, 3, 3, 6
    Tq = F * T
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W, kv_dtype)
    try:
        for c in range(4):
            _, k, v = chunk_qkv(61, 0, c, Tq, H, D)
            ll.ll_kv_append(cache, 0, to_dev(k), to_dev(v))
        slots = (S + W) * T
        data_bytes = 2 * H * slots * (D if kv_dtype == "fp8" else D // 2)
        for call in range(2):                       # two calls in a row, different cache states
            c = 4 + call
            q, k, v = (to_dev(x) for x in chunk_qkv(61, 0, c, Tq, H, D))
            ref = torch.empty_like(q)
            ll.ll_attn_sink_window(q, k, v, cache, 0, ref)
            raw = ll.ll_kv_cache_export(cache, 0)
            codes = torch.frombuffer(bytearray(raw[:data_bytes]), dtype=torch.uint8).cuda()
            scales = torch.frombuffer(bytearray(raw[data_bytes:]), dtype=torch.uint8).cuda()
            out = torch.empty_like(q)
            p = ll.ll_kv_cache_info(cache, 0)[0]
            ll.ll_attn_sink_window_noalloc(q, k, v, codes, scales, kv_dtype, H, D, T, F, S, W, p, out)
            torch.cuda.synchronize()
            assert_attn_close(dev_to_f64(out), dev_to_f64(ref), f"{kv_dtype} call {call}")
            ll.ll_kv_append(cache, 0, k, v)
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()


@pytest.mark.parametrize("kv_dtype", ["fp8", "nvfp4"])
def test_noalloc_partly_filled_caches_after_a_larger_call(kv_dtype):
    """A call on a full cache of one geometry fills the scratch; the calls that
    follow use another geometry (head_dim 64, three heads, 40 tokens per frame)
    on caches that are only partly filled (3 and then 6 of 9 frames held: 120
    and 240 keys, neither a multiple of the 128-key tile), so the tile rows
    past the held keys must be cleared of the earlier call's contents. Each
    output equals ll_attn_sink_window's on a cache holding the same bytes, and
    the no-allocation path's status word stays clear."""
    import torch
    import kv_cache_attention_ll_b200 as ll
    _noalloc_vs_cache(ll, torch, kv_dtype, H=2, D=128, T=64, F=3, S=3, W=6, seed=62, frames=[12])
    _noalloc_vs_cache(ll, torch, kv_dtype, H=3, D=64, T=40, F=3, S=3, W=6, seed=63, frames=[3, 6])
    _noalloc_vs_cache(ll, torch, kv_dtype, H=2, D=128, T=64, F=3, S=3, W=6, seed=64, frames=[0, 3])
    assert ll.ll_noalloc_debug_status() == 0


def _noalloc_vs_cache(ll, torch, kv_dtype, H, D, T, F, S, W, seed, frames):
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    Tq = F * T
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W, kv_dtype)
    slots = (S + W) * T
    data_bytes = 2 * H * slots * (D if kv_dtype == "fp8" else D // 2)
    try:
        c = 0
        for want in frames:
            while ll.ll_kv_cache_info(cache, 0)[0] < want:
                _, k, v = chunk_qkv(seed, 0, c, Tq, H, D)
                ll.ll_kv_append(cache, 0, to_dev(k), to_dev(v))
                c += 1
            q, k, v = (to_dev(x) for x in chunk_qkv(seed, 0, c, Tq, H, D))
            ref = torch.empty_like(q)
            ll.ll_attn_sink_window(q, k, v, cache, 0, ref)
            raw = ll.ll_kv_cache_export(cache, 0)
            codes = torch.frombuffer(bytearray(raw[:data_bytes]), dtype=torch.uint8).cuda()
            scales = torch.frombuffer(bytearray(raw[data_bytes:]), dtype=torch.uint8).cuda()
            out = torch.empty_like(q)
            p = ll.ll_kv_cache_info(cache, 0)[0]
            ll.ll_attn_sink_window_noalloc(q, k, v, codes, scales, kv_dtype, H, D, T, F, S, W, p, out)
            torch.cuda.synchronize()
            assert_attn_close(dev_to_f64(out), dev_to_f64(ref), f"{kv_dtype} H{H} D{D} T{T} p{p}")
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()


def test_noalloc_rejects_geometry_beyond_the_scratch():
    import torch
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    # Wan-1.3B layer: 2 * 12 heads * 18720 slots * 128 * 2 bytes = 115 MB > the static scratch
    st = lib.ll_attn_sink_window_noalloc(p, p, p, p, p, ll.LL_KV_FP8_E4M3, 12, 128, 1560, 3, 3, 9, 12,
                                         p + 4096, None)
    assert st == ll.LL_ERR_INVALID_ARG
    # a bf16 cache has no scratch to dequantise into: not this entry point's job
    st = lib.ll_attn_sink_window_noalloc(p, p, p, p, p, ll.LL_KV_BF16, 1, 64, 4, 1, 1, 1, 2, p + 4096, None)
    assert st == ll.LL_ERR_INVALID_ARG
