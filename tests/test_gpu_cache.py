"""GPU parity of the append/evict and recache kernels against the cache oracle:
the exported cache bytes must equal the oracle's byte for byte (bf16, FP8 and
NVFP4 formats), through long rollouts, early chunks, window shorter than a
chunk, no sink, sink-only, single-layer and all-layer recache."""
import numpy as np
import pytest

from oracle import CacheModel
from seeded_inputs import chunk_qkv, recache_kv, mix_seed, bf16_normal

pytestmark = pytest.mark.gpu


def _ll():
    import kv_cache_attention_ll_b200 as ll
    return ll


CASES = [
    # L, H, D, T, F, S, W
    (2, 2, 64, 16, 3, 3, 6),      # config-0 geometry, two layers
    (1, 3, 128, 7, 3, 3, 9),      # head_dim 128, odd tokens per frame
    (2, 1, 64, 5, 3, 1, 2),       # window shorter than a chunk
    (1, 2, 128, 4, 2, 0, 4),      # no sink
    (1, 2, 64, 3, 2, 3, 0),       # sink only
    (1, 1, 128, 2, 1, 2, 3),      # one frame per chunk
]


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("L,H,D,T,F,S,W", CASES)
def test_cache_bytes_match_oracle(kv_dtype, L, H, D, T, F, S, W):
    import torch
    from gpu_util import to_dev
    ll = _ll()
    cfg_id = hash((L, H, D, T, F, S, W)) & 0xFFFF
    model = CacheModel(L, H, D, T, F, S, W, kv_dtype)
    cache = ll.ll_kv_cache_create(L, H, D, T, F, S, W, kv_dtype)
    Tq = F * T
    n_chunks = 9
    switch = 5
    try:
        for c in range(n_chunks):
            for l in range(L):
                _, k, v = chunk_qkv(cfg_id, l, c, Tq, H, D)
                model.append(l, k, v)
                ll.ll_kv_append(cache, l, to_dev(k), to_dev(v))
            if c == switch:
                s, w = model.held(0)
                # all layers, whole held context
                kn = np.stack([recache_kv(cfg_id, l, 0, (s + w) * T, H, D)[0] for l in range(L)])
                vn = np.stack([recache_kv(cfg_id, l, 0, (s + w) * T, H, D)[1] for l in range(L)])
                model.recache_write(-1, kn, vn, 0, s + w)
                ll.ll_kv_recache_write(cache, -1, to_dev(kn), to_dev(vn), 0, s + w)
                # one layer, a sub-range (window part when there is one)
                first, num = (S, w) if w > 0 else (0, s)
                kn1 = recache_kv(cfg_id, L - 1, 1, num * T, H, D)[0][None]
                vn1 = recache_kv(cfg_id, L - 1, 1, num * T, H, D)[1][None]
                model.recache_write(L - 1, kn1, vn1, first, num)
                ll.ll_kv_recache_write(cache, L - 1, to_dev(kn1), to_dev(vn1), first, num)
            torch.cuda.synchronize()
            for l in range(L):
                got = ll.ll_kv_cache_export(cache, l)
                want = model.export(l)
                assert len(got) == len(want)
                if got != want:
                    a = np.frombuffer(got, np.uint8)
                    b = np.frombuffer(want, np.uint8)
                    bad = np.nonzero(a != b)[0]
                    pytest.fail(f"chunk {c} layer {l}: {len(bad)} bytes differ, first at {bad[0]} "
                                f"(got {a[bad[0]]:#x}, want {b[bad[0]]:#x})")
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_recache_equals_fresh_append_on_gpu():
    """Prompt switch at chunk 20 + recache of the held frames == a fresh cache
    whose history had those K/V all along (compared device bytes to device bytes)."""
    import torch
    from gpu_util import to_dev
    ll = _ll()
    L, H, D, T, F, S, W = 2, 2, 64, 8, 3, 3, 9
    Tq = F * T
    switch = 20
    p = switch * F
    held = list(range(S)) + list(range(p - W, p))
    kn = np.stack([recache_kv(7, l, 0, len(held) * T, H, D)[0] for l in range(L)])
    vn = np.stack([recache_kv(7, l, 0, len(held) * T, H, D)[1] for l in range(L)])
    a = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    b = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    try:
        for c in range(switch):
            for l in range(L):
                _, k, v = chunk_qkv(7, l, c, Tq, H, D)
                ll.ll_kv_append(a, l, to_dev(k), to_dev(v))
                k2, v2 = k.copy(), v.copy()
                for i, fr in enumerate(held):
                    if fr // F == c:
                        t0 = (fr % F) * T
                        k2[t0:t0 + T] = kn[l, i * T:(i + 1) * T]
                        v2[t0:t0 + T] = vn[l, i * T:(i + 1) * T]
                ll.ll_kv_append(b, l, to_dev(k2), to_dev(v2))
        ll.ll_kv_recache_write(a, -1, to_dev(kn), to_dev(vn), 0, len(held))
        torch.cuda.synchronize()
        for l in range(L):
            assert ll.ll_kv_cache_export(a, l) == ll.ll_kv_cache_export(b, l)
    finally:
        a.close()
        b.close()


def test_constant_footprint_over_long_rollout():
    """320 chunks of attention + append with a recache every 40: no allocation
    and no change of free device memory after create."""
    import torch
    from gpu_util import to_dev
    ll = _ll()
    L, H, D, T, F, S, W = 1, 2, 128, 16, 3, 3, 9
    Tq = F * T
    cache = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    try:
        q, k, v = (to_dev(x) for x in chunk_qkv(3, 0, 0, Tq, H, D))
        out = torch.empty_like(q)
        kn = to_dev(bf16_normal(mix_seed(3, 3), ((S + W) * T, H, D)))
        torch.cuda.synchronize()
        n_alloc = ll.ll_allocation_count()
        free0, _ = torch.cuda.mem_get_info()
        for c in range(320):
            ll.ll_attn_sink_window(q, k, v, cache, 0, out)
            ll.ll_kv_append(cache, 0, k, v)
            if c % 40 == 39:
                ll.ll_kv_recache_write(cache, 0, kn, kn, 0, S + W)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert ll.ll_allocation_count() == n_alloc
        assert free1 == free0
        assert ll.ll_kv_cache_info(cache, 0)[0] == 320 * F
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()


def test_invalid_recache_ranges_are_rejected():
    ll = _ll()
    import torch
    cache = ll.ll_kv_cache_create(2, 1, 64, 4, 3, 3, 6)
    try:
        buf = torch.zeros(2 * 9 * 4 * 64, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(ll.LLError):          # nothing held yet
            ll.ll_kv_recache_write(cache, 0, buf, buf, 0, 1)
        ll.ll_kv_append(cache, 0, buf, buf)
        with pytest.raises(ll.LLError):          # layer 1 holds nothing yet
            ll.ll_kv_recache_write(cache, -1, buf, buf, 0, 1)
        with pytest.raises(ll.LLError):          # past the held frames
            ll.ll_kv_recache_write(cache, 0, buf, buf, 2, 2)
        ll.ll_kv_recache_write(cache, 0, buf, buf, 0, 3)
        with pytest.raises(ll.LLError):          # misaligned pointer
            ll.ll_kv_append(cache, 0, buf.data_ptr() + 2, buf.data_ptr())
    finally:
        cache.close()


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "nvfp4"])
def test_append_of_all_layers_in_one_launch(kv_dtype):
    """ll_kv_append(cache, -1, k[L], v[L]) stores every layer's chunk in one
    launch and advances every layer's counters: the cache bytes equal the
    oracle's per-layer appends, with shot starts in between."""
    import torch
    from gpu_util import to_dev
    ll = _ll()
    L, H, D, T, F, G, Ss, W = 3, 2, 128, 20, 3, 2, 1, 4
    model = CacheModel(L, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss)
    cache = ll.ll_kv_cache_create_multishot(L, H, D, T, F, G, Ss, W, kv_dtype)
    try:
        for c in range(7):
            if c in (3, 5):
                ll.ll_kv_shot_begin(cache, -1, c == 5)
                model.shot_begin(-1, c == 5)
            ks = np.stack([chunk_qkv(400, l, c, F * T, H, D)[1] for l in range(L)])
            vs = np.stack([chunk_qkv(400, l, c, F * T, H, D)[2] for l in range(L)])
            ll.ll_kv_append(cache, -1, to_dev(ks), to_dev(vs))
            for l in range(L):
                model.append(l, ks[l], vs[l])
            torch.cuda.synchronize()
            for l in range(L):
                assert ll.ll_kv_cache_export(cache, l) == model.export(l), f"chunk {c} layer {l}"
                assert ll.ll_kv_cache_info(cache, l)[0] == (c + 1) * F
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()
