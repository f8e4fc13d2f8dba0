"""Random sequences of every cache operation against the oracle.

Each case draws a small geometry (with or without a shot sink), a storage
format and a cache kind (the plain ring, or the ring with spare slots for the
fused call), then runs chunks in which shot starts (with or without a
window restart), recaches of random held ranges of one or all layers,
attention and append (separate or fused) happen at random. After every
operation the cache bytes of every layer must equal the oracle's cache model,
and every attention output must match the fp64 oracle over the frames that the
frame-classification definition names. At the end the canary bytes that guard
every region of the cache allocation must be untouched (no stray writes)."""
import random

import numpy as np
import pytest

import oracle
from oracle.attention import multishot_visible_frames
from seeded_inputs import chunk_qkv, bf16_bits_to_f64, recache_kv, mix_seed

pytestmark = pytest.mark.gpu

GEOMS = [  # H, D, T, F, G, Ss, W
    (2, 64, 16, 3, 3, 0, 6),
    (1, 128, 40, 2, 1, 2, 3),
    (2, 128, 24, 1, 2, 1, 4),
    (1, 64, 33, 3, 0, 3, 2),
]


@pytest.mark.parametrize("seed", range(12))
def test_random_operation_sequence(seed):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    rng = random.Random(mix_seed(seed, 4242))
    H, D, T, F, G, Ss, W = GEOMS[seed % len(GEOMS)]
    kv_dtype = ("bf16", "fp8", "nvfp4")[seed % 3]
    kind = "fused" if (seed // 3) % 2 else "plain"          # seeds 3-5 and 9-11: fused caches
    L, Tq, n = 2, F * T, 12
    fused = kind == "fused"
    model = oracle.CacheModel(L, H, D, T, F, G, W, kv_dtype, shot_sink_frames=Ss,
                              ring_slots=W + F if fused else None)
    if fused:
        cache = ll.ll_kv_cache_create_fused(L, H, D, T, F, G, Ss, W, kv_dtype)
    else:
        cache = ll.ll_kv_cache_create_multishot(L, H, D, T, F, G, Ss, W, kv_dtype)
    shots = {}
    try:
        for c in range(n):
            if c > 0 and rng.random() < 0.25:
                clear = rng.random() < 0.5
                shots[c] = clear
                ll.ll_kv_shot_begin(cache, -1, clear)
                model.shot_begin(-1, clear)
            if c > 1 and rng.random() < 0.3 and model.n_held(0) > 0:
                held = model.n_held(0)
                first = rng.randrange(held)
                num = rng.randint(1, held - first)
                layer = rng.choice([-1, 0, 1])
                lp = L if layer < 0 else 1
                kn = np.stack([recache_kv(300 + seed, l, c, num * T, H, D)[0] for l in range(lp)])
                vn = np.stack([recache_kv(300 + seed, l, c, num * T, H, D)[1] for l in range(lp)])
                ll.ll_kv_recache_write(cache, layer, to_dev(kn), to_dev(vn), first, num)
                model.recache_write(layer, kn, vn, first, num)
            vis = multishot_visible_frames(c, G, Ss, W, F, sorted(shots.items()))
            for l in range(L):
                q, k, v = chunk_qkv(300 + seed, l, c, Tq, H, D)
                dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
                out = torch.empty_like(dq)
                if fused and rng.random() < 0.7:
                    ll.ll_attn_sink_window_append(dq, dk, dv, cache, l, out)
                else:
                    ll.ll_attn_sink_window(dq, dk, dv, cache, l, out)
                    ll.ll_kv_append(cache, l, dk, dv)
                n_hist = (c + 1) * Tq
                kh = np.zeros((n_hist, H, D))
                vh = np.zeros((n_hist, H, D))
                for f, vals in model.held_frames(l, 0).items():
                    kh[f * T:(f + 1) * T] = vals
                for f, vals in model.held_frames(l, 1).items():
                    vh[f * T:(f + 1) * T] = vals
                kh[c * Tq:] = bf16_bits_to_f64(k)
                vh[c * Tq:] = bf16_bits_to_f64(v)
                torch.cuda.synchronize()
                ref = oracle.sink_window_attention(q, kh, vh, c, 0, 0, F, T, visible_frames=vis)
                assert_attn_close(dev_to_f64(out), ref, f"seed {seed} chunk {c} layer {l}")
                model.append(l, k, v)
            for l in range(L):
                assert ll.ll_kv_cache_export(cache, l) == model.export(l), f"seed {seed} chunk {c} layer {l}"
                assert ll.ll_kv_cache_held(cache, l) == model.held3(l)
        assert ll.ll_debug_status(cache) == 0
        assert ll.ll_debug_check_canaries(cache) == -1, "a guard byte around the cache regions changed"
    finally:
        cache.close()
