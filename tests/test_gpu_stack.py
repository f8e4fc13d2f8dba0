"""Full-size parity in the launch configuration the benchmark times: the
30-layer Wan-1.3B-shaped stack (12 heads, head_dim 128, 1560 tokens per frame,
chunk 3, sink 3, window 9), attention then append for every layer of every
chunk, and a prompt switch before chunk 20 that rewrites the sink + window of
all 30 layers in one ll_kv_recache_write call.

One layer (the last) carries seeded host inputs and is checked against the
fp64 oracle on sampled query rows at chunks 0, 1, 4 (cache full), 20 (first
chunk after the recache) and 21; the cache bytes of that layer are checked
against the cache oracle at the end. The other layers receive device-random
inputs: layers are independent, they only have to run."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_qkv, recache_kv, bf16_bits_to_f64

pytestmark = pytest.mark.gpu

L, H, D, T, F, S, W = 30, 12, 128, 1560, 3, 3, 9
TQ = F * T
CHECK_LAYER = L - 1
SWITCH = 20
CHECKS = {0, 1, 4, 20, 21}


def test_wan_stack_with_prompt_switch():
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, sample_rows
    torch.manual_seed(3)
    model = oracle.CacheModel(1, H, D, T, F, S, W)
    cache = ll.ll_kv_cache_create(L, H, D, T, F, S, W)
    try:
        other = [torch.randn(3, TQ, H, D, device="cuda").to(torch.bfloat16) for _ in range(2)]
        out = torch.empty(TQ, H, D, device="cuda", dtype=torch.bfloat16)
        for c in range(max(CHECKS) + 1):
            if c == SWITCH:
                # prompt switch: new K/V for the held frames (sink + window) of all layers
                n_held = S + W
                kn = torch.randn(L, n_held * T, H, D, device="cuda").to(torch.bfloat16)
                vn = torch.randn(L, n_held * T, H, D, device="cuda").to(torch.bfloat16)
                k_new, v_new = recache_kv(3, CHECK_LAYER, 0, n_held * T, H, D)
                kn[CHECK_LAYER].copy_(to_dev(k_new))
                vn[CHECK_LAYER].copy_(to_dev(v_new))
                ll.ll_kv_recache_write(cache, -1, kn, vn, 0, n_held)
                model.recache_write(0, k_new[None], v_new[None], 0, n_held)
            q, k, v = chunk_qkv(3, CHECK_LAYER, c, TQ, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            for l in range(L):
                if l == CHECK_LAYER:
                    ll.ll_attn_sink_window(dq, dk, dv, cache, l, out)
                    ll.ll_kv_append(cache, l, dk, dv)
                else:
                    t = other[l % 2]
                    ll.ll_attn_sink_window(t[0], t[1], t[2], cache, l, torch.empty_like(out))
                    ll.ll_kv_append(cache, l, t[1], t[2])
            if c in CHECKS:
                n = (c + 1) * TQ
                kh = np.zeros((n, H, D))
                vh = np.zeros((n, H, D))
                for f, vals in model.held_frames(0, 0).items():
                    kh[f * T:(f + 1) * T] = vals
                for f, vals in model.held_frames(0, 1).items():
                    vh[f * T:(f + 1) * T] = vals
                kh[c * TQ:] = bf16_bits_to_f64(k)
                vh[c * TQ:] = bf16_bits_to_f64(v)
                torch.cuda.synchronize()
                rows = sample_rows(TQ, 128, 1000 + c)
                ref = oracle.sink_window_attention(q, kh, vh, c, S, W, F, T, rows=rows)
                assert_attn_close(dev_to_f64(out)[rows], ref, f"layer {CHECK_LAYER} chunk {c}")
            model.append(0, k, v)
        torch.cuda.synchronize()
        assert ll.ll_kv_cache_export(cache, CHECK_LAYER) == model.export(0)
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()
