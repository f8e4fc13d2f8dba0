"""Head sharding through the existing entry points: P caches of H/P heads, fed
the heads' slices of the chunk, give bit for bit the outputs and cache planes
of one cache of H heads. Heads exchange nothing inside attention, append or
recache, so a rank that holds H/P heads after a sequence-parallel all-to-all
(LongLive-2.0 explainer, wmrh.cn, sec. 15.2) runs the same library calls."""
import numpy as np
import pytest

from seeded_inputs import chunk_qkv, recache_kv

pytestmark = pytest.mark.gpu


def _planes(raw: bytes, heads: int, kv_dtype: str):
    """One layer's export split into [2][heads][...] byte arrays: data, then scales."""
    b = np.frombuffer(raw, np.uint8)
    if kv_dtype == "bf16":
        return [b.reshape(2, heads, -1)]
    n_data = len(b) * 8 // 9
    return [b[:n_data].reshape(2, heads, -1), b[n_data:].reshape(2, heads, -1)]


@pytest.mark.parametrize("kv_dtype", ["bf16", "nvfp4"])
def test_head_sharded_caches_equal_one_full_cache(kv_dtype):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev
    H, D, T, F, S, W, P = 4, 128, 40, 3, 2, 4, 2
    Hp, Tq = H // P, F * T
    full = ll.ll_kv_cache_create(1, H, D, T, F, S, W, kv_dtype)
    shards = [ll.ll_kv_cache_create(1, Hp, D, T, F, S, W, kv_dtype) for _ in range(P)]
    try:
        for c in range(7):
            if c == 4:                                     # a prompt switch: recache every held frame
                n = sum(ll.ll_kv_cache_held(full, 0))
                kn, vn = recache_kv(41, 0, c, n * T, H, D)
                ll.ll_kv_recache_write(full, 0, to_dev(kn), to_dev(vn), 0, n)
                for r, sc in enumerate(shards):
                    hs = slice(r * Hp, (r + 1) * Hp)
                    ll.ll_kv_recache_write(sc, 0, to_dev(np.ascontiguousarray(kn[:, hs])),
                                           to_dev(np.ascontiguousarray(vn[:, hs])), 0, n)
            q, k, v = chunk_qkv(41, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, full, 0, out)
            ll.ll_kv_append(full, 0, dk, dv)
            for r, sc in enumerate(shards):
                hs = slice(r * Hp, (r + 1) * Hp)
                qr, kr, vr = (to_dev(np.ascontiguousarray(x[:, hs])) for x in (q, k, v))
                out_r = torch.empty_like(qr)
                ll.ll_attn_sink_window(qr, kr, vr, sc, 0, out_r)
                ll.ll_kv_append(sc, 0, kr, vr)
                torch.cuda.synchronize()
                assert torch.equal(out_r, out[:, hs]), f"chunk {c} shard {r}"
        # cache bytes, per head plane: K data, V data, then (NVFP4) K and V block
        # scales, D/2 : D/16 = 8 : 1 of the bytes
        full_parts = _planes(ll.ll_kv_cache_export(full, 0), H, kv_dtype)
        for r, sc in enumerate(shards):
            for got, want in zip(_planes(ll.ll_kv_cache_export(sc, 0), Hp, kv_dtype), full_parts):
                np.testing.assert_array_equal(got, want[:, r * Hp:(r + 1) * Hp])
        assert ll.ll_debug_status(full) == 0 and all(ll.ll_debug_status(sc) == 0 for sc in shards)
    finally:
        full.close()
        for sc in shards:
            sc.close()
