"""GPU parity of ll_attn_sink_window against the fp64 oracle on the same seeded
bf16 inputs: max-abs error <= 1e-2 and relative L2 error <= 5e-3.

Each rollout calls attention and then append for every chunk, exactly as a
generator would, and checks chosen chunks against the oracle, which sees the
full frame history and builds the sink + window + block-causal mask itself."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_tensor, bf16_bits_to_f64, KIND_Q, KIND_K, KIND_V

pytestmark = pytest.mark.gpu


def _rollout(cfg_id, H, D, T, F, S, W, n_chunks, check, rows_per_head=None, layers=1, layer=0, qk_scale=1.0):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, assert_attn_close_derived, sample_rows
    Tq = F * T
    cache = ll.ll_kv_cache_create(layers, H, D, T, F, S, W)
    hk, hv = [], []
    results = []
    try:
        for c in range(n_chunks):
            q = chunk_tensor(KIND_Q, cfg_id, layer, c, Tq, H, D, qk_scale)
            k = chunk_tensor(KIND_K, cfg_id, layer, c, Tq, H, D, qk_scale)
            v = chunk_tensor(KIND_V, cfg_id, layer, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, layer, out)
            ll.ll_kv_append(cache, layer, dk, dv)
            hk.append(k)
            hv.append(v)
            if c in check:
                torch.cuda.synchronize()
                got = dev_to_f64(out)
                rows = None if rows_per_head is None else sample_rows(Tq, rows_per_head, cfg_id * 1000 + c)
                ref = oracle.sink_window_attention(q, np.concatenate(hk), np.concatenate(hv), c, S, W, F, T,
                                                   rows=rows)
                g = got if rows is None else got[rows]
                if qk_scale == 1.0:
                    results.append((c, *assert_attn_close(g, ref, f"chunk {c}")))
                else:
                    vmax = float(np.abs(bf16_bits_to_f64(np.concatenate(hv))).max())
                    assert_attn_close_derived(g, ref, vmax, f"chunk {c}")
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()
    return results


def test_config0_all_chunks():
    """Tiny reference: 2 heads, head_dim 64, 16 tokens/frame, chunk 3, sink 3, window 6, 8 chunks."""
    _rollout(0, H=2, D=64, T=16, F=3, S=3, W=6, n_chunks=8, check=set(range(8)))


@pytest.mark.parametrize("H,D,T,F,S,W,n", [
    (3, 128, 50, 3, 2, 5, 7),     # two query tiles, ragged; cache not a multiple of 128
    (2, 64, 43, 2, 0, 4, 6),      # no sink; Tq < 128
    (1, 128, 30, 3, 1, 2, 6),     # window shorter than a chunk
    (2, 128, 40, 3, 3, 0, 5),     # sink only
    (2, 64, 129, 1, 2, 3, 7),     # one frame per chunk, Tq = 129 (one-row tail tile)
    (1, 128, 128, 2, 3, 9, 9),    # exact 128-multiples everywhere
])
def test_odd_shapes_all_chunks(H, D, T, F, S, W, n):
    _rollout(hash((H, D, T, F, S, W)) & 0xFFF, H, D, T, F, S, W, n, check=set(range(n)))


def test_window_covering_history_is_full_causal():
    """With W >= all history the kernel computes plain block-causal attention."""
    _rollout(11, H=2, D=128, T=24, F=3, S=3, W=30, n_chunks=8, check={0, 3, 7})


def test_wan_shape_sampled_rows():
    """Wan-1.3B single-layer shape: 12 heads, head_dim 128, 1560 tokens/frame,
    chunk 3, sink 3, window 9; chunks 0 (own only), 1 (sink only), 2, 5 (full cache)."""
    res = _rollout(1, H=12, D=128, T=1560, F=3, S=3, W=9, n_chunks=6, check={0, 1, 2, 5}, rows_per_head=384)
    assert len(res) == 4


def test_full_causal_largest_history_sampled_rows():
    """The longest history the pages measure: their full-causal comparison runs
    40 chunks (117 latent frames of 1560 tokens) with every earlier frame
    visible (sink 3 + window 114). Chunk 39 attends 187200 keys (117 cached
    frames and its own 3), 8 times the steady-state sink + window count. Two
    heads of the Wan frame size (heads are independent; the key count is what
    grows); chunk 13 (42 cached frames) and chunk 39, sampled rows with the
    ragged last query tile."""
    res = _rollout(41, H=2, D=128, T=1560, F=3, S=3, W=114, n_chunks=40, check={13, 39}, rows_per_head=256)
    assert len(res) == 2


def test_large_logits_rescale_path():
    """Q and K scaled by 4 so that logits span tens of units: exercises the lazy
    rescale of O. The softmax is peaked here, so the max-abs bound is the one
    derived from bf16 rounding (see gpu_util.assert_attn_close_derived)."""
    _rollout(21, H=2, D=128, T=64, F=3, S=3, W=6, n_chunks=6, check={2, 5}, qk_scale=4.0)


def test_large_max_jump_rescale_path():
    """The chunk's own keys scaled by 40: its tiles come after the cache tiles and
    raise a row's maximum logit far above the running reference maximum (much
    more than the lazy-rescale threshold of 8 in log2 units), so the reference
    moves up and the partial output and row sum are rescaled before those
    tiles are added. The softmax is peaked, so the derived bf16 bound applies."""
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close_derived
    from seeded_inputs import f32_to_bf16_bits
    H, D, T, F, S, W = 2, 128, 64, 3, 3, 6
    Tq = F * T
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W)
    hk, hv = [], []
    try:
        for c in range(5):
            q = chunk_tensor(KIND_Q, 31, 0, c, Tq, H, D)
            k = chunk_tensor(KIND_K, 31, 0, c, Tq, H, D)
            v = chunk_tensor(KIND_V, 31, 0, c, Tq, H, D)
            if c >= 3:
                k = f32_to_bf16_bits((bf16_bits_to_f64(k) * 40.0).astype(np.float32))
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            hk.append(k)
            hv.append(v)
            if c >= 3:
                torch.cuda.synchronize()
                ref = oracle.sink_window_attention(q, np.concatenate(hk), np.concatenate(hv), c, S, W, F, T)
                vmax = float(np.abs(bf16_bits_to_f64(np.concatenate(hv))).max())
                assert_attn_close_derived(dev_to_f64(out), ref, vmax, f"chunk {c}")
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()
