"""GPU parity of ll_attn_sink_window on FP8 and NVFP4 caches.

The library quantises on append (bit-exact against the oracle, see
test_gpu_cache.py). Each attention call first converts the layer's held codes
into a bf16 view of the cache (a separate pass of the same call), and the
attention kernel reads that view. The oracle
attends over the exactly dequantised held frames (E4M3 code x power-of-two row scale,
or E2M1 code x E4M3 block scale, in fp64) plus the chunk's own bf16 K/V, with
its explicit sink + window + block-causal mask.

Bound: the standard max-abs 1e-2 and relative-L2 5e-3. The dequantised values
of both formats are exact in bf16 (NVFP4: at most 6 significant bits; FP8: a
4-bit code times a power-of-two row scale), so the view holds the oracle's
values and the kernel's error budget is the bf16 one; the Wan-shape test
checks FP8 against a bf16 cache on the same inputs."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_qkv, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


def _rollout(kv_dtype, cfg_id, H, D, T, F, S, W, n_chunks, check, rows_per_head=None, vs_unquantised=False):
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close, attn_errors, sample_rows
    Tq = F * T
    model = oracle.CacheModel(1, H, D, T, F, S, W, kv_dtype)
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W, kv_dtype)
    results = []
    raw_k, raw_v = [], []        # the unquantised history, for the reported comparison
    try:
        for c in range(n_chunks):
            q, k, v = chunk_qkv(cfg_id, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            if c in check:
                # history as the oracle sees it: held frames dequantised, the own
                # chunk in bf16; frames no longer held are invisible (left zero)
                n = (c + 1) * Tq
                kh = np.zeros((n, H, D))
                vh = np.zeros((n, H, D))
                for f, vals in model.held_frames(0, 0).items():
                    kh[f * T:(f + 1) * T] = vals
                for f, vals in model.held_frames(0, 1).items():
                    vh[f * T:(f + 1) * T] = vals
                kh[c * Tq:] = bf16_bits_to_f64(k)
                vh[c * Tq:] = bf16_bits_to_f64(v)
                torch.cuda.synchronize()
                got = dev_to_f64(out)
                rows = None if rows_per_head is None else sample_rows(Tq, rows_per_head, cfg_id * 77 + c)
                ref = oracle.sink_window_attention(q, kh, vh, c, S, W, F, T, rows=rows)
                g = got if rows is None else got[rows]
                results.append((c, *assert_attn_close(g, ref, f"{kv_dtype} chunk {c}")))
                if vs_unquantised:
                    # the same attention over the bf16 values before quantisation
                    ref_bf16 = oracle.sink_window_attention(q, np.concatenate(raw_k + [k]),
                                                            np.concatenate(raw_v + [v]), c, S, W, F, T, rows=rows)
                    results[-1] += attn_errors(g, ref_bf16)
            if vs_unquantised:
                raw_k.append(k)
                raw_v.append(v)
            model.append(0, k, v)
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()
    return results


@pytest.mark.parametrize("kv_dtype", ["fp8", "nvfp4"])
def test_quantised_config0_all_chunks(kv_dtype):
    """Tiny reference geometry (head_dim 64), all 8 chunks."""
    _rollout(kv_dtype, 40, H=2, D=64, T=16, F=3, S=3, W=6, n_chunks=8, check=set(range(8)))


@pytest.mark.parametrize("kv_dtype", ["fp8", "nvfp4"])
@pytest.mark.parametrize("H,D,T,F,S,W,n", [
    (3, 128, 50, 3, 2, 5, 7),     # two query tiles, ragged; cache not a multiple of 128
    (2, 128, 40, 3, 3, 0, 5),     # sink only
    (1, 64, 129, 1, 2, 3, 7),     # one frame per chunk, one-row tail tile
])
def test_quantised_odd_shapes(kv_dtype, H, D, T, F, S, W, n):
    _rollout(kv_dtype, hash((H, D, T, F, S, W)) & 0xFFF, H, D, T, F, S, W, n, check=set(range(n)))


# Error of quantised-cache attention against attention over the unquantised bf16
# history: reported, not a parity bound (it is the format's own error). The
# sanity ceilings only catch a broken scale: N(0,1) inputs give 2.6 % (FP8)
# and 9.5 % (NVFP4) relative L2 error in the cached values themselves, and
# attention averages part of it away.
UNQUANTISED_CEILING = {"fp8": 0.05, "nvfp4": 0.2}


@pytest.mark.parametrize("kv_dtype", ["fp8", "nvfp4"])
def test_quantised_wan_shape_sampled_rows(kv_dtype):
    """Wan-1.3B single-layer shape, steady state (chunk 5 holds 12 cached frames)."""
    res = _rollout(kv_dtype, 41, H=12, D=128, T=1560, F=3, S=3, W=9, n_chunks=6, check={1, 5}, rows_per_head=256,
                   vs_unquantised=True)
    assert len(res) == 2
    for c, _, _, max_abs_q, rel_q in res:
        print(f"{kv_dtype} chunk {c}: vs unquantised bf16 attention max_abs={max_abs_q:.3e} rel_l2={rel_q:.3e}")
        assert rel_q <= UNQUANTISED_CEILING[kv_dtype]


def test_fp8_error_matches_the_bf16_path_at_the_wan_shape():
    """The same Wan-shape rollout on a bf16 cache and on an FP8 cache, each
    checked on the same sampled rows against the oracle over what that cache
    holds (bf16 values; FP8 codes x power-of-two scales, exact in bf16). The
    FP8 view therefore holds the oracle's values and the kernel rounds where
    the bf16 path does (the probabilities and the output to bf16): the errors
    must be of the same size, within 25 % (the two rollouts attend to
    different values, so their rounding errors differ by chance)."""
    fp8 = _rollout("fp8", 42, H=12, D=128, T=1560, F=3, S=3, W=9, n_chunks=6, check={5}, rows_per_head=256)
    bf16 = _rollout("bf16", 42, H=12, D=128, T=1560, F=3, S=3, W=9, n_chunks=6, check={5}, rows_per_head=256)
    (_, max_f, rel_f), (_, max_b, rel_b) = fp8[0], bf16[0]
    print(f"Wan shape chunk 5: fp8 max_abs={max_f:.3e} rel_l2={rel_f:.3e}; bf16 max_abs={max_b:.3e} rel_l2={rel_b:.3e}")
    assert rel_f <= 1.25 * rel_b and max_f <= 1.5 * max_b
