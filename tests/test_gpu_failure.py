"""Failure detection on the GPU without faulting it: every in-kernel wait is
bounded. The self-test kernel waits on a barrier that nothing completes; after
the limit (about a second) it records the timeout in the cache's status word
and returns. The host reads LL_ERR_TIMEOUT, clears the word, and the same
context keeps working (an attention call afterwards is checked against the
oracle)."""
import numpy as np
import pytest

import oracle
from seeded_inputs import chunk_qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    import torch
    import kv_cache_attention_ll_b200 as ll
    from gpu_util import to_dev, dev_to_f64, assert_attn_close
    H, D, T, F, S, W = 2, 64, 16, 3, 3, 6
    Tq = F * T
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W)
    try:
        assert ll.ll_debug_status(cache) == 0
        ll.ll_debug_wait_selftest(cache)
        torch.cuda.synchronize()
        word = ll.ll_debug_status(cache, clear=True)
        assert word & 0xFF == 1                     # wait timed out
        assert (word >> 8) & 0xFF == 4              # reported by the self-test kernel
        assert ll.ll_debug_status(cache) == 0       # cleared
        hk, hv = [], []
        for c in range(3):
            q, k, v = chunk_qkv(9, 0, c, Tq, H, D)
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            hk.append(k)
            hv.append(v)
        torch.cuda.synchronize()
        ref = oracle.sink_window_attention(q, np.concatenate(hk), np.concatenate(hv), 2, S, W, F, T)
        assert_attn_close(dev_to_f64(out), ref, "after the timeout")
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()
