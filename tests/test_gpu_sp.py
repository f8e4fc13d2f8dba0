"""GPU tests of the head-sharded sequence-parallel step (LongLive-2.0
explainer, wmrh.cn, sec. 18.3 and 15.2).

* ll_sp_pack_heads / ll_sp_unpack_heads against the permutation they define,
  bit for bit, for several rank counts, head_dims and token counts;
* ll_sp_pack_heads_fp8 against the oracle's FP8 rows (codes and scales bit for
  bit) and ll_sp_dequant_fp8 against the oracle's exact dequantisation;
* P ranks emulated on one GPU by host threads, each with its own cache of H/P
  heads, running SequenceParallelAttention with the library's kernels; the
  all-to-all is done by device copies between the threads' buffers, with the
  threads meeting at a host barrier after a device synchronisation (no kernel
  waits for another). Each rank's outputs and cache bytes must equal, bit for
  bit, those of one unsharded cache fed the same chunks (with compress_kv: fed
  the chunks' FP8-rounded K and V), in bf16, FP8 and NVFP4 caches;
* the same step over a real NCCL process group of one rank."""
import threading

import numpy as np
import pytest

from oracle import quant
from seeded_inputs import chunk_qkv

pytestmark = pytest.mark.gpu


def _ll():
    import kv_cache_attention_ll_b200 as ll
    return ll


@pytest.mark.parametrize("P,H,D,tokens", [(1, 4, 64, 50), (2, 4, 128, 130), (3, 12, 128, 390), (4, 12, 64, 7),
                                          (6, 12, 128, 585)])
def test_pack_and_unpack_are_the_head_block_permutation(P, H, D, tokens):
    import torch
    from gpu_util import to_dev
    ll = _ll()
    _, x, _ = chunk_qkv(950, P, tokens, tokens, H, D)
    dx = to_dev(x)
    packed = torch.empty_like(dx)
    ll.ll_sp_pack_heads(dx, tokens, H, D, P, packed)
    back = torch.empty_like(dx)
    ll.ll_sp_unpack_heads(packed, tokens, H, D, P, back)
    torch.cuda.synchronize()
    want = x.reshape(tokens, P, H // P, D).transpose(1, 0, 2, 3).reshape(-1)
    got = packed.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got, want)
    assert np.array_equal(back.view(torch.int16).cpu().numpy().view(np.uint16), x)


@pytest.mark.parametrize("P,H,D,tokens", [(2, 4, 128, 130), (3, 6, 64, 33)])
def test_fp8_pack_and_dequant_match_the_oracle(P, H, D, tokens):
    import torch
    from gpu_util import to_dev
    ll = _ll()
    _, x, _ = chunk_qkv(951, P, tokens, tokens, H, D)
    x = x.copy()
    x[0] = 0                                   # a zero row (scale 1)
    x[1, 0, :] = 0x0001                        # a row of the smallest subnormal (floor scale)
    x[2, 1, 0] = 0x7F7F                        # the largest finite bf16
    rows = tokens * H
    codes = torch.empty(rows * D, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    ll.ll_sp_pack_heads_fp8(to_dev(x), tokens, H, D, P, codes, scales)
    deq = torch.empty(rows * D, dtype=torch.bfloat16, device="cuda")
    ll.ll_sp_dequant_fp8(codes, scales, rows, D, deq)
    torch.cuda.synchronize()
    perm = x.reshape(tokens, P, H // P, D).transpose(1, 0, 2, 3).reshape(rows, D)
    wc, ws = quant.fp8_quantize_rows(perm)
    assert np.array_equal(codes.cpu().numpy().reshape(rows, D), wc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    want = quant.fp8_dequantize_rows(wc, ws)
    got = deq.float().cpu().numpy().astype(np.float64).reshape(rows, D)
    fin = np.abs(want) < 2.0 ** 128                # code x scale of the largest bf16 reaches 2^128
    assert np.array_equal(got[fin], want[fin])


def _thread_exchange(r, P, bar, slots):
    import torch

    def exchange(recv, send):
        torch.cuda.synchronize()
        slots[r] = send
        bar.wait()
        n = recv.numel() // P
        for s in range(P):
            recv[s * n:(s + 1) * n].copy_(slots[s][r * n:(r + 1) * n])
        torch.cuda.synchronize()
        bar.wait()
    return exchange


def _sharded_run(P, H, D, T, F, S, W, kv_dtype, compress, n_chunks, seed):
    """P threads, each a rank with its own H/P-head cache; returns per-rank
    outputs per chunk and cache exports."""
    import torch
    from gpu_util import to_dev
    ll = _ll()
    from kv_cache_attention_ll_b200.sp import SequenceParallelAttention
    N = F * T
    ns = N // P
    chunks = [chunk_qkv(seed, 0, c, N, H, D) for c in range(n_chunks)]
    bar = threading.Barrier(P)
    slots = {}
    res = {}
    errors = []

    def rank(r):
        try:
            cache = ll.ll_kv_cache_create(1, H // P, D, T, F, S, W, kv_dtype)
            try:
                spa = SequenceParallelAttention(cache, P, ns, H, D, compress_kv=compress,
                                                exchange=_thread_exchange(r, P, bar, slots))
                outs = []
                for c in range(n_chunks):
                    q, k, v = (to_dev(x[r * ns:(r + 1) * ns].copy()) for x in chunks[c])
                    out = torch.empty_like(q)
                    spa.step(0, q, k, v, out)
                    torch.cuda.synchronize()
                    outs.append(out.view(torch.int16).cpu().numpy().copy())
                res[r] = (outs, ll.ll_kv_cache_export(cache, 0), ll.ll_debug_status(cache))
            finally:
                cache.close()
        except Exception as e:          # reported by the main thread
            errors.append(e)
            bar.abort()

    th = [threading.Thread(target=rank, args=(r,)) for r in range(P)]
    for t in th:
        t.start()
    for t in th:
        t.join(300)
    assert not errors, errors
    return chunks, res


def _unsharded_run(H, D, T, F, S, W, kv_dtype, chunks, compress):
    import torch
    from gpu_util import to_dev
    ll = _ll()
    N = F * T
    cache = ll.ll_kv_cache_create(1, H, D, T, F, S, W, kv_dtype)
    outs = []
    try:
        for q, k, v in chunks:
            if compress:
                # the FP8 round trip the exchange applies to K and V, with P = 1
                k, v = (_fp8_round_trip(ll, x, N, H, D) for x in (k, v))
            dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
            out = torch.empty_like(dq)
            ll.ll_attn_sink_window(dq, dk, dv, cache, 0, out)
            ll.ll_kv_append(cache, 0, dk, dv)
            torch.cuda.synchronize()
            outs.append(out.view(torch.int16).cpu().numpy().copy())
        export = ll.ll_kv_cache_export(cache, 0)
    finally:
        cache.close()
    return outs, export


def _fp8_round_trip(ll, x, N, H, D):
    """K or V rows through the oracle's FP8 row format and back (exact in bf16)."""
    c, s = quant.fp8_quantize_rows(x)
    f = quant.fp8_dequantize_rows(c, s).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _split_export(export: bytes, P: int, H: int, D: int, slots: int, kv_dtype: str, r: int) -> bytes:
    """The bytes of an unsharded layer export that belong to the heads of rank r."""
    b = np.frombuffer(export, np.uint8)
    row = {"bf16": 2 * D, "fp8": D, "nvfp4": D // 2}[kv_dtype]
    srow = {"bf16": 0, "fp8": 4, "nvfp4": D // 16}[kv_dtype]
    data = b[:2 * H * slots * row].reshape(2, H, slots * row)
    scl = b[2 * H * slots * row:].reshape(2, H, slots * srow)
    hs = slice(r * (H // P), (r + 1) * (H // P))
    return np.concatenate([data[:, hs].reshape(-1), scl[:, hs].reshape(-1)]).tobytes()


@pytest.mark.parametrize("P,H,D,T,F,S,W,kv_dtype,compress", [
    (2, 4, 128, 64, 3, 3, 6, "bf16", False),
    (4, 8, 64, 48, 2, 1, 3, "nvfp4", False),
    (2, 4, 128, 64, 3, 3, 6, "fp8", True),
    (3, 6, 128, 50, 3, 2, 4, "bf16", True),
])
def test_emulated_ranks_equal_one_unsharded_cache(P, H, D, T, F, S, W, kv_dtype, compress):
    n_chunks = 6
    chunks, res = _sharded_run(P, H, D, T, F, S, W, kv_dtype, compress, n_chunks, seed=960 + P)
    ref_outs, ref_export = _unsharded_run(H, D, T, F, S, W, kv_dtype, chunks, compress)
    N = F * T
    ns = N // P
    for c in range(n_chunks):
        got = np.concatenate([res[r][0][c].reshape(ns, H, D) for r in range(P)])
        assert np.array_equal(got, ref_outs[c].reshape(N, H, D)), f"chunk {c}"
    slots = (S + W) * T
    for r in range(P):
        assert res[r][1] == _split_export(ref_export, P, H, D, slots, kv_dtype, r), f"rank {r} cache bytes"
        assert res[r][2] == 0


def test_one_rank_nccl_group():
    """The orchestration over a real NCCL group (one rank: the all-to-alls are
    copies) equals the unsharded call."""
    import os
    import torch
    import torch.distributed as dist
    from gpu_util import to_dev
    from kv_cache_attention_ll_b200.sp import SequenceParallelAttention
    ll = _ll()
    H, D, T, F, S, W = 4, 128, 40, 3, 3, 6
    N = F * T
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(29400 + os.getpid() % 1000)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        a = ll.ll_kv_cache_create(1, H, D, T, F, S, W)
        b = ll.ll_kv_cache_create(1, H, D, T, F, S, W)
        try:
            spa = SequenceParallelAttention(a, 1, N, H, D, compress_kv=False)
            for c in range(4):
                q, k, v = (to_dev(x) for x in chunk_qkv(970, 0, c, N, H, D))
                o1, o2 = torch.empty_like(q), torch.empty_like(q)
                spa.step(0, q, k, v, o1)
                ll.ll_attn_sink_window(q, k, v, b, 0, o2)
                ll.ll_kv_append(b, 0, k, v)
                torch.cuda.synchronize()
                assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
            assert ll.ll_kv_cache_export(a, 0) == ll.ll_kv_cache_export(b, 0)
        finally:
            a.close()
            b.close()
    finally:
        dist.destroy_process_group()
