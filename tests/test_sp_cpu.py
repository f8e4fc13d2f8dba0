"""The sequence-parallel step's orchestration on CPU ranks: world size 2 over
gloo, with host stand-ins for the library's local steps (the pack, unpack and
FP8 exchange layouts restated with torch reshapes and the oracle's FP8 rows;
attention and append by the oracle's cache model and attention).

Each rank feeds its half of the tokens of every chunk; after the two
all-to-alls and the unpack, each rank's output rows must equal the oracle's
attention of the whole chunk over the unsharded history for those tokens and
all heads, and each rank's cache must hold exactly the heads it owns.
(LongLive-2.0 explainer, wmrh.cn, sec. 18.3 and 15.2.)"""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

H, D, T, F, S, W = 4, 64, 8, 2, 1, 3          # 16 tokens per chunk, 8 per rank
N_CHUNKS = 5


class _HostCache:
    """Stand-in of one rank's cache: the oracle's cache model of its heads."""

    def __init__(self, heads, kv_dtype):
        import oracle
        self.heads, self.head_dim, self.tq = heads, D, F * T
        self.model = oracle.CacheModel(1, heads, D, T, F, S, W, kv_dtype)
        self.chunk = 0


def _bits(t):
    import torch
    return t.view(torch.int16).numpy().view(np.uint16)


def _from_bits(bits, out):
    import torch
    out.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).reshape(out.shape))


class _HostOps:
    """The local steps on host tensors, restated without the library."""

    def pack(self, x, tokens, heads, head_dim, ranks, packed):
        packed.copy_(x.reshape(tokens, ranks, heads // ranks, head_dim).permute(1, 0, 2, 3).reshape(-1))

    def unpack(self, packed, tokens, heads, head_dim, ranks, x):
        x.copy_(packed.reshape(ranks, tokens, heads // ranks, head_dim).permute(1, 0, 2, 3).reshape(x.shape))

    def pack_fp8(self, x, tokens, heads, head_dim, ranks, codes, scales):
        import torch
        from oracle import quant
        rows = _bits(x.reshape(tokens, ranks, heads // ranks, head_dim).permute(1, 0, 2, 3).contiguous())
        c, s = quant.fp8_quantize_rows(rows)
        codes.copy_(torch.from_numpy(c.reshape(-1)))
        scales.copy_(torch.from_numpy(s.reshape(-1)))

    def dequant_fp8(self, codes, scales, rows, head_dim, x):
        from oracle import quant
        v = quant.fp8_dequantize_rows(codes.numpy().reshape(rows, head_dim), scales.numpy())
        f = v.astype(np.float32)
        assert np.all(f.astype(np.float64) == v)               # exact in bf16 (power-of-two scales)
        _from_bits((f.view(np.uint32) >> 16).astype(np.uint16), x)

    def attention(self, q, k, v, cache, layer, out):
        import oracle
        c = cache.chunk
        hp = cache.heads
        n = (c + 1) * F * T
        kh = np.zeros((n, hp, D))
        vh = np.zeros((n, hp, D))
        for f, vals in cache.model.held_frames(0, 0).items():
            kh[f * T:(f + 1) * T] = vals
        for f, vals in cache.model.held_frames(0, 1).items():
            vh[f * T:(f + 1) * T] = vals
        kb, vb = _bits(k).reshape(F * T, hp, D), _bits(v).reshape(F * T, hp, D)
        from seeded_inputs import bf16_bits_to_f64
        kh[c * F * T:] = bf16_bits_to_f64(kb)
        vh[c * F * T:] = bf16_bits_to_f64(vb)
        ref = oracle.sink_window_attention(_bits(q).reshape(F * T, hp, D), kh, vh, c, S, W, F, T)
        f = ref.astype(np.float32)                              # then rounded to bf16, nearest even
        _from_bits(((f.view(np.uint32) + 0x7FFF + ((f.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16), out)

    def append(self, cache, layer, k, v):
        hp = cache.heads
        cache.model.append(0, _bits(k).reshape(F * T, hp, D), _bits(v).reshape(F * T, hp, D))
        cache.chunk += 1


def _worker(rank, world, port, compress, kv_dtype, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from seeded_inputs import chunk_qkv
    from kv_cache_attention_ll_b200.sp import SequenceParallelAttention
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ns = F * T // world
        cache = _HostCache(H // world, kv_dtype)
        spa = SequenceParallelAttention(cache, world, ns, H, D, compress_kv=compress, ops=_HostOps(),
                                        device=torch.device("cpu"))
        outs = []
        for c in range(N_CHUNKS):
            qb, kb, vb = chunk_qkv(900, 0, c, F * T, H, D)
            sl = slice(rank * ns, (rank + 1) * ns)
            tq, tk, tv = (torch.from_numpy(x[sl].copy().view(np.int16)).view(torch.bfloat16) for x in (qb, kb, vb))
            out = torch.empty_like(tq)
            spa.step(0, tq, tk, tv, out)
            outs.append(_bits(out).copy())
        q.put((rank, outs, cache.model.export(0), spa.bytes_sent_per_step()))
    finally:
        dist.destroy_process_group()


def _reference(compress, kv_dtype):
    """The unsharded computation on the oracle: all heads, all tokens."""
    import oracle
    from oracle import quant
    from seeded_inputs import chunk_qkv, bf16_bits_to_f64
    model = oracle.CacheModel(1, H, D, T, F, S, W, kv_dtype)
    outs = []
    for c in range(N_CHUNKS):
        qb, kb, vb = chunk_qkv(900, 0, c, F * T, H, D)
        if compress:
            # K and V cross the links as FP8 rows and come back exactly dequantised
            kb, vb = ((quant.fp8_dequantize_rows(*quant.fp8_quantize_rows(x)).astype(np.float32)
                       .view(np.uint32) >> 16).astype(np.uint16) for x in (kb, vb))
        n = (c + 1) * F * T
        kh = np.zeros((n, H, D))
        vh = np.zeros((n, H, D))
        for f, vals in model.held_frames(0, 0).items():
            kh[f * T:(f + 1) * T] = vals
        for f, vals in model.held_frames(0, 1).items():
            vh[f * T:(f + 1) * T] = vals
        kh[c * F * T:] = bf16_bits_to_f64(kb)
        vh[c * F * T:] = bf16_bits_to_f64(vb)
        outs.append(oracle.sink_window_attention(qb, kh, vh, c, S, W, F, T))
        model.append(0, kb, vb)
    return outs, model


@pytest.mark.parametrize("compress,kv_dtype", [(False, "bf16"), (True, "bf16"), (True, "fp8")])
def test_two_gloo_ranks_match_the_unsharded_oracle(compress, kv_dtype):
    from seeded_inputs import bf16_bits_to_f64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 30500 + (os.getpid() % 1500) + (7 if compress else 0) + (3 if kv_dtype == "fp8" else 0)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, compress, kv_dtype, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, outs, cache_bytes, sent = q.get(timeout=240)
        res[rank] = (outs, cache_bytes, sent)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    ref, model = _reference(compress, kv_dtype)
    ns = F * T // 2
    for c in range(N_CHUNKS):
        got = np.concatenate([bf16_bits_to_f64(res[r][0][c]).reshape(ns, H, D) for r in range(2)])
        # the stand-in rounds the oracle's output to bf16 once: at most half a
        # step, i.e. the bf16 unit roundoff 2^-8 relative
        assert np.all(np.abs(got - ref[c]) <= 2.0 ** -8 * np.abs(ref[c])), f"chunk {c}"
    # each rank's cache holds its own heads: the unsharded cache's planes, split by head
    full = np.frombuffer(model.export(0), np.uint8)
    row = {"bf16": 2 * D, "fp8": D}[kv_dtype]
    plane = (S + W) * T * row
    data = full[:2 * H * plane].reshape(2, H, plane)
    scale_plane = (S + W) * T * 4 if kv_dtype == "fp8" else 0
    scl = full[2 * H * plane:].reshape(2, H, scale_plane)
    for r in range(2):
        got = np.frombuffer(res[r][1], np.uint8)
        hs = slice(r * (H // 2), (r + 1) * (H // 2))
        want = np.concatenate([data[:, hs].reshape(-1), scl[:, hs].reshape(-1)])
        assert np.array_equal(got, want), f"rank {r} cache bytes"
    # FP8 K/V exchange: D + 4 bytes per row instead of 2D
    n = F * T * (H // 2) * D
    rows = F * T * (H // 2)
    expect = 2 * n + (2 * (n + 4 * rows) if compress else 4 * n) + 2 * n
    assert res[0][2] == expect
