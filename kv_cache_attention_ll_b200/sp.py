"""Head-sharded sequence-parallel attention step over P ranks.

LongLive-2.0 explainer (wmrh.cn): sec. 18.3, inference can run sequence
parallel across GPUs; sec. 15.2, a low-precision KV cache then also reduces the
traffic between them.

Rank r holds tokens [r*N_s, (r+1)*N_s) of the chunk (N = P*N_s) for all H
heads, as a sequence-sharded model emits them, and a cache of the H/P heads
r*H/P .. (r+1)*H/P-1 (ll_kv_cache_create with heads = H/P). One step of one
layer:

  1. pack q, k_cur, v_cur: [N_s][H][D] -> [P][N_s][H/P][D] (ll_sp_pack_heads),
     or, for K and V with compress_kv, to E4M3 codes + fp32 power-of-two row
     scales (ll_sp_pack_heads_fp8): D + 4 bytes per row instead of 2D;
  2. all-to-all with equal splits: rank r receives block r of every rank,
     [P][N_s][H/P][D] = the whole chunk [N][H/P][D] for its heads (FP8 rows
     are restored to bf16 first, ll_sp_dequant_fp8);
  3. ll_attn_sink_window and ll_kv_append on the rank's own cache;
  4. all-to-all of the outputs [N][H/P][D] = [P][N_s][H/P][D] back to the
     ranks that own the tokens, and ll_sp_unpack_heads to [N_s][H][D].

Heads never interact inside attention, append or recache, so each rank's
results equal an unsharded cache's for the same heads (with compress_kv: for
the FP8-rounded K and V of the chunk). The collectives are torch.distributed
(NCCL on GPUs); every local step is one of the library's kernels, passed in as
`ops` so that the same orchestration runs with host stand-ins in CPU tests.
"""
from __future__ import annotations


class LibraryOps:
    """The local steps, as the library's CUDA kernels (the product path)."""

    def __init__(self):
        import kv_cache_attention_ll_b200 as ll
        self.ll = ll

    def pack(self, x, tokens, heads, head_dim, ranks, packed):
        self.ll.ll_sp_pack_heads(x, tokens, heads, head_dim, ranks, packed)

    def unpack(self, packed, tokens, heads, head_dim, ranks, x):
        self.ll.ll_sp_unpack_heads(packed, tokens, heads, head_dim, ranks, x)

    def pack_fp8(self, x, tokens, heads, head_dim, ranks, codes, scales):
        self.ll.ll_sp_pack_heads_fp8(x, tokens, heads, head_dim, ranks, codes, scales)

    def dequant_fp8(self, codes, scales, rows, head_dim, x):
        self.ll.ll_sp_dequant_fp8(codes, scales, rows, head_dim, x)

    def attention(self, q, k, v, cache, layer, out):
        self.ll.ll_attn_sink_window(q, k, v, cache, layer, out)

    def append(self, cache, layer, k, v):
        self.ll.ll_kv_append(cache, layer, k, v)


class SequenceParallelAttention:
    """One rank's side of the head-sharded step; see the module docstring.

    cache: this rank's cache of heads // ranks heads (any storage format).
    tokens_per_rank: N_s; the chunk has ranks * N_s tokens.
    group: the torch.distributed process group (None = the default group).
    compress_kv: send K and V as FP8 rows (the receiver restores them to bf16).
    exchange: the all-to-all, exchange(recv, send), equal splits; defaults to
    torch.distributed.all_to_all_single on `group`.
    """

    def __init__(self, cache, ranks: int, tokens_per_rank: int, heads: int, head_dim: int, group=None,
                 compress_kv: bool = False, ops=None, device=None, exchange=None):
        import torch
        if heads % ranks:
            raise ValueError(f"heads ({heads}) must be divisible by ranks ({ranks})")
        if cache.heads != heads // ranks or cache.head_dim != head_dim:
            raise ValueError("the cache must hold heads // ranks heads of the same head_dim")
        if ranks * tokens_per_rank != cache.tq:
            raise ValueError(f"ranks x tokens_per_rank must be the chunk's {cache.tq} tokens")
        self.cache, self.P, self.Ns, self.H, self.D = cache, ranks, tokens_per_rank, heads, head_dim
        self.Hp = heads // ranks
        self.compress_kv = compress_kv
        self.ops = ops if ops is not None else LibraryOps()
        self.group = group
        if exchange is None:
            import torch.distributed as dist

            def exchange(recv, send):
                dist.all_to_all_single(recv, send, group=group)
        self.exchange = exchange
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        n = ranks * tokens_per_rank * self.Hp * head_dim          # elements of every exchanged block set

        def buf(dtype=torch.bfloat16, count=n):
            return torch.empty(count, dtype=dtype, device=dev)
        self.send = [buf() for _ in range(3)]                    # packed q, k, v
        self.recv = [buf() for _ in range(3)]                    # q, k, v of the whole chunk, this rank's heads
        self.out_full = buf()                                    # attention output [N][H/P][D]
        self.out_recv = buf()
        if compress_kv:
            rows = ranks * tokens_per_rank * self.Hp
            # codes are exchanged as int32 words (D bytes per row, D a multiple of 4)
            self.code_send = [buf(torch.uint8, n) for _ in range(2)]
            self.code_recv = [buf(torch.uint8, n) for _ in range(2)]
            self.scale_send = [buf(torch.float32, rows) for _ in range(2)]
            self.scale_recv = [buf(torch.float32, rows) for _ in range(2)]

    def bytes_sent_per_step(self) -> int:
        """Bytes this rank's all-to-alls move per step (its own block included)."""
        n = self.P * self.Ns * self.Hp * self.D
        rows = self.P * self.Ns * self.Hp
        kv = 2 * (n + 4 * rows) if self.compress_kv else 2 * 2 * n
        return 2 * n + kv + 2 * n                                # q, k and v, the outputs

    def step(self, layer: int, q, k_cur, v_cur, out):
        """q, k_cur, v_cur: this rank's tokens [N_s][H][D]; out: [N_s][H][D], written."""
        import torch
        o, P, Ns, H, D = self.ops, self.P, self.Ns, self.H, self.D
        o.pack(q, Ns, H, D, P, self.send[0])
        self.exchange(self.recv[0], self.send[0])
        if self.compress_kv:
            for i, x in enumerate((k_cur, v_cur)):
                o.pack_fp8(x, Ns, H, D, P, self.code_send[i], self.scale_send[i])
                self.exchange(self.code_recv[i].view(torch.int32), self.code_send[i].view(torch.int32))
                self.exchange(self.scale_recv[i], self.scale_send[i])
                o.dequant_fp8(self.code_recv[i], self.scale_recv[i], P * Ns * self.Hp, D, self.recv[1 + i])
        else:
            for i, x in enumerate((k_cur, v_cur)):
                o.pack(x, Ns, H, D, P, self.send[1 + i])
                self.exchange(self.recv[1 + i], self.send[1 + i])
        q_all, k_all, v_all = self.recv
        o.attention(q_all, k_all, v_all, self.cache, layer, self.out_full)
        o.append(self.cache, layer, k_all, v_all)
        self.exchange(self.out_recv, self.out_full)
        o.unpack(self.out_recv, Ns, H, D, P, out)
