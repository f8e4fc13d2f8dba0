// attn_sink_window.cuh - sink + window + own-chunk attention for sm_100a.
//
// Computes, per head h and query row i of the current chunk,
//   out[i,h,:] = softmax_j( q[i,h,:] . k_j / sqrt(D) ) v_j
// over the keys j of the visible cache slots of layer l and the chunk's own
// k_cur/v_cur (Tq keys, no mask inside the chunk). The key set follows the
// LongLive pages: KV cache = sink frames + recent window (dpshk.com LongLive
// explainer, sec. 五 and 六); with several shots, a global sink plus the
// current shot's sink (LongLive-2.0 explainer, wmrh.cn, sec. 16); own chunk
// visible, future invisible (wmrh.cn sec. 6). The visible cache slots form at
// most three row ranges (cache_layout.cuh); in a single-shot rollout they are
// the one range [0, (s + w) T).
//
// Work unit: one 128-row query tile of one head (one CTA). The key range is cut
// into 128-key tiles; even tiles go to softmax warpgroup 0, odd tiles to
// warpgroup 1 (split-KV inside the CTA), each with its own S and O accumulators
// in tensor memory; the two partial results are merged with their row maxima
// and sums in the epilogue. Tiles past the valid keys are never visited; only
// the last tile of each key range masks its tail columns.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup 0 (thread t owns query row t = TMEM lane t)
//   warps 4-7  softmax warpgroup 1
//   warp 8     TMA producer (Q once, then K and V tiles into an NST-deep ring)
//   warp 9     TMEM allocator and tcgen05.mma issuer
//   warps 10-11 idle (they complete the third warpgroup for register reallocation),
//              or, when the call also appends (fused append), they store this
//              CTA's 128 own-chunk rows of k_cur/v_cur of head h into the cache
//
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D). P_g (bf16) overwrites the first 64 columns of S_g and is
// the A operand of the PV product straight from tensor memory.
//
// Per tile j of warpgroup g the MMA issue order is
//   S_g = Q K_j^T  (SS, K-major both)   ...   O_g += P_g V_j  (TS, V MN-major)
// and S for tile j+2 is issued after PV_j; tcgen05 MMAs of one thread execute in
// order, so P_g is consumed before S_g is overwritten.
#pragma once
#include <cuda_bf16.h>

#include "cache_layout.cuh"
#include "kv_codec.cuh"
#include "sm100_ptx.cuh"

namespace llk {

struct AttnParams {
  CUtensorMap tm_q;      // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_kcur;   // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_vcur;   // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_cache;  // (D, slots, L*2*H) bf16, box (64, 128, 1)
  __nv_bfloat16 *out;    // [Tq][H][D]
  unsigned *err;         // status word (see sm100_ptx.cuh)
  const LayerCtr *ctr;   // this layer's counters (device), or null: then slots [0, n_cache) are visible
  int H;
  int Tq;
  int n_cache;           // visible cache keys when ctr is null
  int G, Ss, W, R, T;    // global sink, shot sink, window frames, ring slots; tokens per frame (with ctr)
  // fused append (append != 0): the chunk's own K/V also go into the cache, in
  // the same launch; needs R >= W + F so that no written slot is one this
  // launch reads. The last CTA to finish advances the layer's counters.
  int append;
  int fmt;               // cache storage format (CacheFormat)
  int F;                 // frames per chunk
  int plane_k_cache;     // (l*2 + 0) * H in the cache itself (plane_k may address a bf16 view)
  int slots;             // rows per cache plane
  const uint4 *kcur, *vcur;  // k_cur / v_cur as 16-byte vectors
  uint8_t *cache_data, *cache_scales;
  LayerCtr *ctr_rw;      // the layer's counters, advanced by the last CTA
  unsigned *done;        // the layer's completion count (zero between launches)
  int plane_k;           // (l*2 + 0) * H : plane of head 0 of this layer's K
  int plane_v;           // (l*2 + 1) * H
  int num_q_tiles;
  float scale_log2;      // log2(e) / sqrt(D)
  int map_rows;          // rows per plane and planes of tm_cache, and planes of the
  int map_planes;        // cache itself (fused append): the bounds-checking build
  int cache_planes;      // checks every tile coordinate and store against them
};

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;                    // query rows per CTA
  static constexpr int BN = 128;                    // keys per tile
  static constexpr int NBOX = D / 64;               // 128-byte-wide TMA boxes per row
  static constexpr int BOX_BYTES = 128 * 128;       // one box: 128 rows x 128 B
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int TILE_BYTES = BN * D * 2;
  static constexpr int NST = (D == 128) ? 3 : 4;    // K/V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NST * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NST * TILE_BYTES;
  // barriers: q_full, k_full[NST], k_empty[NST], v_full[NST], v_empty[NST],
  //           s_full[2], p_full[2], o_full[2], mma_done
  static constexpr int NBAR = 1 + 4 * NST + 7;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // tmem base, abort flag, tile counts
  static constexpr int OFF_RANGES = OFF_MISC + 32;          // the visible key ranges (KeyRanges)
  // m[2][128], l[2][128] of the epilogue merge reuse the Q tile: by then every
  // MMA (all of which read Q before the last PV) has completed
  static constexpr int OFF_STATS = OFF_Q;
  static constexpr int OFF_CTR = OFF_RANGES + 64;           // counters seen at launch (fused append)
  static constexpr int SMEM_BYTES = OFF_CTR + 32;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;      // slack for 1024-byte alignment
  static constexpr int THREADS = 384;   // 3 warpgroups; warps 10-11 idle unless the call appends
  // registers: launched with 384 x 168 = 64512; the producer/MMA warpgroup drops
  // to 64 and the softmax warpgroups rise to 216: 128*64 + 256*216 = 63488 <= 64512
  static constexpr uint32_t REGS_SOFTMAX = 216;
  static constexpr uint32_t REGS_ISSUE = 64;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, D, 0, 1);
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Which pairs of probabilities (bit e%8 for pair e) take exp2 on the FMA pipe
// instead of MUFU. MUFU runs 4 lanes per clock per sub-partition, so one softmax
// warp alone needs 1024 clocks for 128 exp2 per row; moving a share of them to
// FMA-pipe polynomials balances the two pipes.
constexpr unsigned kPolyPairs = 0x88u;

// The visible cache keys as up to three row ranges of the layer's planes, and
// their 128-key tiles: ranges are read from the layer's device counters
// (advanced by the append kernel), so one launch is right for any state, as
// when a captured graph is replayed.
struct KeyRanges {
  int r0, n0, r1, n1, r2, n2;  // first row and row count of each range
  int t1, t2, nc;              // first tile of ranges 1 and 2; cache tiles in all
};

__device__ __forceinline__ KeyRanges visible_key_ranges(const AttnParams &prm) {
  KeyRanges k = {0, prm.n_cache, 0, 0, 0, 0, 0, 0, 0};
  if (prm.ctr) {
    const long long ring_count = __ldcg(&prm.ctr->ring_count);
    const HeldFrames hf = held_frames(__ldcg(&prm.ctr->p), __ldcg(&prm.ctr->shot_fill), ring_count,
                                      __ldcg(&prm.ctr->ring_start), prm.G, prm.W);
    const FrameRanges fr = visible_ranges(hf, ring_count, prm.G, prm.Ss, prm.R);
    k.r0 = fr.start[0] * prm.T;
    k.n0 = fr.len[0] * prm.T;
    k.r1 = fr.start[1] * prm.T;
    k.n1 = fr.len[1] * prm.T;
    k.r2 = fr.start[2] * prm.T;
    k.n2 = fr.len[2] * prm.T;
  }
  k.t1 = (k.n0 + 127) / 128;
  k.t2 = k.t1 + (k.n1 + 127) / 128;
  k.nc = k.t2 + (k.n2 + 127) / 128;
  return k;
}

// The ranges live in shared memory (written once by thread 0) and are read
// where needed, so that they hold no registers across the tile loops.
// first cache row of cache tile j (j < nc)
__device__ __forceinline__ int cache_tile_row(const volatile KeyRanges *k, int j) {
  if (j < k->t1) return k->r0 + j * 128;
  if (j < k->t2) return k->r1 + (j - k->t1) * 128;
  return k->r2 + (j - k->t2) * 128;
}

// valid keys of tile j: cache tiles, then the own chunk's tiles
__device__ __forceinline__ int tile_valid(const volatile KeyRanges *k, int j, int Tq) {
  const int t1 = k->t1, t2 = k->t2, nc = k->nc;
  if (j < t1) return min(128, k->n0 - j * 128);
  if (j < t2) return min(128, k->n1 - (j - t1) * 128);
  if (j < nc) return min(128, k->n2 - (j - t2) * 128);
  return min(128, Tq - (j - nc) * 128);
}

template <int D>
__global__ void __launch_bounds__(384, 1) attn_sink_window_kernel(const __grid_constant__ AttnParams prm) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = k_full + C::NST;
  uint64_t *v_full = k_empty + C::NST;
  uint64_t *v_empty = v_full + C::NST;
  uint64_t *s_full = v_empty + C::NST;
  uint64_t *p_full = s_full + 2;
  uint64_t *o_full = p_full + 2;
  uint64_t *mma_done = o_full + 2;
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  int *tile_count = reinterpret_cast<int *>(smem + C::OFF_MISC + 8);
  float *stat_m = reinterpret_cast<float *>(smem + C::OFF_STATS);
  float *stat_l = stat_m + 2 * 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int unit = blockIdx.x;
  const int h = unit / prm.num_q_tiles;
  const int q0 = (unit % prm.num_q_tiles) * C::BM;
  volatile KeyRanges *kr = reinterpret_cast<volatile KeyRanges *>(smem + C::OFF_RANGES);
  const int nown = (prm.Tq + C::BN - 1) / C::BN;

  LayerCtr *ctr_seen = reinterpret_cast<LayerCtr *>(smem + C::OFF_CTR);
  if (threadIdx.x == 0) {
    if (prm.append) {
      // the counters as this CTA sees them, read before its completion count
      ctr_seen->p = __ldcg(&prm.ctr->p);
      ctr_seen->ring_count = __ldcg(&prm.ctr->ring_count);
      ctr_seen->shot_fill = __ldcg(&prm.ctr->shot_fill);
    }
    const KeyRanges k = visible_key_ranges(prm);
    kr->r0 = k.r0; kr->n0 = k.n0; kr->r1 = k.r1; kr->n1 = k.n1; kr->r2 = k.r2; kr->n2 = k.n2;
    kr->t1 = k.t1; kr->t2 = k.t2; kr->nc = k.nc;
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(s_full + g, 1);
      mbar_init(p_full + g, 128);
      mbar_init(o_full + g, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_base_smem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&prm.tm_q);
    prefetch_tensormap(&prm.tm_kcur);
    prefetch_tensormap(&prm.tm_vcur);
    prefetch_tensormap(&prm.tm_cache);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;
  const int nc = kr->nc;
  const int n_tiles = nc + nown;
  // column bases: S_g = tmem + 128 g, O_g = tmem + 256 + D g
#define TM_S(g) (tmem + 128u * static_cast<uint32_t>(g))
#define TM_O(g) (tmem + 256u + static_cast<uint32_t>(D) * static_cast<uint32_t>(g))

  if (warp >= 8) {
  // each role sets its register budget inside its own branch, so that the
  // allocation limit is unambiguous at every point of the role's code
  regs_dec<C::REGS_ISSUE>();
  if (warp == 8) {
    // ------------------------------------------------------------- producer
    // The whole warp runs this loop converged; one elected lane issues.
    uint8_t *sq = smem + C::OFF_Q;
    if (elect_one()) {
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int b = 0; b < C::NBOX; ++b) tma_load_3d(sq + b * C::BOX_BYTES, &prm.tm_q, q_full, b * 64, h, q0);
    }
    __syncwarp();
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % C::NST;
      const uint32_t par = ((j / C::NST) & 1) ^ 1;
      uint8_t *sk = smem + C::OFF_K + st * C::TILE_BYTES;
      uint8_t *sv = smem + C::OFF_V + st * C::TILE_BYTES;
      if (!__all_sync(0xffffffffu, mbar_wait(k_empty + st, par, abort_flag, prm.err, KID_ATTN))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(k_full + st, C::TILE_BYTES);
        if (j < nc) {
          int row0 = cache_tile_row(kr, j);
          // (bounds-checking build) a tile outside the map is flagged and replaced
          // by row 0, so that the barrier still completes
          if (!LL_BOUNDS(row0 >= 0 && row0 + tile_valid(kr, j, prm.Tq) <= prm.map_rows &&
                             prm.plane_v + h < prm.map_planes,
                         prm.err, KID_ATTN))
            row0 = 0;
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sk + b * C::BOX_BYTES, &prm.tm_cache, k_full + st, b * 64, row0, prm.plane_k + h);
        } else {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sk + b * C::BOX_BYTES, &prm.tm_kcur, k_full + st, b * 64, h, (j - nc) * C::BN);
        }
      }
      __syncwarp();
      issued_k = j + 1;
      if (!__all_sync(0xffffffffu, mbar_wait(v_empty + st, par, abort_flag, prm.err, KID_ATTN))) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(v_full + st, C::TILE_BYTES);
        if (j < nc) {
          int row0 = cache_tile_row(kr, j);
          if (!LL_BOUNDS(row0 >= 0 && row0 + tile_valid(kr, j, prm.Tq) <= prm.map_rows, prm.err, KID_ATTN)) row0 = 0;
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sv + b * C::BOX_BYTES, &prm.tm_cache, v_full + st, b * 64, row0, prm.plane_v + h);
        } else {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sv + b * C::BOX_BYTES, &prm.tm_vcur, v_full + st, b * 64, h, (j - nc) * C::BN);
        }
      }
      __syncwarp();
      issued_v = j + 1;
    }
    if (*abort_flag && lane == 0) {
      mbar_wait_drain(q_full, 0);
      // every load issued must land before the CTA exits: wait for the last
      // NST of each kind (earlier ones were consumed, so they have landed)
      for (int j = issued_k > C::NST ? issued_k - C::NST : 0; j < issued_k; ++j)
        mbar_wait_drain(k_full + j % C::NST, (j / C::NST) & 1);
      for (int j = issued_v > C::NST ? issued_v - C::NST : 0; j < issued_v; ++j)
        mbar_wait_drain(v_full + j % C::NST, (j / C::NST) & 1);
    }
    __syncwarp();
  } else if (warp >= 10) {
    if (prm.append) {
      // ---------------------------------------------------- fused append
      // Own-chunk rows q0 .. q0+127 of head h: each (token, head) row is D/8
      // consecutive lanes; the trip count is uniform, so the quantising
      // formats' row shuffles always see whole warps.
      constexpr int VPR = D / 8;
      const int tid = threadIdx.x - 320;                       // 0 .. 63
      const int rows = min(C::BM, prm.Tq - q0);
      const long long p = ctr_seen->p, ring_count = ctr_seen->ring_count;
      const int shot_fill = ctr_seen->shot_fill;
      const long long plane_k = prm.plane_k_cache + h, plane_v = plane_k + prm.H;
      for (int base = 0; base < C::BM * VPR; base += 64) {
        const int i = base + tid;
        const int r = i / VPR, vec = i % VPR;
        const int t = q0 + r;                                  // token of the chunk
        const int fi = t / prm.T;
        const int slot = r < rows ? append_slot(p, shot_fill, ring_count, prm.G, prm.Ss, prm.R, prm.F, fi) : -1;
        const long long drow = static_cast<long long>(slot) * prm.T + (t - fi * prm.T);
        const bool act = slot >= 0 && LL_BOUNDS(drow < prm.slots && plane_v < prm.cache_planes, prm.err, KID_ATTN);
        uint4 vk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        if (act) {
          const long long src = (static_cast<long long>(t) * prm.H + h) * VPR + vec;
          vk = __ldg(prm.kcur + src);
          vv = __ldg(prm.vcur + src);
        }
        if (prm.fmt == FMT_FP8)
          store_kv_vec<FMT_FP8>(prm.cache_data, prm.cache_scales, plane_k, plane_v, prm.slots, drow, D, vec, vk, vv,
                                act);
        else if (prm.fmt == FMT_NVFP4)
          store_kv_vec<FMT_NVFP4>(prm.cache_data, prm.cache_scales, plane_k, plane_v, prm.slots, drow, D, vec, vk, vv,
                                  act);
        else
          store_kv_vec<FMT_BF16>(prm.cache_data, prm.cache_scales, plane_k, plane_v, prm.slots, drow, D, vec, vk, vv,
                                 act);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged (operands stay warp-uniform);
    // one elected lane issues each tcgen05 instruction.
    bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, prm.err, KID_ATTN));
    // Shared-memory descriptors are built once; each MMA only adds a constant
    // to the start-address field (bits 0-13, address >> 4). Every operand lies
    // below 256 KB of shared memory, so the field never carries into LBO.
    const uint64_t dq0 = smem_desc(smem_u32(smem + C::OFF_Q), 16, 1024, 2);
    const uint64_t dk0 = smem_desc(smem_u32(smem + C::OFF_K), 16, 1024, 2);
    const uint64_t dv0 = smem_desc(smem_u32(smem + C::OFF_V), C::BOX_BYTES, 1024, 2);
    // S_j = Q K_j^T into S_{j%2}, then the commits that free K_j's stage and
    // tell the softmax; issued by the elected lane, its K tile already waited for
    auto issue_s_mmas = [&](int j) {
      const int st = j % C::NST;
      const uint64_t dk = dk0 + static_cast<uint64_t>((st * C::TILE_BYTES) >> 4);
      const uint32_t d_tmem = TM_S(j & 1);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // K step kk: box kk/4 (64 head-dim columns each), 32-byte slice kk%4 of the 128-byte row
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4);
        mma_bf16_ss(d_tmem, dq0 + off, dk + off, C::IDESC_S, kk > 0 ? 1u : 0u);
      }
      mma_commit(k_empty + st);
      mma_commit(s_full + (j & 1));
    };
    // the first two S: one elected block each (an elect per MMA costs more than
    // the MMA itself; operands are computed by the converged warp)
    for (int j = 0; ok && j < 2 && j < n_tiles; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(k_full + j, 0, abort_flag, prm.err, KID_ATTN));
      if (ok) {
        tc_fence_after();
        if (elect_one()) issue_s_mmas(j);
        __syncwarp();
      }
    }
    for (int j = 0; ok && j < n_tiles; ++j) {
      const int g = j & 1, it = j >> 1, st = j % C::NST;
      // the V tile of this PV and the K tile of the next S are waited for first:
      // neither depends on the softmax (the producer loads them once earlier
      // MMAs free their stages), so the wait for P is the last before the issue
      // and PV and the next S go out together, in one elected block, as soon as P
      // is complete (together 3-5 % fewer cycles than waiting for P first)
      if (!__all_sync(0xffffffffu, mbar_wait(v_full + st, (j / C::NST) & 1, abort_flag, prm.err, KID_ATTN))) break;
      if (j + 2 < n_tiles && !__all_sync(0xffffffffu, mbar_wait(k_full + (j + 2) % C::NST, ((j + 2) / C::NST) & 1,
                                                                 abort_flag, prm.err, KID_ATTN)))
        break;
      if (!__all_sync(0xffffffffu, mbar_wait(p_full + g, it & 1, abort_flag, prm.err, KID_ATTN))) break;
      tc_fence_after();
      const uint64_t dv = dv0 + static_cast<uint64_t>((st * C::TILE_BYTES) >> 4);
      const uint32_t o_tmem = TM_O(g), p_tmem = TM_S(g);
      const uint32_t acc0 = it > 0 ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // V tile: rows = keys (the K dim of this product), 16 keys = 2048 bytes per
          // step; boxes of 64 head-dim columns C::BOX_BYTES apart (MN-major operand);
          // P_g: 16 keys = 8 bf16x2 columns of tensor memory per step
          mma_bf16_ts(o_tmem, p_tmem + kk * 8, dv + static_cast<uint64_t>((kk * 16 * 128) >> 4), C::IDESC_O,
                      kk > 0 ? 1u : acc0);
        }
        mma_commit(v_empty + st);
        mma_commit(o_full + g);
        // and S_{j+2} in the same elected block (its K tile was waited for above)
        if (j + 2 < n_tiles) issue_s_mmas(j + 2);
      }
      __syncwarp();
    }
    // every MMA issued must finish before tensor memory is released
    if (elect_one()) {
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
    __syncwarp();
  }
  } else {
    regs_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------- softmax groups
    const int g = warp >> 2;              // warpgroup 0 or 1
    const int row = threadIdx.x & 127;    // TMEM lane == query row in the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY, l_run = 0.f;
    int it = 0;
    bool ok = true;
    for (int j = g; j < n_tiles; j += 2, ++it) {
      // the tile's valid keys, read from shared memory while S is still computed
      const int valid = tile_valid(kr, j, prm.Tq);
      // wait results are made warp-uniform: a warp never splits across the
      // .sync.aligned tensor-memory instructions that follow
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + g, it & 1, abort_flag, prm.err, KID_ATTN))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // S_g of this tile is complete, and with it every MMA issued before it,
      // among them the previous PV into O_g: O_g may be rescaled right away, and
      // no separate wait for that PV is needed (only the last one is awaited).
      uint32_t sr[128];
      tmem_ld64(TM_S(g) + lane_off, sr);
      tmem_ld64(TM_S(g) + lane_off + 64, sr + 64);
      if (valid < 128) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= valid) sr[e] = __float_as_uint(-INFINITY);
      }
      // row max: four independent chains of 3-input maxima
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 128; e += 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m4[i] = fmax3(m4[i], __uint_as_float(sr[e + 2 * i]), __uint_as_float(sr[e + 2 * i + 1]));
      }
      const float m_tile = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sl2;
      // lazy rescale: the reference max moves only when a tile's max exceeds it
      // by more than 8 (log2 units), so probabilities stay below 2^8
      const bool grow = m_tile > m_ref + 8.0f;
      const float m_new = grow ? m_tile : m_ref;
      const float alpha = (grow && it > 0) ? ex2_approx(m_ref - m_new) : 1.0f;
      if (it > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(TM_O(g) + lane_off + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(TM_O(g) + lane_off + c * 32, r);
        }
      }
      // probabilities in pairs: x = s * log2(e)/sqrt(D) - m (packed FMA); pairs
      // selected by kPolyPairs use the FMA-pipe exp2, the rest MUFU; four packed
      // partial sums; bf16 pairs written back over S as the A operand of PV
      const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_new, -m_new);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pr[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2x2, nm2);
        float2 pp;
        if ((kPolyPairs >> (e & 7)) & 1) {
          pp = exp2_poly2(x);
        } else {
          pp.x = ex2_approx(x.x);
          pp.y = ex2_approx(x.y);
        }
        acc[e & 3] = __fadd2_rn(acc[e & 3], pp);
        pr[e] = pack_bf16x2(pp.x, pp.y);
      }
      tmem_st64(TM_S(g) + lane_off, pr);
      const float2 a03 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
      l_run = (it > 0 ? l_run * alpha : 0.f) + (a03.x + a03.y);
      m_ref = m_new;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full + g);
    }
    if (ok && it > 0) {
      if (__all_sync(0xffffffffu, mbar_wait(o_full + g, (it - 1) & 1, abort_flag, prm.err, KID_ATTN)))
        tc_fence_after();
      else
        ok = false;
    }
    // ---- merge the two split-KV halves and write the output tile
    // both groups have seen their last PV complete (or aborted) before the Q
    // region is reused for the row statistics
    tc_fence_before();
    named_bar_sync(1, 256);
    if (!*abort_flag) {
      stat_m[g * 128 + row] = m_ref;
      stat_l[g * 128 + row] = l_run;
      if (row == 0) tile_count[g] = it;
    }
    named_bar_sync(1, 256);
    tc_fence_after();
    if (!*abort_flag) {
      const int it1 = tile_count[1];
      const float m0 = stat_m[row], m1 = stat_m[128 + row];
      const float l0 = stat_l[row], l1 = stat_l[128 + row];
      const float M = it1 > 0 ? fmaxf(m0, m1) : m0;
      const float a0 = ex2_approx(m0 - M);
      const float a1 = it1 > 0 ? ex2_approx(m1 - M) : 0.f;
      const float inv = 1.0f / (a0 * l0 + a1 * l1);
      const float c0 = a0 * inv, c1 = a1 * inv;
      const int qrow = q0 + row;
      __nv_bfloat16 *dst = prm.out + (static_cast<size_t>(qrow) * prm.H + h) * D;
#pragma unroll 1
      for (int c = g * (D / 64); c < (g + 1) * (D / 64); ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld32(TM_O(0) + lane_off + c * 32, r0);
        if (it1 > 0) tmem_ld32(TM_O(1) + lane_off + c * 32, r1);
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0 = __uint_as_float(r0[2 * e]) * c0, x1 = __uint_as_float(r0[2 * e + 1]) * c0;
          if (it1 > 0) {
            x0 = fmaf(__uint_as_float(r1[2 * e]), c1, x0);
            x1 = fmaf(__uint_as_float(r1[2 * e + 1]), c1, x1);
          }
          packed[e] = pack_bf16x2(x0, x1);
        }
        if (qrow < prm.Tq) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        }
      }
    }
  }

  if (warp < 8) tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (prm.append && threadIdx.x == 0) {
    // the last CTA to finish advances the layer's counters; every CTA read them
    // at its start, before its increment of the completion count
    __threadfence();
    const unsigned prev = atomicAdd(prm.done, 1u);
    if (prev == gridDim.x - 1) {
      int fill;
      long long rc;
      append_advance(ctr_seen->p, ctr_seen->shot_fill, ctr_seen->ring_count, prm.G, prm.Ss, prm.F, &fill, &rc);
      prm.ctr_rw->p = ctr_seen->p + prm.F;
      prm.ctr_rw->shot_fill = fill;
      prm.ctr_rw->ring_count = rc;
      *prm.done = 0;
      __threadfence();
    }
  }
#undef TM_S
#undef TM_O
}

}  // namespace llk
