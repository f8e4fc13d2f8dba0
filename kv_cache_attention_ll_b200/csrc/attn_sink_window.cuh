// attn_sink_window.cuh - sink + window + own-chunk attention for sm_100a.
//
// Computes, per head h and query row i of the current chunk,
//   out[i,h,:] = softmax_j( q[i,h,:] . k_j / sqrt(D) ) v_j
// over the keys j of cache slots [0, n_cache) of layer l (sink frames followed
// by the held window frames; the two are one contiguous slot range because the
// window only holds frames once all S sink slots are filled) and the chunk's
// own k_cur/v_cur (Tq keys, no mask inside the chunk). The key set follows the
// LongLive pages: KV cache = sink frames + recent window (dpshk.com LongLive
// explainer, sec. 五 and 六); own chunk visible, future invisible (LongLive-2.0
// explainer, wmrh.cn, sec. 6).
//
// Work unit: one 128-row query tile of one head (one CTA). The key range is cut
// into 128-key tiles; even tiles go to softmax warpgroup 0, odd tiles to
// warpgroup 1 (split-KV inside the CTA), each with its own S and O accumulators
// in tensor memory; the two partial results are merged with their row maxima
// and sums in the epilogue. Tiles past the valid keys are never visited; only
// the last tile of each segment masks its tail columns.
//
// Roles (320 threads):
//   warps 0-3  softmax warpgroup 0 (thread t owns query row t = TMEM lane t)
//   warps 4-7  softmax warpgroup 1
//   warp 8     TMA producer (Q once, then K and V tiles into an NST-deep ring)
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
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

#include "sm100_ptx.cuh"

namespace llk {

struct AttnParams {
  CUtensorMap tm_q;      // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_kcur;   // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_vcur;   // (D, H, Tq) bf16, box (64, 1, 128)
  CUtensorMap tm_cache;  // (D, slots, L*2*H) bf16, box (64, 128, 1)
  __nv_bfloat16 *out;    // [Tq][H][D]
  unsigned *err;         // status word (see sm100_ptx.cuh)
  int H;
  int Tq;
  int n_cache;           // visible cache keys: slots [0, n_cache)
  int plane_k;           // (l*2 + 0) * H : plane of head 0 of this layer's K
  int plane_v;           // (l*2 + 1) * H
  int num_q_tiles;
  float scale_log2;      // log2(e) / sqrt(D)
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
  // m[2][128], l[2][128] of the epilogue merge reuse the Q tile: by then every
  // MMA (all of which read Q before the last PV) has completed
  static constexpr int OFF_STATS = OFF_Q;
  static constexpr int SMEM_BYTES = OFF_MISC + 32;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;      // slack for 1024-byte alignment
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, D, 0, 1);
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

__device__ __forceinline__ int tile_valid(int j, int nc, int n_cache, int Tq) {
  if (j < nc) return min(128, n_cache - j * 128);
  return min(128, Tq - (j - nc) * 128);
}

template <int D>
__global__ void __launch_bounds__(320, 1) attn_sink_window_kernel(const __grid_constant__ AttnParams prm) {
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
  const int nc = (prm.n_cache + C::BN - 1) / C::BN;
  const int nown = (prm.Tq + C::BN - 1) / C::BN;
  const int n_tiles = nc + nown;

  if (threadIdx.x == 0) {
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
  // column bases: S_g = tmem + 128 g, O_g = tmem + 256 + D g
#define TM_S(g) (tmem + 128u * static_cast<uint32_t>(g))
#define TM_O(g) (tmem + 256u + static_cast<uint32_t>(D) * static_cast<uint32_t>(g))

  if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      uint8_t *sq = smem + C::OFF_Q;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int b = 0; b < C::NBOX; ++b) tma_load_3d(sq + b * C::BOX_BYTES, &prm.tm_q, q_full, b * 64, h, q0);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % C::NST;
        const uint32_t par = ((j / C::NST) & 1) ^ 1;
        uint8_t *sk = smem + C::OFF_K + st * C::TILE_BYTES;
        uint8_t *sv = smem + C::OFF_V + st * C::TILE_BYTES;
        if (!mbar_wait(k_empty + st, par, abort_flag, prm.err, KID_ATTN)) break;
        mbar_arrive_expect_tx(k_full + st, C::TILE_BYTES);
        if (j < nc) {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sk + b * C::BOX_BYTES, &prm.tm_cache, k_full + st, b * 64, j * C::BN, prm.plane_k + h);
        } else {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sk + b * C::BOX_BYTES, &prm.tm_kcur, k_full + st, b * 64, h, (j - nc) * C::BN);
        }
        issued_k = j + 1;
        if (!mbar_wait(v_empty + st, par, abort_flag, prm.err, KID_ATTN)) break;
        mbar_arrive_expect_tx(v_full + st, C::TILE_BYTES);
        if (j < nc) {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sv + b * C::BOX_BYTES, &prm.tm_cache, v_full + st, b * 64, j * C::BN, prm.plane_v + h);
        } else {
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(sv + b * C::BOX_BYTES, &prm.tm_vcur, v_full + st, b * 64, h, (j - nc) * C::BN);
        }
        issued_v = j + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(q_full, 0);
        // every load issued must land before the CTA exits: wait for the last
        // NST of each kind (earlier ones were consumed, so they have landed)
        for (int j = issued_k > C::NST ? issued_k - C::NST : 0; j < issued_k; ++j)
          mbar_wait_drain(k_full + j % C::NST, (j / C::NST) & 1);
        for (int j = issued_v > C::NST ? issued_v - C::NST : 0; j < issued_v; ++j)
          mbar_wait_drain(v_full + j % C::NST, (j / C::NST) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag, prm.err, KID_ATTN);
      const uint32_t sq = smem_u32(smem + C::OFF_Q);
      auto issue_s = [&](int j) -> bool {
        const int st = j % C::NST;
        if (!mbar_wait(k_full + st, (j / C::NST) & 1, abort_flag, prm.err, KID_ATTN)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + C::OFF_K + st * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
          const uint64_t da = smem_desc(sq + off, 16, 1024, 2);
          const uint64_t db = smem_desc(sk + off, 16, 1024, 2);
          mma_bf16_ss(TM_S(j & 1), da, db, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(k_empty + st);
        mma_commit(s_full + (j & 1));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int g = j & 1, it = j >> 1, st = j % C::NST;
        if (!mbar_wait(p_full + g, it & 1, abort_flag, prm.err, KID_ATTN)) break;
        if (!mbar_wait(v_full + st, (j / C::NST) & 1, abort_flag, prm.err, KID_ATTN)) break;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + C::OFF_V + st * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // V tile: rows = keys (K dim of this product), 128-byte rows of 64 head-dim
          // values, boxes of 64 head-dim columns C::BOX_BYTES apart (MN-major operand)
          const uint64_t db = smem_desc(sv + kk * 16 * 128, C::BOX_BYTES, 1024, 2);
          mma_bf16_ts(TM_O(g), TM_S(g) + kk * 8, db, C::IDESC_O, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(v_empty + st);
        mma_commit(o_full + g);
        if (j + 2 < n_tiles) ok = issue_s(j + 2);
      }
      // every MMA issued must finish before tensor memory is released
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------- softmax groups
    const int g = warp >> 2;              // warpgroup 0 or 1
    const int row = threadIdx.x & 127;    // TMEM lane == query row in the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = prm.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int it = 0;
    bool ok = true;
    for (int j = g; j < n_tiles; j += 2, ++it) {
      // wait results are made warp-uniform: a warp never splits across the
      // .sync.aligned tensor-memory instructions that follow
      if (!__all_sync(0xffffffffu, mbar_wait(s_full + g, it & 1, abort_flag, prm.err, KID_ATTN))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(TM_S(g) + lane_off + c * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
      }
      const int valid = tile_valid(j, nc, prm.n_cache, prm.Tq);
      if (valid < 128) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= valid) s[e] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int e = 1; e < 128; ++e) mx = fmaxf(mx, s[e]);
      const float m_tile = mx * sl2;
      const bool grow = m_tile > m_run + 8.0f;     // lazy rescale: only when the max grows by > 2^8
      const float m_new = grow ? m_tile : m_run;
      const float alpha = (grow && it > 0) ? ex2_approx(m_run - m_new) : 1.0f;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pr[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2_approx(fmaf(s[c * 64 + 2 * e], sl2, -m_new));
          const float p1 = ex2_approx(fmaf(s[c * 64 + 2 * e + 1], sl2, -m_new));
          sum += p0 + p1;
          pr[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(TM_S(g) + lane_off + c * 32, pr);
      }
      l_run = (it > 0 ? l_run * alpha : 0.f) + sum;
      m_run = m_new;
      if (it > 0) {
        // the previous PV of this group must be complete before O is touched
        if (!__all_sync(0xffffffffu, mbar_wait(o_full + g, (it - 1) & 1, abort_flag, prm.err, KID_ATTN))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(TM_O(g) + lane_off + c * 32, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(TM_O(g) + lane_off + c * 32, r);
          }
        }
      }
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
      stat_m[g * 128 + row] = m_run;
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
#undef TM_S
#undef TM_O
}

}  // namespace llk
