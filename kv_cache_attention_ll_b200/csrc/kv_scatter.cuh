// kv_scatter.cuh - append/evict and KV-recache writes into the ring cache.
//
// Both operations copy whole frames of token-major K/V ([tokens][H][D] bf16, as
// a QKV projection emits them) into the head-major cache planes
// ([plane][slots][D], plane = (layer*2 + kv)*H + head), frame f of the source
// landing in the frame slot that cache_layout.cuh assigns:
//   append  (LongLive explainer, dpshk.com, sec. 五/六: sink kept, oldest window
//            frame evicted; LongLive-2.0 explainer, wmrh.cn, sec. 16: shot sink):
//            global sink, else the current shot's sink while it has room, else
//            the next ring slot (append_slot)
//   recache (dpshk.com sec. 三.5; techwalker.com LONGLIVE article sec. 六): logical
//            frame k of the held context (global sink, shot sink, window) to its
//            slot (logical_slot)
// Work split: the source rows ((token, head) pairs, D values each) are cut
// into units of kRows rows of K and the same rows of V (8 KB of bf16 each for
// an append, 16 KB for a recache), and every CTA owns a contiguous range of
// units. A producer warp copies whole units into shared memory with
// cp.async.bulk (one instruction per unit of K or V, completion counted on the
// stage's mbarrier), so each CTA has kStages units in flight once it has read
// the layer's counters; eight consumer warps take a stage, convert its
// rows and store them to their planes, then hand the stage back. Everything
// that depends on a layer's frame counters (the destination slot of a frame,
// or that nothing is stored) is decided by the producer, once per unit.
// A row is handled by D/16 consecutive lanes, 16 values each, so an FP8 row
// maximum takes log2(D/16) shuffle rounds, an NVFP4 block is one lane's values,
// and each row is written as one contiguous run of its plane.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "cache_layout.cuh"
#include "kv_codec.cuh"
#include "sm100_ptx.cuh"

namespace llk {

enum ScatterMode : int { SCATTER_APPEND = 0, SCATTER_RECACHE = 1 };

struct ScatterParams {
  const uint4 *src_k;        // [n_layers][n_frames*T][H][D] bf16
  const uint4 *src_v;
  uint8_t *data;             // cache data base (all layers)
  uint8_t *scales;           // cache scale base (quantised formats) or null
  int H, D, T, slots;        // slots = (G+Ss+R)*T rows per plane
  int layer0;                // first destination layer
  int n_layers;              // source layers (consecutive destination layers)
  int n_frames;              // frames per source layer
  int mode;                  // ScatterMode
  int G, Ss, W, R, F;        // cache geometry: global sink, shot sink, window, ring slots, chunk frames
  int first;                 // recache: first logical frame
  LayerCtr *ctr;             // per-layer counters (device); append advances its layer's
  unsigned *done;            // per-layer count of append units whose counters were read (zero
                             // between launches), kept away from the counters that CTAs read
  unsigned *err;             // status word: recache beyond the held frames, a wait that gave up
  long long planes;          // planes of the cache (L*2*H), for the bounds-checking build
};

// Tile of the bulk scatter for head dimension D, with PASSES passes of the 8
// consumer warps per unit: 8 KB units (6 stages, 2 CTAs per SM) for the
// append, where the launch is short and small units spread it over more CTAs;
// 16 KB units (2 stages, 3 CTAs per SM) for the recache, a long stream where
// fewer, larger copies and more converting warps per SM pay.
template <int D, int PASSES>
struct ScatterTile {
  static constexpr int kLPR = D / 16;                   // lanes per row, 16 values each
  static constexpr int kPasses = PASSES;
  static constexpr int kPassRows = 256 / kLPR;          // rows of one pass
  static constexpr int kRows = kPasses * kPassRows;     // rows per unit
  static constexpr int kRowBytes = D * 2;               // one bf16 source row
  static constexpr int kUnitBytes = kRows * kRowBytes;  // kPasses x 8 KB of K (and as much of V)
  static constexpr int kStages = PASSES == 2 ? 2 : 6;
  static constexpr int kCtasPerSm = PASSES == 2 ? 3 : 2;
  static constexpr int kThreads = 288;                  // warps 0-7 consume, warp 8 produces
  // stages, then per stage a full and an empty barrier (8 bytes each) and a
  // unit record (16 bytes), then the abort flag (16 bytes), then the NVFP4
  // reciprocal table (128 floats)
  static constexpr int kBookBytes = kStages * (8 + 8 + 16) + 16 + 512;
  static constexpr int kSmem = kStages * 2 * kUnitBytes + kBookBytes;
  static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

// x / b from the correctly rounded reciprocal inv = 1/b: q = x * inv, the
// residual r = x - q * b (exact, one fma), then q + r * inv rounded once
// (Markstein's correction step), with the sign of x kept for x = -0. Away from
// underflow this is the correctly rounded quotient; for the NVFP4 operands
// (bf16 x, b an E4M3 value >= 2^-9 or 6) it can differ from it only where the
// residual is subnormal (|x| < 2^-103, so |x / b| < 2^-94), where every E2M1
// or E4M3 rounding gives zero.
__device__ __forceinline__ float div_corrected(float x, float b, float inv) {
  const float q = __fmul_rn(x, inv);
  const float r = __fmaf_rn(-q, b, x);
  return copysignf(__fmaf_rn(r, inv, q), x);
}

__device__ __forceinline__ float div_by_6(float x) {
  constexpr float kInv6 = 1.0f / 6.0f;   // correctly rounded at compile time
  return div_corrected(x, 6.0f, kInv6);
}

// E4M3 code of one fp32 value (round to nearest even, saturating)
__device__ __forceinline__ uint32_t e4m3_code(float y) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(y));
  return h & 0xFFu;
}

// One lane's 16 consecutive values (lo: the first 8, hi: the next 8) of row
// `row` (= plane * slots + slot row) of a plane, quantised and stored (FP8 or
// NVFP4). The kLPR lanes of a row are consecutive lanes and every lane of the
// warp calls it: the FP8 row maximum is reduced with shuffles. Lanes with
// act = false take part in the shuffles and store nothing.
template <int FMT, int D>
__device__ __forceinline__ void store_row16(uint8_t *data, uint8_t *scales, long long row, int j, const uint4 &lo,
                                            const uint4 &hi, bool act, const float *rcp_tab) {
  constexpr int kLPR = D / 16;
  static_assert(FMT == FMT_FP8 || FMT == FMT_NVFP4, "quantised formats only");
  float x0[8], x1[8];
  bf16x8_to_f32(lo, x0);
  bf16x8_to_f32(hi, x1);
  float m0 = 0.f, m1 = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    m0 = fmaxf(m0, fabsf(x0[e]));
    m1 = fmaxf(m1, fabsf(x1[e]));
  }
  float amax = fmaxf(m0, m1);
  if constexpr (FMT == FMT_FP8) {
    // per (token, head) row: scale = the smallest power of two 2^k with
    // amax <= 448 * 2^k, k >= -124 (1 if amax == 0); codes = E4M3(x * 2^-k)
#pragma unroll
    for (int o = 1; o < kLPR; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int k = fp8_scale_log2(amax);
    const float scale = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x0[e] = __fmul_rn(x0[e], inv);
      x1[e] = __fmul_rn(x1[e], inv);
    }
    const uint2 c0 = e4m3x8(x0), c1 = e4m3x8(x1);
    if (act) {
      *reinterpret_cast<uint4 *>(data + row * D + 16 * j) = make_uint4(c0.x, c0.y, c1.x, c1.y);
      if (j == 0) reinterpret_cast<float *>(scales)[row] = scale;
    }
  } else {
    // NVFP4: the lane's 16 values are one block: sb = E4M3(amax/6);
    // codes = E2M1(x / sb), round to nearest even, all +0 if sb == 0. Both
    // quotients are a product with the correctly rounded reciprocal,
    // corrected once with the exact residual (div_by_6 and below); the codes
    // are those of the IEEE quotients for every bf16 input and E4M3 scale.
    const uint32_t sb_code = e4m3_code(div_by_6(amax));
    const float sb = e4m3_to_f32(sb_code);
    uint32_t c0 = 0u, c1 = 0u;
    if (sb != 0.f) {
      const float inv = rcp_tab[sb_code];   // the correctly rounded 1 / sb
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x0[e] = div_corrected(x0[e], sb, inv);
        x1[e] = div_corrected(x1[e], sb, inv);
      }
      c0 = e2m1x8(x0);
      c1 = e2m1x8(x1);
    }
    if (act) {
      *reinterpret_cast<uint2 *>(data + row * (D / 2) + 8 * j) = make_uint2(c0, c1);
      scales[row * (D / 16) + j] = static_cast<uint8_t>(sb_code);
    }
  }
}

template <int FMT, int D, int PASSES>
__global__ void __launch_bounds__(ScatterTile<D, PASSES>::kThreads, ScatterTile<D, PASSES>::kCtasPerSm) kv_scatter_kernel(const ScatterParams q) {
  using C = ScatterTile<D, PASSES>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kStages * 2 * C::kUnitBytes);
  uint64_t *empty = full + C::kStages;
  int4 *unit_rec = reinterpret_cast<int4 *>(empty + C::kStages);   // (layer, slot or -1, first row, rows)
  volatile int *abort_flag = reinterpret_cast<volatile int *>(unit_rec + C::kStages);
  float *rcp_tab = reinterpret_cast<float *>(smem + C::kStages * 2 * C::kUnitBytes + C::kStages * 32 + 16);

  const int rows_frame = q.T * q.H;                               // source rows of one frame
  const int per_frame = (rows_frame + C::kRows - 1) / C::kRows;   // units of one frame
  const long long per_layer = static_cast<long long>(q.n_frames) * per_frame;
  const long long n_units = q.n_layers * per_layer;
  const long long u0 = n_units * blockIdx.x / gridDim.x;
  const long long u1 = n_units * (blockIdx.x + 1) / gridDim.x;
  const int n_my = static_cast<int>(u1 - u0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 8) {
    if (lane != 0) return;
    // ---- producer: per unit, the slot of its frame (from the layer's
    // counters, read when the CTA enters the layer), the unit record, the
    // arrival with the byte count, and the two bulk copies ----
    const char *src_k = reinterpret_cast<const char *>(q.src_k);
    const char *src_v = reinterpret_cast<const char *>(q.src_v);
    const long long src_rows = q.n_layers * static_cast<long long>(q.n_frames) * rows_frame;
    (void)src_rows;                  // read by the bounds-checking build only
    int issued = 0;                  // units handed to the consumers (in order)
    int cur = -1, shot_fill = 0;
    long long p = 0, ring_count = 0, ring_start = 0;
    HeldFrames hf{0, 0, 0};
    bool reject = false;
    unsigned count_pending = 0;      // append: this CTA's units of layer `cur`, not yet counted
    // The completion count of layer `cur` (append), taken when the CTA leaves
    // the layer or has armed all its units: off the path of the copies and
    // arrivals. The CTA whose count completes the layer advances its counters.
    auto count_layer = [&]() {
      if (!count_pending) return;
      __threadfence();               // this CTA's counter read before its count
      const unsigned prev = atomicAdd(q.done + cur, count_pending);
      if (prev + count_pending == static_cast<unsigned>(per_layer)) {
        int fill;
        long long rc;
        append_advance(p, shot_fill, ring_count, q.G, q.Ss, q.F, &fill, &rc);
        LayerCtr *c = q.ctr + cur;
        c->p = p + q.F;
        c->shot_fill = fill;
        c->ring_count = rc;
        q.done[cur] = 0;
        __threadfence();
      }
      count_pending = 0;
    };
    for (int jj = 0; jj < n_my; ++jj) {
      const long long u = u0 + jj;
      const int li = static_cast<int>(u / per_layer);
      const int rem = static_cast<int>(u - li * per_layer);
      const int fi = rem / per_frame;
      const int row0 = (rem - fi * per_frame) * C::kRows;
      const int nrows = rows_frame - row0 < C::kRows ? rows_frame - row0 : C::kRows;
      const long long srow = (static_cast<long long>(li) * q.n_frames + fi) * rows_frame + row0;
      const int layer = q.layer0 + li;
      if (layer != cur) {
        // the layer's counters, read once per CTA and layer before this CTA's
        // completion count: the append's advance (by the CTA whose count
        // completes the layer) comes after every CTA's read
        count_layer();
        cur = layer;
        const LayerCtr *lc = q.ctr + layer;
        p = __ldcg(&lc->p);
        ring_count = __ldcg(&lc->ring_count);
        ring_start = __ldcg(&lc->ring_start);
        shot_fill = __ldcg(&lc->shot_fill);
        if (q.mode == SCATTER_APPEND) {
          const long long end = u1 < (li + 1) * per_layer ? u1 : (li + 1) * per_layer;
          count_pending = static_cast<unsigned>(end - u);
        } else {
          hf = held_frames(p, shot_fill, ring_count, ring_start, q.G, q.W);
          // recache of frames the layer does not hold: nothing of that layer is written
          reject = q.first + q.n_frames > hf.g + hf.sf + hf.w;
          if (reject && rem == 0) atomicOr(q.err, KID_SCATTER | ERR_RANGE);
        }
      }
      if (*abort_flag) continue;     // keep the completion counts of the remaining layers
      int slot;
      if (q.mode == SCATTER_APPEND) slot = append_slot(p, shot_fill, ring_count, q.G, q.Ss, q.R, q.F, fi);
      else slot = reject ? -1 : logical_slot(hf, ring_count, q.G, q.Ss, q.R, q.first + fi);
      if (slot >= 0 && !LL_BOUNDS(srow >= 0 && srow + nrows <= src_rows, q.err, KID_SCATTER)) slot = -1;
      const int s = jj % C::kStages;
      if (jj >= C::kStages &&
          !mbar_wait(&empty[s], ((jj / C::kStages) - 1) & 1, abort_flag, q.err, KID_SCATTER))
        continue;
      unit_rec[s] = make_int4(layer, slot, row0, nrows);
      if (slot >= 0) {
        const uint32_t bytes = static_cast<uint32_t>(nrows) * C::kRowBytes;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_load(smem + (2 * s) * C::kUnitBytes, src_k + srow * C::kRowBytes, bytes, &full[s]);
        bulk_load(smem + (2 * s + 1) * C::kUnitBytes, src_v + srow * C::kRowBytes, bytes, &full[s]);
      } else {
        mbar_arrive(&full[s]);       // nothing to copy: the consumers skip the unit
      }
      issued = jj + 1;
    }
    count_layer();
    // after an abort, copies may still be landing in this CTA's shared memory:
    // wait (bounded) for the last phase issued on each stage before exiting
    if (*abort_flag)
      for (int jj = issued - C::kStages < 0 ? 0 : issued - C::kStages; jj < issued; ++jj)
        mbar_wait_drain(&full[jj % C::kStages], (jj / C::kStages) & 1);
    return;
  }

  // ---- consumers: warps 0-7, rows r0 + kPassRows * pass of each unit, 16 values per lane ----
  if constexpr (FMT == FMT_NVFP4) {
    // 1 / sb for every E4M3 block-scale code (code 0 is never a divisor), filled
    // while the first copies are in flight; the eight warps alone meet here
    if (threadIdx.x < 128) rcp_tab[threadIdx.x] = threadIdx.x == 0 ? 0.f : __frcp_rn(e4m3_to_f32(threadIdx.x));
    named_bar_sync(1, 256);
  }
  const int r0 = threadIdx.x / C::kLPR;
  const int j = threadIdx.x % C::kLPR;
  // the two 16-byte halves of a lane's 32 bytes are read in an order that puts
  // the 8 lanes of each quarter warp on 8 different bank groups
  const int half_first = (threadIdx.x >> 2) & 1;
  for (int jj = 0; jj < n_my; ++jj) {
    const int s = jj % C::kStages;
    if (!mbar_wait(&full[s], (jj / C::kStages) & 1, abort_flag, q.err, KID_SCATTER)) break;
    const int4 rec = unit_rec[s];
#pragma unroll
    for (int pass = 0; pass < C::kPasses; ++pass) {
      if (rec.y < 0) break;
      const int r = r0 + pass * C::kPassRows;
      const int rf = rec.z + r;                  // row inside the frame: token * H + head
      const int t = rf / q.H;
      const int hh = rf - t * q.H;
      const long long plane_k = static_cast<long long>(rec.x) * 2 * q.H + hh;
      const long long drow = static_cast<long long>(rec.y) * q.T + t;
      const bool act = r < rec.w &&
                       LL_BOUNDS(drow < q.slots && plane_k + q.H < q.planes, q.err, KID_SCATTER);
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const long long plane = plane_k + kv * q.H;
        const uint8_t *srow = smem + (2 * s + kv) * C::kUnitBytes + r * C::kRowBytes;
        if constexpr (FMT == FMT_BF16) {
          const uint4 a = *reinterpret_cast<const uint4 *>(srow + 16 * j);
          const uint4 c = *reinterpret_cast<const uint4 *>(srow + 16 * (j + C::kLPR));
          if (act) {
            uint4 *d = reinterpret_cast<uint4 *>(q.data + (plane * q.slots + drow) * D * 2);
            d[j] = a;
            d[j + C::kLPR] = c;
          }
        } else {
          const uint8_t *src = srow + 32 * j;
          const uint4 a = *reinterpret_cast<const uint4 *>(src + 16 * half_first);
          const uint4 c = *reinterpret_cast<const uint4 *>(src + 16 * (1 - half_first));
          store_row16<FMT, D>(q.data, q.scales, plane * q.slots + drow, j, half_first ? c : a, half_first ? a : c,
                              act, rcp_tab);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace llk

namespace llk {

// ---------------------------------------------------------------------------
// Dequantisation of one layer's held frames into a bf16 view.
//
// The LongLive-2.0 explainer (wmrh.cn, sec. 15.2-15.3) stores the history KV
// cache in FP4 and dequantises it in parallel when it is used. Here the
// visible rows [0, n_rows) of the layer's 2H planes (K then V) are converted
// once per attention call into the cache's bf16 view [2H][slots][D], which the
// bf16 attention kernel then reads through TMA; every query tile of a head
// shares the converted rows instead of converting them again.
//   FP8:   e4m3 -> f16 (exact) -> fp32, times the row scale (a power of two at
//          or above 2^-124): the product has at most 4 significant bits and
//          lies at or above 2^-133, so it and its bf16 conversion are exact
//   NVFP4: e2m1 -> f16 and E4M3 block scale -> f16 (both exact); the product has
//          at most 6 significant bits and lies inside the f16 range, so it is
//          exact, and so is its bf16 conversion.
// One thread writes 8 bf16 values (16 bytes); reads and writes are coalesced.
struct DequantParams {
  const uint8_t *data;     // codes of all layers
  const uint8_t *scales;   // scales of all layers
  uint4 *view;             // [2H][slots][D] bf16
  const LayerCtr *ctr;     // the layer's counters, or null: then rows [0, n_rows) are converted
  int H, D, slots, n_rows;
  int G, Ss, W, R, T;      // with ctr: the visible frame ranges of cache_layout.cuh are converted
  int plane0;              // first plane of the layer: layer * 2H
  long long planes;        // planes of the codes and scales (bounds-checking build)
  unsigned *err;           // status word (bounds-checking build), or null
};

__device__ __forceinline__ uint32_t f16x2_of_e4m3x2(uint32_t two_codes) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(static_cast<uint16_t>(two_codes)));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_of_e2m1x2(uint32_t byte) {
  uint32_t d;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(d) : "r"(byte));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_of_f32(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Grid: blockIdx.y = one of the layer's 2H planes, blockIdx.x strides over the
// plane's visible rows; VPR = D/8 vectors per row is a compile-time constant,
// so the index arithmetic is shifts and masks in 32 bits (rows * VPR < 2^30,
// checked at create).
template <int FMT, int VPR>
__global__ void __launch_bounds__(256) kv_dequant_kernel(const DequantParams q) {
  // visible rows as up to three slot-row ranges; rows are counted through them in order
  int r0 = 0, n0 = q.n_rows, r1 = 0, n1 = 0, r2 = 0, n2 = 0;
  if (q.ctr) {
    const long long ring_count = __ldcg(&q.ctr->ring_count);
    const HeldFrames hf = held_frames(__ldcg(&q.ctr->p), __ldcg(&q.ctr->shot_fill), ring_count,
                                      __ldcg(&q.ctr->ring_start), q.G, q.W);
    const FrameRanges fr = visible_ranges(hf, ring_count, q.G, q.Ss, q.R);
    r0 = fr.start[0] * q.T;
    n0 = fr.len[0] * q.T;
    r1 = fr.start[1] * q.T;
    n1 = fr.len[1] * q.T;
    r2 = fr.start[2] * q.T;
    n2 = fr.len[2] * q.T;
  }
  const int total = (n0 + n1 + n2) * VPR;          // vectors of this plane
  const int lp = blockIdx.y;                        // 0 .. 2H-1
  const long long src_plane = static_cast<long long>(q.plane0 + lp) * q.slots;
  const long long dst_plane = static_cast<long long>(lp) * q.slots;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int vec = i % VPR;
    const int vr = i / VPR;                         // visible row
    const int row = vr < n0 ? r0 + vr : (vr < n0 + n1 ? r1 + (vr - n0) : r2 + (vr - n0 - n1));
    if (!LL_BOUNDS(row >= 0 && row < q.slots && q.plane0 + lp < q.planes, q.err, KID_ATTN)) continue;
    const long long src_row = src_plane + row;
    uint32_t o[4];
    if constexpr (FMT == FMT_FP8) {
      const uint2 c = __ldg(reinterpret_cast<const uint2 *>(q.data + src_row * (VPR * 8)) + vec);
      const float s = __ldg(reinterpret_cast<const float *>(q.scales) + src_row);
      const uint32_t w[2] = {c.x, c.y};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t h2 = f16x2_of_e4m3x2(w[k >> 1] >> (16 * (k & 1)));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
        o[k] = bf16x2_of_f32(f.x * s, f.y * s);
      }
    } else {
      const uint32_t c = __ldg(reinterpret_cast<const uint32_t *>(q.data + src_row * (VPR * 4)) + vec);
      const uint32_t sb = __ldg(q.scales + src_row * (VPR / 2) + (vec >> 1));
      const uint32_t s2 = f16x2_of_e4m3x2(sb * 0x101u);   // the block scale in both halves
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t h2 = f16x2_of_e2m1x2((c >> (8 * k)) & 0xFFu);
        const __half2 prod = __hmul2(*reinterpret_cast<const __half2 *>(&h2), *reinterpret_cast<const __half2 *>(&s2));
        const float2 f = __half22float2(prod);
        o[k] = bf16x2_of_f32(f.x, f.y);
      }
    }
    q.view[(dst_plane + row) * VPR + vec] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace llk
