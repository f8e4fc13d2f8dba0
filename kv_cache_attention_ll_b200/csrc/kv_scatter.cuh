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
// Grid: blockIdx.x = one (source layer, source frame) pair, blockIdx.y strides
// over that frame's T*H*D/8 16-byte vectors. Everything that depends on the
// layer's frame counter (the destination slot, or that nothing is stored) is
// decided once per block. One thread moves one vector (8 values) of K and the
// same vector of V; the D/8 threads of one (token, head) row are consecutive
// lanes, so reads are fully coalesced and each row is written as one
// contiguous 128/256-byte run.
// Quantising formats reduce the row (FP8) or the 16-value block (NVFP4) with
// lane shuffles inside that group and write codes + scales.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "cache_layout.cuh"
#include "sm100_ptx.cuh"

namespace llk {

enum ScatterMode : int { SCATTER_APPEND = 0, SCATTER_RECACHE = 1 };
enum CacheFormat : int { FMT_BF16 = 0, FMT_FP8 = 1, FMT_NVFP4 = 2 };

struct ScatterParams {
  const uint4 *src_k;        // [n_layers][n_frames*T][H][D] bf16
  const uint4 *src_v;
  uint8_t *data;             // cache data base (all layers)
  uint8_t *scales;           // cache scale base (quantised formats) or null
  int frame_vec;             // T * H * (D/8): vectors of one frame (< 2^30)
  int H, D, T, slots;        // slots = (S+W)*T per plane
  int layer0;                // first destination layer
  int n_frames;              // frames per source layer
  int mode;                  // ScatterMode
  int G, Ss, W, R, F;        // cache geometry: global sink, shot sink, window, ring slots, chunk frames
  int first;                 // recache: first logical frame
  LayerCtr *ctr;             // per-layer counters (device); append advances its layer's
  unsigned *done;            // per-layer count of finished append blocks (zero between launches),
                             // kept away from the counters that every block reads
  unsigned *err;             // status word: recache beyond the held frames is flagged there
  long long planes;          // planes of the cache (L*2*H), for the bounds-checking build
  long long src_vec;         // 16-byte vectors of the source (all source layers and frames)
};

// 8 fp32 -> 8 E4M3 codes (round to nearest even, saturating), element 0 in byte 0
__device__ __forceinline__ uint2 e4m3x8(const float (&y)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(y[2 * i + 1]), "f"(y[2 * i]));
    w[i] = h;
  }
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// 8 fp32 -> 8 E2M1 codes packed in 4 bytes, element 2i in the low nibble of byte i
__device__ __forceinline__ uint32_t e2m1x8(const float (&y)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

// one E4M3 code -> its fp32 value (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  // the code sits in both bytes, so either half of the f16 pair holds its value
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>((code & 0xFF) * 0x101u)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFF)));
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// log2 of the FP8 row scale: the smallest k >= -124 with amax <= 448 * 2^k
// (0 for amax == 0). amax lies in [2^E, 2^(E+1)), so amax/448 lies in
// (2^(E-9), 2^(E-7)) and k is E-8 or E-7: E-8 exactly when amax <= 448 * 2^(E-8)
// = 1.75 * 2^E. Below 2^-118 the floor applies (amax/448 < 2^-126).
__device__ __forceinline__ int fp8_scale_log2(float amax) {
  if (amax == 0.f) return 0;
  const int eb = static_cast<int>(__float_as_uint(amax) >> 23);   // biased exponent, amax >= 0
  if (eb < 9) return -124;
  const float thr = __uint_as_float((static_cast<uint32_t>(eb) << 23) | 0x600000u);   // 1.75 * 2^E
  const int k = eb - 127 - 8 + (amax > thr ? 1 : 0);
  return k < -124 ? -124 : k;
}

// Stores one 16-byte vector (8 values) of K and the same vector of V of one
// (token, head) row at row `drow` of planes plane_k / plane_v, quantising for
// FP8 (per-row scale) and NVFP4 (16-value blocks). The D/8 lanes of a row must
// be consecutive lanes of the warp, and every lane of the warp must call it:
// the quantising formats reduce with shuffles. Lanes with act = false take
// part in the shuffles and store nothing.
template <int FMT>
__device__ __forceinline__ void store_kv_vec(uint8_t *data, uint8_t *scales, long long plane_k, long long plane_v,
                                             int slots, long long drow, int D, int vec, uint4 vk, uint4 vv,
                                             bool act) {
  const int vpr = D >> 3;
  if constexpr (FMT == FMT_BF16) {
    if (act) {
      uint4 *dk = reinterpret_cast<uint4 *>(data) + (plane_k * slots + drow) * vpr + vec;
      uint4 *dv = reinterpret_cast<uint4 *>(data) + (plane_v * slots + drow) * vpr + vec;
      *dk = vk;
      *dv = vv;
    }
  } else if constexpr (FMT == FMT_FP8) {
    // per (token, head) row: scale = the smallest power of two 2^k with
    // amax <= 448 * 2^k, k >= -124 (1 if amax == 0); codes = E4M3(x * 2^-k).
    // Both the quotient and code x scale are then exact (the latter in bf16).
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      float x[8];
      bf16x8_to_f32(kv == 0 ? vk : vv, x);
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
      for (int o = 1; o < vpr; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const int k = fp8_scale_log2(amax);
      const float scale = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
      const float inv = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(x[e], inv);
      const uint2 codes = e4m3x8(y);
      if (act) {
        const long long plane = kv == 0 ? plane_k : plane_v;
        uint2 *dc = reinterpret_cast<uint2 *>(data + (plane * slots + drow) * D) + vec;
        *dc = codes;
        if (vec == 0) reinterpret_cast<float *>(scales)[plane * slots + drow] = scale;
      }
    }
  } else {
    // NVFP4: per 16-value block (two lanes): sb = E4M3(amax/6); codes = E2M1(x / sb)
    // (IEEE division, then the hardware round-to-nearest-even), all +0 if sb == 0
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      float x[8];
      bf16x8_to_f32(kv == 0 ? vk : vv, x);
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      float sv[8] = {__fdiv_rn(amax, 6.0f), 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint32_t sb_code = e4m3x8(sv).x & 0xFFu;
      const float sb = e4m3_to_f32(sb_code);
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = sb == 0.f ? 0.f : __fdiv_rn(x[e], sb);
      const uint32_t codes = sb == 0.f ? 0u : e2m1x8(y);
      if (act) {
        const long long plane = kv == 0 ? plane_k : plane_v;
        uint32_t *dc = reinterpret_cast<uint32_t *>(data + (plane * slots + drow) * (D / 2)) + vec;
        *dc = codes;
        if ((vec & 1) == 0) scales[(plane * slots + drow) * (D / 16) + (vec >> 1)] = static_cast<uint8_t>(sb_code);
      }
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(256) kv_scatter_kernel(const ScatterParams q) {
  const int vpr = q.D >> 3;                    // vectors per (token, head) row: 8 or 16
  const int lg_vpr = vpr == 16 ? 4 : 3;
  const int li = blockIdx.x / q.n_frames;      // source layer
  const int fi = blockIdx.x % q.n_frames;      // source frame
  const int layer = q.layer0 + li;
  const long long src0 = static_cast<long long>(blockIdx.x) * q.frame_vec;   // first vector of the frame
  const int stride = gridDim.y * blockDim.x;
  // the source does not depend on the counters: each thread loads its first
  // vectors now, while thread 0 reads the counters, and then stays one
  // iteration ahead
  uint4 nk = make_uint4(0, 0, 0, 0), nv = make_uint4(0, 0, 0, 0);
  {
    const int i0 = blockIdx.y * blockDim.x + threadIdx.x;
    if (i0 < q.frame_vec) {
      nk = __ldg(q.src_k + src0 + i0);
      nv = __ldg(q.src_v + src0 + i0);
    }
  }
  // the layer's counters, read once per block by thread 0 before the block's
  // completion count below, so the append's advance (by the last block) comes
  // after every block's read
  __shared__ LayerCtr blk_ctr;
  if (threadIdx.x == 0) {
    const LayerCtr *lc = q.ctr + layer;
    blk_ctr.p = __ldcg(&lc->p);
    blk_ctr.ring_count = __ldcg(&lc->ring_count);
    blk_ctr.ring_start = __ldcg(&lc->ring_start);
    blk_ctr.shot_fill = __ldcg(&lc->shot_fill);
  }
  __syncthreads();
  const long long p = blk_ctr.p;
  const long long ring_count = blk_ctr.ring_count;
  const long long ring_start = blk_ctr.ring_start;
  const int shot_fill = blk_ctr.shot_fill;
  int slot;
  if (q.mode == SCATTER_APPEND) {
    slot = append_slot(p, shot_fill, ring_count, q.G, q.Ss, q.R, q.F, fi);
  } else {
    const HeldFrames hf = held_frames(p, shot_fill, ring_count, ring_start, q.G, q.W);
    // recache of frames the layer does not hold: nothing of that layer is written
    const bool reject = q.first + q.n_frames > hf.g + hf.sf + hf.w;
    if (reject && fi == 0 && blockIdx.y == 0 && threadIdx.x == 0) atomicOr(q.err, KID_SCATTER | ERR_RANGE);
    slot = reject ? -1 : logical_slot(hf, ring_count, q.G, q.Ss, q.R, q.first + fi);
  }
  // block-uniform trip count (slot is uniform too): every lane runs every
  // iteration, so the row-group shuffles of the quantising formats see all 32
  for (int base = slot < 0 ? q.frame_vec : blockIdx.y * blockDim.x; base < q.frame_vec; base += stride) {
    const int i = base + threadIdx.x;
    const bool act = i < q.frame_vec;
    const int ic = act ? i : 0;
    const int vec = ic & (vpr - 1);
    const int row = ic >> lg_vpr;                           // token * H + head
    const int t = row / q.H;
    const int hh = row - t * q.H;
    const long long plane_k = (static_cast<long long>(layer) * 2 + 0) * q.H + hh;
    const long long plane_v = plane_k + q.H;
    const long long drow = static_cast<long long>(slot) * q.T + t;   // row inside a plane
    const uint4 vk = nk, vv = nv;                             // this iteration's vectors (loaded ahead)
    if (i + stride < q.frame_vec) {
      nk = __ldg(q.src_k + src0 + i + stride);
      nv = __ldg(q.src_v + src0 + i + stride);
    }
    const bool in = LL_BOUNDS(drow >= 0 && drow < q.slots && plane_v < q.planes && src0 + ic < q.src_vec, q.err,
                              KID_SCATTER);
    store_kv_vec<FMT>(q.data, q.scales, plane_k, plane_v, q.slots, drow, q.D, vec, vk, vv, act && in);
  }
  if (q.mode == SCATTER_APPEND) {
    // per layer, the last of its n_frames x gridDim.y blocks to finish advances
    // the layer's counters; every block read them above, before its increment
    // of the layer's completion count
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      LayerCtr *c = q.ctr + layer;
      const unsigned prev = atomicAdd(q.done + layer, 1u);
      if (prev == static_cast<unsigned>(q.n_frames) * gridDim.y - 1) {
        int fill;
        long long rc;
        append_advance(p, shot_fill, ring_count, q.G, q.Ss, q.F, &fill, &rc);
        c->p = p + q.F;
        c->shot_fill = fill;
        c->ring_count = rc;
        q.done[layer] = 0;
        __threadfence();
      }
    }
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
