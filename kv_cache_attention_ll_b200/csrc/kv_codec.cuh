// kv_codec.cuh - the cache formats' encoders, shared by the append/recache
// kernels, the fused append of the attention kernel and the FP8 K/V exchange.
//
// Formats (LongLive-2.0 explainer, wmrh.cn, sec. 15.2: the history KV cache
// kept in low precision): bf16 as is; FP8 E4M3 codes with one power-of-two
// scale per (token, head) row; NVFP4 E2M1 codes with one E4M3 scale per block
// of 16 values. Rounding is round-to-nearest-even with saturation, by the
// hardware conversions.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace llk {

enum CacheFormat : int { FMT_BF16 = 0, FMT_FP8 = 1, FMT_NVFP4 = 2 };

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

}  // namespace llk
