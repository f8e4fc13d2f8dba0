// sp_exchange.cu - the local halves of the head-sharded sequence-parallel
// attention step (LongLive-2.0 explainer, wmrh.cn, sec. 18.3: sequence
// parallel inference; sec. 15.2: a low-precision KV cache also cuts the
// traffic between GPUs when inference is sequence parallel).
//
// P ranks each hold N_s = N/P tokens of the chunk for all H heads. An
// all-to-all (the caller's collective) turns that into all N tokens for
// H/P heads per rank, which is what a rank's H/P-head cache attends to; a
// second all-to-all brings the outputs back. Around the collectives:
//   pack    [N_s][H][D] -> [P][N_s][H/P][D]: the part for rank r is contiguous,
//           so a plain equal-split all-to-all sends it; what a rank receives,
//           [P][N_s][H/P][D] from ranks 0..P-1, is [N][H/P][D] in token order.
//   unpack  [P][N_s][H/P][D] -> [N_s][H][D]: the inverse, for the outputs.
//   pack_fp8: as pack, but each (token, head) row leaves as E4M3 codes plus
//           one fp32 power-of-two scale (the cache's FP8 row format), so K and
//           V cross the links in D + 4 bytes per row instead of 2D;
//   dequant_fp8: codes x scale back to bf16 (exact) on the receiving side.
// All four move 16-byte vectors with one thread per vector; consecutive
// threads cover consecutive vectors of a row, so reads and writes coalesce.
#include <cuda_runtime.h>

#include <cstdint>

#include "ll_kvattn.h"
#include "kv_codec.cuh"

namespace llk {

// dst row of source row (t, h) for pack, or source row of destination row
// (t, h) for unpack: rank r = h / hp owns heads [r*hp, (r+1)*hp)
__device__ __forceinline__ long long packed_row(int t, int h, int n_s, int hp) {
  const int r = h / hp;
  return (static_cast<long long>(r) * n_s + t) * hp + (h - r * hp);
}

// PACK = true: x [n_s][H][D] -> packed; false: packed -> x. VPR = D/8 vectors per row.
template <bool PACK, int VPR>
__global__ void __launch_bounds__(256) sp_permute_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                         int n_s, int H, int hp, long long n_vec) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int vec = static_cast<int>(i % VPR);
    const long long row = i / VPR;                   // token-major row t*H + h
    const int t = static_cast<int>(row / H);
    const int h = static_cast<int>(row - static_cast<long long>(t) * H);
    const long long prow = packed_row(t, h, n_s, hp);
    if (PACK)
      dst[prow * VPR + vec] = __ldg(src + i);
    else
      dst[i] = __ldg(src + prow * VPR + vec);
  }
}

// FP8 pack: the D/8 lanes of a (token, head) row reduce its maximum with
// shuffles, then each writes its 8 codes; lane 0 of the row writes the scale.
// The trip count is uniform (whole warps), so the shuffles see every lane.
template <int VPR>
__global__ void __launch_bounds__(256) sp_pack_fp8_kernel(const uint4 *__restrict__ src, uint2 *__restrict__ codes,
                                                          float *__restrict__ scales, int n_s, int H, int hp,
                                                          long long n_vec) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long base = blockIdx.x * static_cast<long long>(blockDim.x); base < n_vec; base += stride) {
    const long long i = base + threadIdx.x;
    const bool act = i < n_vec;
    const long long ic = act ? i : 0;
    const int vec = static_cast<int>(ic % VPR);
    const long long row = ic / VPR;
    const int t = static_cast<int>(row / H);
    const int h = static_cast<int>(row - static_cast<long long>(t) * H);
    float x[8];
    bf16x8_to_f32(act ? __ldg(src + ic) : make_uint4(0, 0, 0, 0), x);
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int o = 1; o < VPR; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int k = fp8_scale_log2(amax);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(x[e], inv);
    const uint2 c = e4m3x8(y);
    if (act) {
      const long long prow = packed_row(t, h, n_s, hp);
      codes[prow * VPR + vec] = c;
      if (vec == 0) scales[prow] = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
    }
  }
}

// FP8 rows back to bf16: 8 codes per thread, times the row's power-of-two
// scale (exact), converted to bf16 (exact).
template <int VPR>
__global__ void __launch_bounds__(256) sp_dequant_fp8_kernel(const uint2 *__restrict__ codes,
                                                             const float *__restrict__ scales,
                                                             uint4 *__restrict__ dst, long long n_vec) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint2 c = __ldg(codes + i);
    const float s = __ldg(scales + i / VPR);
    const uint32_t w[2] = {c.x, c.y};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(w[q >> 1] >> (16 * (q & 1)))));
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
      uint32_t d;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(f.y * s), "f"(f.x * s));
      o[q] = d;
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace llk

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// grid of 256-thread blocks for n vectors: at most about 8 blocks per SM
unsigned grid_for(long long n_vec) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long g = (n_vec + 255) / 256;
  const long long cap = static_cast<long long>(sms > 0 ? sms : 148) * 8;
  if (g > cap) g = cap;
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

ll_status check_geometry(int tokens, int heads, int head_dim, int ranks) {
  if (tokens < 0 || heads < 1 || ranks < 1 || heads % ranks != 0) return LL_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LL_ERR_INVALID_ARG;
  if (static_cast<long long>(tokens) * heads >= (1ll << 31)) return LL_ERR_INVALID_ARG;
  return LL_OK;
}

}  // namespace

extern "C" {

ll_status ll_sp_pack_heads(const void *x, int tokens, int heads, int head_dim, int ranks, void *packed,
                           ll_stream_t stream) {
  const ll_status g = check_geometry(tokens, heads, head_dim, ranks);
  if (g != LL_OK) return g;
  if (!x || !packed || !aligned16(x) || !aligned16(packed) || x == packed) return LL_ERR_INVALID_ARG;
  const long long n_vec = static_cast<long long>(tokens) * heads * (head_dim / 8);
  if (n_vec == 0) return LL_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int hp = heads / ranks;
  const uint4 *s = static_cast<const uint4 *>(x);
  uint4 *d = static_cast<uint4 *>(packed);
  if (head_dim == 128) llk::sp_permute_kernel<true, 16><<<grid_for(n_vec), 256, 0, st>>>(s, d, tokens, heads, hp, n_vec);
  else llk::sp_permute_kernel<true, 8><<<grid_for(n_vec), 256, 0, st>>>(s, d, tokens, heads, hp, n_vec);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status ll_sp_unpack_heads(const void *packed, int tokens, int heads, int head_dim, int ranks, void *x,
                             ll_stream_t stream) {
  const ll_status g = check_geometry(tokens, heads, head_dim, ranks);
  if (g != LL_OK) return g;
  if (!x || !packed || !aligned16(x) || !aligned16(packed) || x == packed) return LL_ERR_INVALID_ARG;
  const long long n_vec = static_cast<long long>(tokens) * heads * (head_dim / 8);
  if (n_vec == 0) return LL_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int hp = heads / ranks;
  const uint4 *s = static_cast<const uint4 *>(packed);
  uint4 *d = static_cast<uint4 *>(x);
  if (head_dim == 128) llk::sp_permute_kernel<false, 16><<<grid_for(n_vec), 256, 0, st>>>(s, d, tokens, heads, hp, n_vec);
  else llk::sp_permute_kernel<false, 8><<<grid_for(n_vec), 256, 0, st>>>(s, d, tokens, heads, hp, n_vec);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status ll_sp_pack_heads_fp8(const void *x, int tokens, int heads, int head_dim, int ranks, void *codes,
                               void *scales, ll_stream_t stream) {
  const ll_status g = check_geometry(tokens, heads, head_dim, ranks);
  if (g != LL_OK) return g;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes) || !aligned16(scales)) return LL_ERR_INVALID_ARG;
  const long long n_vec = static_cast<long long>(tokens) * heads * (head_dim / 8);
  if (n_vec == 0) return LL_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int hp = heads / ranks;
  const uint4 *s = static_cast<const uint4 *>(x);
  uint2 *c = static_cast<uint2 *>(codes);
  float *sc = static_cast<float *>(scales);
  if (head_dim == 128) llk::sp_pack_fp8_kernel<16><<<grid_for(n_vec), 256, 0, st>>>(s, c, sc, tokens, heads, hp, n_vec);
  else llk::sp_pack_fp8_kernel<8><<<grid_for(n_vec), 256, 0, st>>>(s, c, sc, tokens, heads, hp, n_vec);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status ll_sp_dequant_fp8(const void *codes, const void *scales, long long rows, int head_dim, void *x,
                            ll_stream_t stream) {
  if (rows < 0 || (head_dim != 64 && head_dim != 128) || rows >= (1ll << 31)) return LL_ERR_INVALID_ARG;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes) || !aligned16(scales)) return LL_ERR_INVALID_ARG;
  const long long n_vec = rows * (head_dim / 8);
  if (n_vec == 0) return LL_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint2 *c = static_cast<const uint2 *>(codes);
  const float *sc = static_cast<const float *>(scales);
  uint4 *d = static_cast<uint4 *>(x);
  if (head_dim == 128) llk::sp_dequant_fp8_kernel<16><<<grid_for(n_vec), 256, 0, st>>>(c, sc, d, n_vec);
  else llk::sp_dequant_fp8_kernel<8><<<grid_for(n_vec), 256, 0, st>>>(c, sc, d, n_vec);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

}  // extern "C"
