// ll_kvattn.cu - host side of the C ABI declared in include/ll_kvattn.h:
// the cache object (one device allocation per cache, zero-filled, never grown),
// argument validation, TMA descriptor setup and the kernel launches.
//
// Frame counters live in device memory: the kernels read a layer's p there and
// the append kernel advances it, so a captured sequence of calls stays right
// when it is replayed. The host keeps a mirror for argument checks and
// ll_kv_cache_info until an append is enqueued inside a stream capture; from
// then on replays move the device counters without the host seeing them, so
// info reads the device and recache range checks happen in the kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "ll_kvattn.h"
#include "attn_sink_window.cuh"
#include "kv_scatter.cuh"

struct ll_kv_cache {
  int L, H, D, T, F, S, W;
  int Ss;                     // shot-sink frames (0: a single-shot cache)
  int R;                      // ring slots: W, or W + F for a cache made for fused append
  ll_kv_dtype dtype;
  int device;
  long long slots;            // (S+Ss+R)*T rows per plane
  uint8_t *base;              // the one allocation
  size_t bytes;               // its size
  uint8_t *data;              // [L][2][H][slots][row bytes]
  uint8_t *scales;            // quantised formats: [L][2][H][slots][...]
  unsigned *err;              // device status word
  size_t data_plane_bytes;    // bytes of one plane's data
  size_t scale_plane_bytes;   // bytes of one plane's scales
  std::vector<llk::LayerCtr> hc;  // host mirror of the counters (exact while host_counters)
  bool host_counters;         // false once an append or shot start was enqueued inside a stream capture
  llk::LayerCtr *ctr;         // device counters [L]
  unsigned *done;             // device append-completion counts [L] (own cache lines)
  CUtensorMap tm_cache;       // bf16 cache planes (D, slots, L*2*H)
  uint8_t *view;              // quantised caches: bf16 view of one layer [2H][slots][D]
  CUtensorMap tm_view;        // (D, slots, 2H) over the view
  std::vector<std::pair<size_t, size_t>> guards;  // canary ranges [begin, end) of the allocation
};

namespace {

std::atomic<long long> g_alloc_count{0};

// every region of a cache allocation is followed by a guard of this many extra
// bytes (beyond the padding to 256), filled with kCanary at create
constexpr size_t kGuardBytes = 256;
constexpr int kCanary = 0xA5;

bool test_fail_alloc() {
  const char *v = std::getenv("LL_KVATTN_TEST_FAIL_ALLOC");
  return v && v[0] && !(v[0] == '0' && v[1] == 0);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernels of a cache run on the device that owns it: a launch on another
// current device would reach memory of a device it may not be able to access.
bool on_cache_device(const ll_kv_cache *c) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == c->device;
}

// 3-D bf16 tensor map: dims (d0 innermost, d1, d2), strides of d1 and d2 in bytes,
// box (b0, b1, b2), 128-byte swizzle, zero fill outside the tensor.
bool make_map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                 uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// key rows per attention tile: every TMA box of keys (and of queries) is 64
// head-dim columns x kKeyTile rows
constexpr uint32_t kKeyTile = llk::AttnCfg<128>::BN;

// token-major activation [Tq][H][D] viewed as (D, H, Tq), box (64, 1, kKeyTile)
bool make_act_map(CUtensorMap *m, const void *p, int Tq, int H, int D) {
  return make_map_3d(m, p, D, H, Tq, static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(H) * D * 2, 64, 1, kKeyTile);
}

// held frames of a layer according to the host mirror
llk::HeldFrames held(const ll_kv_cache *c, int layer) {
  const llk::LayerCtr &h = c->hc[layer];
  return llk::held_frames(h.p, h.shot_fill, h.ring_count, h.ring_start, c->S, c->W);
}

// counter updates of one append of layer `layer` on the host mirror; an append
// enqueued inside a stream capture ends the mirror's exactness
void mirror_append(ll_kv_cache *c, int layer, cudaStreamCaptureStatus cs) {
  llk::LayerCtr &h = c->hc[layer];
  int fill = 0;
  long long rc = 0;
  llk::append_advance(h.p, h.shot_fill, h.ring_count, c->S, c->Ss, c->F, &fill, &rc);
  h.p += c->F;
  h.shot_fill = fill;
  h.ring_count = rc;
  if (cs != cudaStreamCaptureStatusNone) c->host_counters = false;
}

// the device counters of one layer (after a device-wide synchronisation)
bool read_device_counters(const ll_kv_cache *c, int layer, llk::LayerCtr *out) {
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(c->device) != cudaSuccess) return false;
  const bool ok = cudaDeviceSynchronize() == cudaSuccess &&
                  cudaMemcpy(out, c->ctr + layer, sizeof(*out), cudaMemcpyDeviceToHost) == cudaSuccess;
  cudaSetDevice(prev);
  return ok;
}

int num_sms(int device) {
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
  return n > 0 ? n : 148;
}

// Raises a kernel's dynamic shared-memory limit once per device (devices 0..63
// remembered in `mask`; any other device sets it on every call).
template <typename K>
bool ensure_smem(K kernel, int bytes, std::atomic<unsigned long long> &mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  if (bit && (mask.load() & bit)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  mask.fetch_or(bit);
  return true;
}

template <int D>
bool prepare_attn() {
  static std::atomic<unsigned long long> configured{0};
  return ensure_smem(llk::attn_sink_window_kernel<D>, llk::AttnCfg<D>::SMEM_ALLOC, configured);
}

template <int FMT, int D, int PASSES>
bool prepare_scatter() {
  static std::atomic<unsigned long long> configured{0};
  return ensure_smem(llk::kv_scatter_kernel<FMT, D, PASSES>, llk::ScatterTile<D, PASSES>::kSmem, configured);
}

template <int D>
ll_status launch_attn(const llk::AttnParams &prm, int grid, cudaStream_t stream) {
  using C = llk::AttnCfg<D>;
  if (!prepare_attn<D>()) return LL_ERR_CUDA;
  llk::attn_sink_window_kernel<D><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(prm);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

// Quantised caches: the layer's held rows of K and V (their number follows the
// layer's device counter), dequantised into the cache's bf16 view.
// Grid (x, 2H): x-blocks stride over one plane's visible rows, one y per plane;
// about 8 blocks of 256 threads per SM in all.
ll_status launch_dequant_kernel(const llk::DequantParams &q, ll_kv_dtype dtype, int device, cudaStream_t stream) {
  const long long plane_blocks = (static_cast<long long>(q.slots) * (q.D / 8) + 255) / 256;
  const long long target = static_cast<long long>(num_sms(device)) * 8;
  long long gx = (target + 2 * q.H - 1) / (2 * q.H);
  if (gx > plane_blocks) gx = plane_blocks;
  if (gx < 1) gx = 1;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(2 * q.H));
  if (dtype == LL_KV_FP8_E4M3) {
    if (q.D == 128) llk::kv_dequant_kernel<llk::FMT_FP8, 16><<<grid, 256, 0, stream>>>(q);
    else llk::kv_dequant_kernel<llk::FMT_FP8, 8><<<grid, 256, 0, stream>>>(q);
  } else {
    if (q.D == 128) llk::kv_dequant_kernel<llk::FMT_NVFP4, 16><<<grid, 256, 0, stream>>>(q);
    else llk::kv_dequant_kernel<llk::FMT_NVFP4, 8><<<grid, 256, 0, stream>>>(q);
  }
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status launch_dequant(ll_kv_cache *c, int layer, cudaStream_t stream) {
  llk::DequantParams q;
  q.data = c->data;
  q.scales = c->scales;
  q.view = reinterpret_cast<uint4 *>(c->view);
  q.H = c->H;
  q.D = c->D;
  q.slots = static_cast<int>(c->slots);
  q.ctr = c->ctr + layer;
  q.n_rows = 0;
  q.G = c->S;
  q.Ss = c->Ss;
  q.W = c->W;
  q.R = c->R;
  q.T = c->T;
  q.plane0 = layer * 2 * c->H;
  q.planes = static_cast<long long>(c->L) * 2 * c->H;
  q.err = c->err;
  return launch_dequant_kernel(q, c->dtype, c->device, stream);
}

template <int FMT, int D, int PASSES>
ll_status launch_scatter_kernel(const llk::ScatterParams &p, int device, cudaStream_t stream) {
  using C = llk::ScatterTile<D, PASSES>;
  const long long rows_frame = static_cast<long long>(p.T) * p.H;
  const long long units = static_cast<long long>(p.n_layers) * p.n_frames * ((rows_frame + C::kRows - 1) / C::kRows);
  if (units < 1 || units >= (1ll << 31)) return LL_ERR_INVALID_ARG;
  if (!prepare_scatter<FMT, D, PASSES>()) return LL_ERR_CUDA;
  // kCtasPerSm CTAs per SM, each owning a contiguous range of units (at least one)
  long long grid = static_cast<long long>(num_sms(device)) * C::kCtasPerSm;
  if (grid > units) grid = units;
  llk::kv_scatter_kernel<FMT, D, PASSES><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

template <int FMT, int D>
ll_status launch_scatter_mode(const llk::ScatterParams &p, int device, cudaStream_t stream) {
  return p.mode == llk::SCATTER_APPEND ? launch_scatter_kernel<FMT, D, 1>(p, device, stream)
                                       : launch_scatter_kernel<FMT, D, 2>(p, device, stream);
}

// Units of ScatterTile<D, passes>::kRows source rows, K and V apart.
ll_status launch_scatter(ll_kv_cache *c, const llk::ScatterParams &q, int n_layers, cudaStream_t stream) {
  llk::ScatterParams p = q;
  p.n_layers = n_layers;
  const int dev = c->device;
  switch (c->dtype) {
    case LL_KV_BF16:
      return q.D == 128 ? launch_scatter_mode<llk::FMT_BF16, 128>(p, dev, stream)
                        : launch_scatter_mode<llk::FMT_BF16, 64>(p, dev, stream);
    case LL_KV_FP8_E4M3:
      return q.D == 128 ? launch_scatter_mode<llk::FMT_FP8, 128>(p, dev, stream)
                        : launch_scatter_mode<llk::FMT_FP8, 64>(p, dev, stream);
    case LL_KV_NVFP4:
      return q.D == 128 ? launch_scatter_mode<llk::FMT_NVFP4, 128>(p, dev, stream)
                        : launch_scatter_mode<llk::FMT_NVFP4, 64>(p, dev, stream);
  }
  return LL_ERR_INVALID_ARG;
}

llk::ScatterParams scatter_base(const ll_kv_cache *c, const void *k, const void *v) {
  llk::ScatterParams q;
  std::memset(&q, 0, sizeof(q));
  q.src_k = static_cast<const uint4 *>(k);
  q.src_v = static_cast<const uint4 *>(v);
  q.data = c->data;
  q.scales = c->scales;
  q.H = c->H;
  q.D = c->D;
  q.T = c->T;
  q.slots = static_cast<int>(c->slots);
  q.G = c->S;
  q.Ss = c->Ss;
  q.W = c->W;
  q.R = c->R;
  q.F = c->F;
  q.ctr = c->ctr;
  q.done = c->done;
  q.err = c->err;
  q.planes = static_cast<long long>(c->L) * 2 * c->H;
  return q;
}

ll_status attention(const void *q, const void *k_cur, const void *v_cur, ll_kv_cache *c, int layer, void *out,
                    ll_stream_t stream, bool append);

// one cache; spare_slots adds F ring slots (the layout the fused append needs)
ll_status create_cache(int layers, int heads, int head_dim, int tokens_per_frame, int frames_per_chunk,
                       int global_sink_frames, int shot_sink_frames, int window_frames, bool spare_slots,
                       ll_kv_dtype kv_dtype, ll_kv_cache **out);

}  // namespace

extern "C" {

const char *ll_status_string(ll_status s) {
  switch (s) {
    case LL_OK: return "ok";
    case LL_ERR_INVALID_ARG: return "invalid argument";
    case LL_ERR_OOM: return "out of device memory";
    case LL_ERR_CUDA: return "CUDA error";
    case LL_ERR_UNSUPPORTED: return "unsupported";
    case LL_ERR_TIMEOUT: return "in-kernel wait timed out";
  }
  return "unknown status";
}

long long ll_allocation_count(void) { return g_alloc_count.load(); }

ll_status ll_kv_cache_create(int layers, int heads, int head_dim, int tokens_per_frame, int frames_per_chunk,
                             int sink_frames, int window_frames, ll_kv_dtype kv_dtype, ll_kv_cache **out) {
  return ll_kv_cache_create_multishot(layers, heads, head_dim, tokens_per_frame, frames_per_chunk, sink_frames, 0,
                                      window_frames, kv_dtype, out);
}

ll_status ll_kv_cache_create_multishot(int layers, int heads, int head_dim, int tokens_per_frame,
                                       int frames_per_chunk, int global_sink_frames, int shot_sink_frames,
                                       int window_frames, ll_kv_dtype kv_dtype, ll_kv_cache **out) {
  return create_cache(layers, heads, head_dim, tokens_per_frame, frames_per_chunk, global_sink_frames,
                      shot_sink_frames, window_frames, false, kv_dtype, out);
}

ll_status ll_kv_cache_create_fused(int layers, int heads, int head_dim, int tokens_per_frame, int frames_per_chunk,
                                   int global_sink_frames, int shot_sink_frames, int window_frames,
                                   ll_kv_dtype kv_dtype, ll_kv_cache **out) {
  return create_cache(layers, heads, head_dim, tokens_per_frame, frames_per_chunk, global_sink_frames,
                      shot_sink_frames, window_frames, true, kv_dtype, out);
}

}  // extern "C"

namespace llk {
// the shot start of ll_kv_shot_begin: empties the shot sink of layers
// [l0, l0 + nl) and, if asked, restarts their window
__global__ void shot_begin_kernel(LayerCtr *ctr, int l0, int nl, int clear_window) {
  for (int i = threadIdx.x; i < nl; i += blockDim.x) {
    LayerCtr *c = ctr + l0 + i;
    c->shot_fill = 0;
    if (clear_window) c->ring_start = c->ring_count;
  }
}
}  // namespace llk

namespace {
// Loads every kernel a chunk step can launch (and raises the shared-memory
// limits) once per device, at the first cache creation there: with lazy module
// loading a kernel's first launch would otherwise take device memory for its
// code in the middle of a rollout, after the cache's footprint is fixed.
bool preload_kernels(int dev) {
  static std::atomic<unsigned long long> loaded{0};
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  if (bit && (loaded.load() & bit)) return true;
  bool ok = prepare_attn<64>() && prepare_attn<128>();
  ok = ok && prepare_scatter<llk::FMT_BF16, 64, 1>() && prepare_scatter<llk::FMT_BF16, 64, 2>() &&
       prepare_scatter<llk::FMT_BF16, 128, 1>() && prepare_scatter<llk::FMT_BF16, 128, 2>() &&
       prepare_scatter<llk::FMT_FP8, 64, 1>() && prepare_scatter<llk::FMT_FP8, 64, 2>() &&
       prepare_scatter<llk::FMT_FP8, 128, 1>() && prepare_scatter<llk::FMT_FP8, 128, 2>() &&
       prepare_scatter<llk::FMT_NVFP4, 64, 1>() && prepare_scatter<llk::FMT_NVFP4, 64, 2>() &&
       prepare_scatter<llk::FMT_NVFP4, 128, 1>() && prepare_scatter<llk::FMT_NVFP4, 128, 2>();
  cudaFuncAttributes a;
  ok = ok && cudaFuncGetAttributes(&a, llk::kv_dequant_kernel<llk::FMT_FP8, 8>) == cudaSuccess &&
       cudaFuncGetAttributes(&a, llk::kv_dequant_kernel<llk::FMT_FP8, 16>) == cudaSuccess &&
       cudaFuncGetAttributes(&a, llk::kv_dequant_kernel<llk::FMT_NVFP4, 8>) == cudaSuccess &&
       cudaFuncGetAttributes(&a, llk::kv_dequant_kernel<llk::FMT_NVFP4, 16>) == cudaSuccess &&
       cudaFuncGetAttributes(&a, llk::shot_begin_kernel) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return false;
  }
  loaded.fetch_or(bit);
  return true;
}

ll_status create_cache(int layers, int heads, int head_dim, int tokens_per_frame, int frames_per_chunk,
                       int global_sink_frames, int shot_sink_frames, int window_frames, bool spare_slots,
                       ll_kv_dtype kv_dtype, ll_kv_cache **out) {
  if (!out) return LL_ERR_INVALID_ARG;
  *out = nullptr;
  const int sink_frames = global_sink_frames;
  if (layers < 1 || heads < 1 || tokens_per_frame < 1 || frames_per_chunk < 1) return LL_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LL_ERR_INVALID_ARG;
  if (sink_frames < 0 || shot_sink_frames < 0 || window_frames < 0) return LL_ERR_INVALID_ARG;
  if (static_cast<long long>(sink_frames) + shot_sink_frames + window_frames < 1) return LL_ERR_INVALID_ARG;
  if (kv_dtype != LL_KV_BF16 && kv_dtype != LL_KV_FP8_E4M3 && kv_dtype != LL_KV_NVFP4) return LL_ERR_INVALID_ARG;
  const long long ring_slots = static_cast<long long>(window_frames) + (spare_slots ? frames_per_chunk : 0);
  const long long slots = (static_cast<long long>(sink_frames) + shot_sink_frames + ring_slots) * tokens_per_frame;
  const long long tq = static_cast<long long>(frames_per_chunk) * tokens_per_frame;
  if (slots >= (1ll << 31) || tq >= (1ll << 31)) return LL_ERR_INVALID_ARG;
  if (static_cast<long long>(tokens_per_frame) * heads * (head_dim / 8) >= (1ll << 30)) return LL_ERR_INVALID_ARG;
  if (slots * (head_dim / 8) >= (1ll << 30) || heads >= 32768) return LL_ERR_INVALID_ARG;
  const long long planes = static_cast<long long>(layers) * 2 * heads;
  if (planes >= (1ll << 31)) return LL_ERR_INVALID_ARG;

  size_t row_bytes = 0, scale_row_bytes = 0;
  switch (kv_dtype) {
    case LL_KV_BF16: row_bytes = head_dim * 2; break;
    case LL_KV_FP8_E4M3: row_bytes = head_dim; scale_row_bytes = 4; break;
    case LL_KV_NVFP4: row_bytes = head_dim / 2; scale_row_bytes = head_dim / 16; break;
  }
  const size_t data_plane = static_cast<size_t>(slots) * row_bytes;
  const size_t scale_plane = static_cast<size_t>(slots) * scale_row_bytes;
  const size_t data_bytes = data_plane * planes;
  const size_t scale_bytes = scale_plane * planes;
  // Regions, each followed by a guard of canary bytes (the padding to the next
  // 256-byte boundary plus kGuardBytes more): data | scales | status word |
  // counters | append-completion counts | (quantised caches) the bf16 view of
  // one layer's K and V planes, the input of the attention kernel after each
  // call's dequantisation. ll_debug_check_canaries reads the guards back.
  std::vector<std::pair<size_t, size_t>> guards;           // [begin, end) of each guard
  size_t off = 0;
  auto region = [&](size_t bytes) {
    const size_t begin = off;
    const size_t end = begin + bytes;
    off = ((end + 255) & ~size_t(255)) + kGuardBytes;
    guards.emplace_back(end, off);
    return begin;
  };
  region(data_bytes);
  const size_t scale_off = region(scale_bytes);
  const size_t err_off = region(sizeof(unsigned));
  const size_t ctr_off = region(static_cast<size_t>(layers) * sizeof(llk::LayerCtr));
  const size_t done_off = region(static_cast<size_t>(layers) * sizeof(unsigned));
  const size_t view_bytes =
      kv_dtype == LL_KV_BF16 ? 0 : static_cast<size_t>(2 * heads) * slots * head_dim * 2;
  const size_t view_off = region(view_bytes);
  const size_t total = off;

  if (test_fail_alloc()) return LL_ERR_OOM;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LL_ERR_CUDA;
  if (!preload_kernels(dev)) return LL_ERR_CUDA;
  ll_kv_cache *c = new (std::nothrow) ll_kv_cache();
  if (!c) return LL_ERR_OOM;
  c->L = layers; c->H = heads; c->D = head_dim; c->T = tokens_per_frame; c->F = frames_per_chunk;
  c->S = sink_frames; c->W = window_frames; c->dtype = kv_dtype; c->device = dev; c->slots = slots;
  c->Ss = shot_sink_frames;
  c->R = static_cast<int>(ring_slots);
  c->hc.assign(layers, llk::LayerCtr{0, 0, 0, 0, 0});
  c->host_counters = true;
  c->data_plane_bytes = data_plane;
  c->scale_plane_bytes = scale_plane;
  void *mem = nullptr;
  cudaError_t e = cudaMalloc(&mem, total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    delete c;
    return e == cudaErrorMemoryAllocation ? LL_ERR_OOM : LL_ERR_CUDA;
  }
  g_alloc_count.fetch_add(1);
  c->base = static_cast<uint8_t *>(mem);
  c->bytes = total;
  c->data = c->base;
  c->scales = scale_bytes ? c->base + scale_off : nullptr;
  c->err = reinterpret_cast<unsigned *>(c->base + err_off);
  c->ctr = reinterpret_cast<llk::LayerCtr *>(c->base + ctr_off);
  c->done = reinterpret_cast<unsigned *>(c->base + done_off);
  c->view = view_bytes ? c->base + view_off : nullptr;
  c->guards = guards;
  bool filled = cudaMemset(mem, 0, total) == cudaSuccess;
  for (const auto &g : guards)
    filled = filled && cudaMemset(c->base + g.first, kCanary, g.second - g.first) == cudaSuccess;
  if (!filled || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(mem);
    g_alloc_count.fetch_sub(1);
    delete c;
    return LL_ERR_CUDA;
  }
  std::memset(&c->tm_cache, 0, sizeof(c->tm_cache));
  std::memset(&c->tm_view, 0, sizeof(c->tm_view));
  const bool map_ok =
      kv_dtype == LL_KV_BF16
          ? make_map_3d(&c->tm_cache, c->data, head_dim, slots, planes, static_cast<uint64_t>(head_dim) * 2,
                        static_cast<uint64_t>(slots) * head_dim * 2, 64, kKeyTile, 1)
          : make_map_3d(&c->tm_view, c->view, head_dim, slots, 2 * heads, static_cast<uint64_t>(head_dim) * 2,
                        static_cast<uint64_t>(slots) * head_dim * 2, 64, kKeyTile, 1);
  if (!map_ok) {
    cudaFree(mem);
    g_alloc_count.fetch_sub(1);
    delete c;
    return LL_ERR_CUDA;
  }
  *out = c;
  return LL_OK;
}
}  // namespace

extern "C" {

ll_status ll_kv_cache_destroy(ll_kv_cache *c) {
  if (!c) return LL_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  const cudaError_t e = cudaFree(c->base);
  g_alloc_count.fetch_sub(1);
  cudaSetDevice(prev);
  delete c;
  return e == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status ll_kv_cache_info(const ll_kv_cache *c, int layer, long long *frames_seen, size_t *device_bytes) {
  if (!c || layer < 0 || layer >= c->L) return LL_ERR_INVALID_ARG;
  if (frames_seen) {
    if (c->host_counters) {
      *frames_seen = c->hc[layer].p;
    } else {
      // replays of captured appends have moved the device counter: wait for all
      // work on the device, then read it
      llk::LayerCtr d;
      if (!read_device_counters(c, layer, &d)) return LL_ERR_CUDA;
      *frames_seen = d.p;
    }
  }
  if (device_bytes) *device_bytes = c->bytes;
  return LL_OK;
}

size_t ll_kv_export_bytes(const ll_kv_cache *c) {
  if (!c) return 0;
  return 2 * (c->data_plane_bytes + c->scale_plane_bytes) * static_cast<size_t>(c->H);
}

ll_status ll_kv_cache_export(const ll_kv_cache *c, int layer, void *host_dst, size_t bytes, ll_stream_t stream) {
  if (!c || !host_dst || layer < 0 || layer >= c->L || bytes != ll_kv_export_bytes(c)) return LL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *dst = static_cast<uint8_t *>(host_dst);
  const size_t dlayer = 2 * c->data_plane_bytes * c->H;
  if (cudaMemcpyAsync(dst, c->data + dlayer * layer, dlayer, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LL_ERR_CUDA;
  if (c->scales) {
    const size_t slayer = 2 * c->scale_plane_bytes * c->H;
    if (cudaMemcpyAsync(dst + dlayer, c->scales + slayer * layer, slayer, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return LL_ERR_CUDA;
  }
  return cudaStreamSynchronize(s) == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

ll_status ll_debug_check_canaries(const ll_kv_cache *c, size_t *bad_offset) {
  if (!c) return LL_ERR_INVALID_ARG;
  if (bad_offset) *bad_offset = static_cast<size_t>(-1);
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(c->device) != cudaSuccess) return LL_ERR_CUDA;
  ll_status r = cudaDeviceSynchronize() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
  std::vector<uint8_t> buf;
  for (const auto &g : c->guards) {
    if (r != LL_OK) break;
    buf.resize(g.second - g.first);
    if (cudaMemcpy(buf.data(), c->base + g.first, buf.size(), cudaMemcpyDeviceToHost) != cudaSuccess) {
      r = LL_ERR_CUDA;
      break;
    }
    for (size_t i = 0; i < buf.size(); ++i) {
      if (buf[i] != static_cast<uint8_t>(kCanary)) {
        if (bad_offset) *bad_offset = g.first + i;
        r = LL_ERR_INVALID_ARG;
        break;
      }
    }
  }
  cudaSetDevice(prev);
  return r;
}

ll_status ll_debug_status(ll_kv_cache *c, unsigned int *word, int clear, ll_stream_t stream) {
  if (!c || !word) return LL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned w = 0;
  if (cudaMemcpyAsync(&w, c->err, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LL_ERR_CUDA;
  if (clear && cudaMemsetAsync(c->err, 0, sizeof(unsigned), s) != cudaSuccess) return LL_ERR_CUDA;
  *word = w;
  if (w & llk::ERR_WAIT_TIMEOUT) return LL_ERR_TIMEOUT;
  return w ? LL_ERR_INVALID_ARG : LL_OK;
}

ll_status ll_kv_append(ll_kv_cache *c, int layer, const void *k_cur, const void *v_cur, ll_stream_t stream) {
  if (!c || layer < -1 || layer >= c->L || !k_cur || !v_cur || !aligned16(k_cur) || !aligned16(v_cur))
    return LL_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return LL_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  const int l0 = layer < 0 ? 0 : layer;
  const int nl = layer < 0 ? c->L : 1;
  llk::ScatterParams q = scatter_base(c, k_cur, v_cur);
  q.mode = llk::SCATTER_APPEND;
  q.layer0 = l0;
  q.n_frames = c->F;
  const ll_status r = launch_scatter(c, q, nl, st);
  if (r == LL_OK)
    for (int l = l0; l < l0 + nl; ++l) mirror_append(c, l, cs);
  return r;
}

ll_status ll_kv_recache_write(ll_kv_cache *c, int layer, const void *k_new, const void *v_new, int first_frame,
                              int num_frames, ll_stream_t stream) {
  if (!c || layer < -1 || layer >= c->L || !k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))
    return LL_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return LL_ERR_INVALID_ARG;
  if (first_frame < 0 || num_frames < 1) return LL_ERR_INVALID_ARG;
  const int l0 = layer < 0 ? 0 : layer;
  const int nl = layer < 0 ? c->L : 1;
  if (static_cast<long long>(first_frame) + num_frames > static_cast<long long>(c->S) + c->Ss + c->W)
    return LL_ERR_INVALID_ARG;
  // every addressed layer must hold the frames addressed; each layer maps logical
  // frames to slots with its own counter. While the host mirror is exact this is
  // checked here; otherwise the kernel skips such a layer and flags ERR_RANGE.
  if (c->host_counters) {
    for (int l = l0; l < l0 + nl; ++l) {
      const llk::HeldFrames h = held(c, l);
      if (static_cast<long long>(first_frame) + num_frames > h.g + h.sf + h.w) return LL_ERR_INVALID_ARG;
    }
  }
  llk::ScatterParams q = scatter_base(c, k_new, v_new);
  q.mode = llk::SCATTER_RECACHE;
  q.layer0 = l0;
  q.n_frames = num_frames;
  q.first = first_frame;
  return launch_scatter(c, q, nl, reinterpret_cast<cudaStream_t>(stream));
}

ll_status ll_attn_sink_window(const void *q, const void *k_cur, const void *v_cur, ll_kv_cache *c, int layer,
                              void *out, ll_stream_t stream) {
  return attention(q, k_cur, v_cur, c, layer, out, stream, false);
}

ll_status ll_attn_sink_window_append(const void *q, const void *k_cur, const void *v_cur, ll_kv_cache *c, int layer,
                                     void *out, ll_stream_t stream) {
  return attention(q, k_cur, v_cur, c, layer, out, stream, true);
}

}  // extern "C"

namespace {
// attention of one layer's chunk; with append, the same launch also stores the
// chunk in the cache (which must have F spare ring slots) and advances the
// layer's counters, exactly as ll_kv_append after the attention would
ll_status attention(const void *q, const void *k_cur, const void *v_cur, ll_kv_cache *c, int layer, void *out,
                    ll_stream_t stream, bool append) {
  if (!c || layer < 0 || layer >= c->L || !q || !k_cur || !v_cur || !out) return LL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out)) return LL_ERR_INVALID_ARG;
  if (out == q || out == k_cur || out == v_cur) return LL_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return LL_ERR_INVALID_ARG;
  if (append && c->R < c->W + c->F) return LL_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (append && cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  const int Tq = c->F * c->T;
  llk::AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!make_act_map(&prm.tm_q, q, Tq, c->H, c->D) || !make_act_map(&prm.tm_kcur, k_cur, Tq, c->H, c->D) ||
      !make_act_map(&prm.tm_vcur, v_cur, Tq, c->H, c->D))
    return LL_ERR_CUDA;
  // quantised caches: the layer's held rows are dequantised into the bf16 view
  // first, and the kernel reads the view (planes: K heads 0..H-1, V heads H..2H-1)
  const bool quantised = c->dtype != LL_KV_BF16;
  prm.tm_cache = quantised ? c->tm_view : c->tm_cache;
  prm.out = static_cast<__nv_bfloat16 *>(out);
  prm.err = c->err;
  prm.ctr = c->ctr + layer;   // the kernel derives the visible keys from the layer's counters
  prm.G = c->S;
  prm.Ss = c->Ss;
  prm.W = c->W;
  prm.R = c->R;
  prm.T = c->T;
  prm.H = c->H;
  prm.Tq = Tq;
  prm.plane_k = quantised ? 0 : (layer * 2 + 0) * c->H;
  prm.plane_v = quantised ? c->H : (layer * 2 + 1) * c->H;
  prm.num_q_tiles = (Tq + 127) / 128;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->D)));
  prm.map_rows = static_cast<int>(c->slots);
  prm.cache_planes = c->L * 2 * c->H;
  prm.map_planes = quantised ? 2 * c->H : prm.cache_planes;
  if (append) {
    prm.append = 1;
    prm.fmt = c->dtype == LL_KV_BF16 ? llk::FMT_BF16 : (c->dtype == LL_KV_FP8_E4M3 ? llk::FMT_FP8 : llk::FMT_NVFP4);
    prm.F = c->F;
    prm.plane_k_cache = layer * 2 * c->H;
    prm.slots = static_cast<int>(c->slots);
    prm.kcur = static_cast<const uint4 *>(k_cur);
    prm.vcur = static_cast<const uint4 *>(v_cur);
    prm.cache_data = c->data;
    prm.cache_scales = c->scales;
    prm.ctr_rw = c->ctr + layer;
    prm.done = c->done + layer;
  }
  const int grid = prm.num_q_tiles * c->H;
  if (quantised) {
    const ll_status ds = launch_dequant(c, layer, st);
    if (ds != LL_OK) return ds;
  }
  const ll_status r = c->D == 128 ? launch_attn<128>(prm, grid, st) : launch_attn<64>(prm, grid, st);
  if (r == LL_OK && append) mirror_append(c, layer, cs);
  return r;
}
}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Shot start (several shots per video): shot_begin_kernel (above, before the
// cache creation that preloads it) empties the shot sink of the addressed
// layers and, if asked, restarts their window. A kernel, so that it is ordered
// with the appends on the stream and can be recorded in a graph.

extern "C" ll_status ll_kv_shot_begin(ll_kv_cache *c, int layer, int clear_window, ll_stream_t stream) {
  if (!c || layer < -1 || layer >= c->L) return LL_ERR_INVALID_ARG;
  if (!on_cache_device(c)) return LL_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return LL_ERR_CUDA;
  }
  const int l0 = layer < 0 ? 0 : layer;
  const int nl = layer < 0 ? c->L : 1;
  llk::shot_begin_kernel<<<1, 256, 0, st>>>(c->ctr, l0, nl, clear_window ? 1 : 0);
  if (cudaGetLastError() != cudaSuccess) return LL_ERR_CUDA;
  for (int l = l0; l < l0 + nl; ++l) {
    c->hc[l].shot_fill = 0;
    if (clear_window) c->hc[l].ring_start = c->hc[l].ring_count;
  }
  if (cs != cudaStreamCaptureStatusNone) c->host_counters = false;
  return LL_OK;
}

extern "C" ll_status ll_kv_cache_held(const ll_kv_cache *c, int layer, int *global_frames, int *shot_frames,
                                      int *window_frames) {
  if (!c || layer < 0 || layer >= c->L) return LL_ERR_INVALID_ARG;
  llk::HeldFrames h;
  if (c->host_counters) {
    h = held(c, layer);
  } else {
    llk::LayerCtr d;
    if (!read_device_counters(c, layer, &d)) return LL_ERR_CUDA;
    h = llk::held_frames(d.p, d.shot_fill, d.ring_count, d.ring_start, c->S, c->W);
  }
  if (global_frames) *global_frames = h.g;
  if (shot_frames) *shot_frames = h.sf;
  if (window_frames) *window_frames = h.w;
  return LL_OK;
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait: one thread waits on a barrier nothing completes.
namespace llk {
__global__ void wait_selftest_kernel(unsigned *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  mbar_wait(&bar, 0, &abort_flag, err, KID_SELFTEST);
}
}  // namespace llk

namespace llk {
// The reporting path of the index checks: one check that fails; nothing is
// accessed either way (the check decides only whether a store would happen).
__global__ void bounds_selftest_kernel(unsigned *err) {
  volatile int n = 1, idx = 1;
  if (bounds_ok(idx < n, err, KID_SELFTEST)) atomicOr(err, 0u);
}
}  // namespace llk

extern "C" ll_status ll_debug_bounds_selftest(ll_kv_cache *c, ll_stream_t stream) {
  if (!c || !on_cache_device(c)) return LL_ERR_INVALID_ARG;
  llk::bounds_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c->err);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

extern "C" int ll_bounds_checked(void) {
#ifdef LL_BOUNDS_CHECK
  return 1;
#else
  return 0;
#endif
}

extern "C" ll_status ll_debug_wait_selftest(ll_kv_cache *c, ll_stream_t stream) {
  if (!c || !on_cache_device(c)) return LL_ERR_INVALID_ARG;
  llk::wait_selftest_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c->err);
  return cudaGetLastError() == cudaSuccess ? LL_OK : LL_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// No-allocation entry point. Its scratch (the dequantised bf16 view of one
// layer) is this file-scope device array, so the call needs no cudaMalloc. In
// host code the name is only a stand-in: its device address is looked up once
// per device with cudaGetSymbolAddress (with that device current) and passed
// to the kernels.
static __device__ __align__(256) uint8_t g_noalloc_view[LL_NOALLOC_SCRATCH_BYTES];
// the status word of this path's kernels (the cache path keeps its own in the
// cache allocation): a bounded wait that gives up is recorded here
static __device__ __align__(256) unsigned g_noalloc_status;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kMaxDevices] = {};
unsigned *g_noalloc_status_addr[kMaxDevices] = {};

// device addresses of g_noalloc_view and g_noalloc_status on device `dev`,
// which must be current (false on failure)
bool noalloc_scratch(int dev, void **view, unsigned **status) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void *v = nullptr, *st = nullptr;
    if (cudaGetSymbolAddress(&v, g_noalloc_view) != cudaSuccess ||
        cudaGetSymbolAddress(&st, g_noalloc_status) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    g_noalloc_status_addr[dev] = static_cast<unsigned *>(st);
    g_noalloc_addr[dev] = v;
  }
  *view = g_noalloc_addr[dev];
  *status = g_noalloc_status_addr[dev];
  return true;
}
}  // namespace

ll_status ll_attn_sink_window_noalloc(const void *q, const void *k_cur, const void *v_cur, const void *layer_codes,
                                      const void *layer_scales, ll_kv_dtype kv_dtype, int heads, int head_dim,
                                      int tokens_per_frame, int frames_per_chunk, int sink_frames, int window_frames,
                                      long long frames_seen, void *out, ll_stream_t stream) {
  if (!q || !k_cur || !v_cur || !layer_codes || !layer_scales || !out) return LL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out) || !aligned16(layer_codes) ||
      !aligned16(layer_scales))
    return LL_ERR_INVALID_ARG;
  if (out == q || out == k_cur || out == v_cur) return LL_ERR_INVALID_ARG;
  if (kv_dtype != LL_KV_FP8_E4M3 && kv_dtype != LL_KV_NVFP4) return LL_ERR_INVALID_ARG;
  if (heads < 1 || tokens_per_frame < 1 || frames_per_chunk < 1 || (head_dim != 64 && head_dim != 128))
    return LL_ERR_INVALID_ARG;
  if (sink_frames < 0 || window_frames < 0 || sink_frames + window_frames < 1 || frames_seen < 0)
    return LL_ERR_INVALID_ARG;
  const long long slots = static_cast<long long>(sink_frames + window_frames) * tokens_per_frame;
  const long long tq = static_cast<long long>(frames_per_chunk) * tokens_per_frame;
  if (slots >= (1ll << 31) || tq >= (1ll << 31)) return LL_ERR_INVALID_ARG;
  if (slots * (head_dim / 8) >= (1ll << 30) || heads >= 32768) return LL_ERR_INVALID_ARG;
  // the view of the layer must fit the static scratch
  const unsigned long long view_bytes = 2ull * heads * static_cast<unsigned long long>(slots) * head_dim * 2;
  if (view_bytes > LL_NOALLOC_SCRATCH_BYTES) return LL_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LL_ERR_CUDA;
  void *view_ptr = nullptr;
  unsigned *status = nullptr;
  if (!noalloc_scratch(dev, &view_ptr, &status)) return LL_ERR_CUDA;
  uint8_t *view = static_cast<uint8_t *>(view_ptr);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // held context, as for a cache whose layer counter is frames_seen
  const long long s_held = frames_seen < sink_frames ? frames_seen : sink_frames;
  long long w_held = frames_seen - sink_frames;
  if (w_held < 0) w_held = 0;
  if (w_held > window_frames) w_held = window_frames;
  const int n_cache = static_cast<int>((s_held + w_held) * tokens_per_frame);
  const int Tq = static_cast<int>(tq);

  // 1) dequantise the held rows into the view; the rows the ragged last tile
  //    also reads, [n_cache, min(slots, kKeyTile * ceil(n_cache / kKeyTile))), are cleared
  //    so that they are finite (the array keeps the previous call's contents)
  if (n_cache > 0) {
    llk::DequantParams dq;
    dq.data = static_cast<const uint8_t *>(layer_codes);
    dq.scales = static_cast<const uint8_t *>(layer_scales);
    dq.view = reinterpret_cast<uint4 *>(view);
    dq.H = heads;
    dq.D = head_dim;
    dq.slots = static_cast<int>(slots);
    dq.ctr = nullptr;
    dq.n_rows = n_cache;
    dq.G = sink_frames;
    dq.Ss = 0;
    dq.W = window_frames;
    dq.R = window_frames;
    dq.T = tokens_per_frame;
    dq.plane0 = 0;
    dq.planes = 2ll * heads;
    dq.err = status;
    const ll_status ds = launch_dequant_kernel(dq, kv_dtype, dev, st);
    if (ds != LL_OK) return ds;
    long long tail_end = (static_cast<long long>(n_cache) + kKeyTile - 1) / kKeyTile * kKeyTile;
    if (tail_end > slots) tail_end = slots;
    if (tail_end > n_cache) {
      const size_t row_b = static_cast<size_t>(head_dim) * 2;
      if (cudaMemset2DAsync(view + n_cache * row_b, static_cast<size_t>(slots) * row_b, 0,
                            static_cast<size_t>(tail_end - n_cache) * row_b, static_cast<size_t>(2 * heads),
                            st) != cudaSuccess)
        return LL_ERR_CUDA;
    }
  }

  // 2) the bf16 attention kernel over the view (planes: K heads 0..H-1, V heads H..2H-1)
  llk::AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!make_act_map(&prm.tm_q, q, Tq, heads, head_dim) || !make_act_map(&prm.tm_kcur, k_cur, Tq, heads, head_dim) ||
      !make_act_map(&prm.tm_vcur, v_cur, Tq, heads, head_dim) ||
      !make_map_3d(&prm.tm_cache, view, head_dim, slots, 2 * heads, static_cast<uint64_t>(head_dim) * 2,
                   static_cast<uint64_t>(slots) * head_dim * 2, 64, kKeyTile, 1))
    return LL_ERR_CUDA;
  prm.out = static_cast<__nv_bfloat16 *>(out);
  prm.err = status;
  prm.H = heads;
  prm.Tq = Tq;
  prm.n_cache = n_cache;
  prm.plane_k = 0;
  prm.plane_v = heads;
  prm.num_q_tiles = (Tq + 127) / 128;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  prm.map_rows = static_cast<int>(slots);
  prm.map_planes = 2 * heads;
  prm.cache_planes = 2 * heads;
  const int grid = prm.num_q_tiles * heads;
  return head_dim == 128 ? launch_attn<128>(prm, grid, st) : launch_attn<64>(prm, grid, st);
}

ll_status ll_noalloc_debug_status(unsigned int *word, int clear, ll_stream_t stream) {
  if (!word) return LL_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LL_ERR_CUDA;
  void *view = nullptr;
  unsigned *status = nullptr;
  if (!noalloc_scratch(dev, &view, &status)) return LL_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned w = 0;
  if (cudaMemcpyAsync(&w, status, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LL_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LL_ERR_CUDA;
  if (clear && cudaMemsetAsync(status, 0, sizeof(unsigned), s) != cudaSuccess) return LL_ERR_CUDA;
  *word = w;
  if (w & llk::ERR_WAIT_TIMEOUT) return LL_ERR_TIMEOUT;
  return w ? LL_ERR_INVALID_ARG : LL_OK;
}

}  // extern "C"
