/*
 * ll_kvattn.h - C ABI of the LongLive sink + window chunk-attention library
 * for NVIDIA B200 (sm_100a).
 *
 * The library implements the per-layer hot path of frame-level causal
 * autoregressive video generation with a bounded KV cache:
 *
 *   - a KV cache per layer holding the K/V of a permanently kept frame sink and
 *     of a short sliding window of recent frames (LongLive explainer, dpshk.com,
 *     sec. 五 "Short Window Attention" and sec. 六 "Frame Sink": KV cache = sink
 *     frames' KV + recent window's KV);
 *   - the append/evict step after each generated chunk (same sections; the
 *     techwalker.com LONGLIVE article, sec. 六, clears old cache entries
 *     progressively);
 *   - the bulk rewrite of the held K/V after a prompt switch, "KV-recache"
 *     (dpshk.com sec. 三.3 and 三.5; techwalker.com sec. 六);
 *   - attention of the current chunk's queries over sink + window + the chunk's
 *     own K/V, full inside the chunk and causal across chunks (LongLive-2.0
 *     explainer, wmrh.cn, sec. 6).
 *
 * Conventions shared by every call
 *   Notation: L layers, H heads, D head_dim, T tokens per latent frame,
 *   F frames per chunk, S sink frames, W window frames, Tq = F*T.
 *   Activation tensors (q, k_cur, v_cur, out, k_new, v_new) are caller-owned
 *   DEVICE pointers to contiguous bf16 (IEEE bfloat16 bit patterns), token-major
 *   [tokens][H][D], batch 1, 16-byte aligned. The library never frees them.
 *   The cache owns all of its device memory from create to destroy; no call
 *   between those allocates device memory (constant footprint).
 *   Every call that takes a stream only enqueues work on it; none synchronises
 *   the host. Calls touching the same layer must be ordered by the caller, on
 *   one stream or with events. The host-side frame counter of a layer advances
 *   when ll_kv_append is called (enqueue order = logical order).
 *   A cache lives on the device that was current at create: calls that launch
 *   work on it must be made with that device current (else
 *   LL_ERR_INVALID_ARG), and their tensors must live on that device. Calls on
 *   one cache from several host threads must be serialised by the caller.
 *   Errors are returned, never raised or aborted; on an error nothing was
 *   enqueued unless the status is LL_ERR_CUDA (a launch failed), and the cache
 *   handle stays valid.
 *   `stream` is a cudaStream_t (NULL = legacy default stream); it is declared
 *   through the CUDA runtime's own opaque struct so that this header needs no
 *   CUDA include.
 *
 * Window reading: W counts cached frames of EARLIER chunks; the own chunk is
 * always added on top. A frame below S is a sink frame only; the window holds
 * the last W non-sink frames before the current chunk.
 */
#ifndef LL_KVATTN_H
#define LL_KVATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define LL_API __attribute__((visibility("default")))
#else
#define LL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ll_stream_t;     /* == cudaStream_t */
typedef struct ll_kv_cache ll_kv_cache;      /* opaque; owns the cache memory */

typedef enum {
  LL_KV_BF16 = 0,       /* K/V stored as bf16 */
  LL_KV_FP8_E4M3 = 1,   /* E4M3 codes + one fp32 scale per (token, head) row: the
                           smallest power of two 2^k >= amax/448 with k >= -124
                           (1 for an all-zero row); codes = E4M3(x / scale),
                           round to nearest even, saturating */
  LL_KV_NVFP4 = 2       /* E2M1 codes, 16-value blocks along D, E4M3 block scale */
} ll_kv_dtype;

typedef enum {
  LL_OK = 0,
  LL_ERR_INVALID_ARG = 1,   /* a range, null, alignment or state check failed */
  LL_ERR_OOM = 2,           /* device allocation failed at create */
  LL_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed */
  LL_ERR_UNSUPPORTED = 4,   /* valid request the library does not serve (e.g. fused call on a plain cache) */
  LL_ERR_TIMEOUT = 5        /* a bounded in-kernel wait gave up (see ll_debug_status) */
} ll_status;

/* ll_kv_cache_create - allocate the cache of `layers` layers.
 *   Layout (device, one allocation): for each layer l and each of K (0), V (1):
 *   [H][(S+W)*T][D] elements; slots 0..S-1 (frame granularity) hold the sink
 *   frames, slots S..S+W-1 form a frame-granular ring holding the window.
 *   Quantised formats add a scale array per layer and K/V:
 *   FP8 [H][(S+W)*T] fp32; NVFP4 [H][(S+W)*T][D/16] E4M3 bytes; and a bf16
 *   view of ONE layer's K and V planes (2*H*(S+W)*T*D*2 bytes) that each
 *   ll_attn_sink_window call refills with the dequantised held frames.
 *   The memory is zero-filled at create; frame counters start at 0. The
 *   frame counter p of each layer lives in device memory: the kernels read it
 *   and ll_kv_append advances it, so calls recorded in a CUDA graph (stream
 *   capture) stay right when the graph is replayed chunk after chunk.
 *   Supported: layers, heads, tokens_per_frame, frames_per_chunk >= 1;
 *   head_dim in {64, 128}; sink_frames >= 0, window_frames >= 0,
 *   sink_frames + window_frames >= 1; (S+W)*T and F*T < 2^31; T*H*D/8 and
 *   (S+W)*T*D/8 < 2^30; heads < 32768.
 *   The first cache created on a device also loads there every kernel a
 *   chunk step can launch, so that no later call takes device memory for
 *   kernel code (the footprint is fixed from here on).
 *   Returns LL_ERR_INVALID_ARG on a bad parameter or null `out`,
 *   LL_ERR_OOM if the allocation fails, LL_ERR_CUDA if no device is usable.
 *   On success *out owns the memory until ll_kv_cache_destroy.           */
LL_API ll_status ll_kv_cache_create(int layers, int heads, int head_dim, int tokens_per_frame,
                             int frames_per_chunk, int sink_frames, int window_frames,
                             ll_kv_dtype kv_dtype, ll_kv_cache **out);

/* ll_kv_cache_create_multishot - a cache for videos of several shots.
 *   LongLive-2.0 explainer (wmrh.cn), sec. 16: a global-level sink that every
 *   shot attends to and a shot-level sink for the current shot. Per layer and
 *   K/V plane the layout is [H][(G+Ss+W)*T][D]: slots 0..G-1 global sink (the
 *   first G frames of the video), slots G..G+Ss-1 the current shot's sink (its
 *   first Ss frames that are not global-sink frames), then a W-slot ring for
 *   all other frames; the window is the ring's last W frames (since the last
 *   window restart, see ll_kv_shot_begin). Each frame is stored in exactly one
 *   region, so no key is attended twice. shot_sink_frames = 0 gives exactly
 *   the single-shot cache of ll_kv_cache_create (which calls this with 0).
 *   Other arguments, limits and errors as for ll_kv_cache_create, with
 *   G + Ss + W >= 1 and (G+Ss+W)*T < 2^31.                                   */
LL_API ll_status ll_kv_cache_create_multishot(int layers, int heads, int head_dim, int tokens_per_frame,
                                              int frames_per_chunk, int global_sink_frames, int shot_sink_frames,
                                              int window_frames, ll_kv_dtype kv_dtype, ll_kv_cache **out);

/* ll_kv_cache_create_fused - a cache that ll_attn_sink_window_append can use:
 *   as ll_kv_cache_create_multishot, but the ring has F spare slots (W + F
 *   in all), so per layer and K/V plane the layout is [H][(G+Ss+W+F)*T][D].
 *   The window is still the last W ring frames; the spare slots hold frames
 *   that have just left it. That is what lets one launch attend over the
 *   window and store the chunk: the chunk's frames land in slots the launch
 *   does not read. Costs F frames of memory per layer and K/V (25 % at chunk
 *   3, sink 3, window 9). Every other call works on it as on any cache.
 *   The pages describe no such layout: it exists only so that attention and
 *   append can share one launch.                                             */
LL_API ll_status ll_kv_cache_create_fused(int layers, int heads, int head_dim, int tokens_per_frame,
                                          int frames_per_chunk, int global_sink_frames, int shot_sink_frames,
                                          int window_frames, ll_kv_dtype kv_dtype, ll_kv_cache **out);

/* ll_kv_shot_begin - a new shot starts with the next appended chunk.
 *   layer: 0..L-1, or -1 for all layers. Empties the shot sink (its frames are
 *   no longer attended; the next Ss non-global frames refill it). With
 *   clear_window != 0 the window restarts too: it holds only frames appended
 *   after this call. Enqueued on `stream` (a one-block kernel), so it is ordered
 *   with the appends and can be recorded in a graph. A no-op on the shot sink
 *   of a cache made with shot_sink_frames = 0. Pages: wmrh.cn sec. 16.          */
LL_API ll_status ll_kv_shot_begin(ll_kv_cache *cache, int layer, int clear_window, ll_stream_t stream);

/* ll_kv_append - store the chunk just generated in layer `layer` and evict.
 *   layer: 0..L-1, or -1 for every layer in one launch.
 *   k_cur, v_cur: [F*T][H][D] bf16 device pointers (the chunk's K and V), or
 *   [L][F*T][H][D] with layer -1.
 *   Frame f = p..p+F-1 (p = frames appended to this layer so far) goes to slot
 *   f if f < S; otherwise, if f >= p+F-W, to ring slot S + ((f-S) mod W),
 *   overwriting (evicting) the oldest window frame; other frames (only when
 *   W < F) are not stored. For a multi-shot cache, a non-global frame goes to
 *   the current shot's sink while it has room, else to the next ring slot.
 *   Quantised caches quantise here. Then p += F, on the device, at the end of
 *   the launch (the counters are read from device memory).
 *   An append enqueued inside a stream capture ends the host's knowledge of
 *   p (see ll_kv_cache_info and ll_kv_recache_write).
 *   Pages: dpshk.com sec. 五/六; techwalker.com sec. 六.                    */
LL_API ll_status ll_kv_append(ll_kv_cache *cache, int layer, const void *k_cur, const void *v_cur,
                       ll_stream_t stream);

/* ll_kv_recache_write - KV-recache: overwrite held frames with new K/V.
 *   layer: 0..L-1, or -1 for all layers at once.
 *   k_new, v_new: [L'][num_frames*T][H][D] bf16 device pointers, L' = 1 for a
 *   single layer or L for all layers; frame i of the source replaces logical
 *   frame first_frame+i of the held context, whose logical order is: sink
 *   frames 0..s-1, then (multi-shot caches) the current shot's sink frames in
 *   fill order, then window frames oldest to newest (s = min(p,S),
 *   w = min(W, max(0, p-S)) for a single-shot cache, p the layer's own
 *   counter; ll_kv_cache_held gives the counts). Requires
 *   0 <= first_frame, num_frames >= 1, first_frame + num_frames <= S + Ss + W
 *   (else LL_ERR_INVALID_ARG) and <= s + w of every addressed layer: checked
 *   by the host (LL_ERR_INVALID_ARG) while it knows p; after a captured
 *   append, by the kernel, which then writes nothing to such a layer and sets
 *   ERR_RANGE in the status word (ll_debug_status).
 *   Frame counters and the ring position are unchanged.
 *   Sink + window is the default context (dpshk.com sec. 三.3); first_frame = S,
 *   num_frames = W gives the window-only variant with the sink unchanged
 *   (techwalker.com sec. 六).                                                */
LL_API ll_status ll_kv_recache_write(ll_kv_cache *cache, int layer, const void *k_new, const void *v_new,
                              int first_frame, int num_frames, ll_stream_t stream);

/* ll_attn_sink_window - attention of the current chunk of layer `layer`.
 *   q, k_cur, v_cur: [F*T][H][D] bf16 device pointers (the chunk's Q, K, V);
 *   out: [F*T][H][D] bf16 device pointer, written. out may not alias inputs.
 *   For each head: out = softmax(q K^T / sqrt(D)) V over the keys of
 *   cache slots [0, s*T) (sink), [S*T, (S+w)*T) (window; held frames in any
 *   ring order, softmax is order-free) - for a multi-shot cache the global
 *   sink, the current shot's sink and the window - and the chunk's own k_cur/v_cur
 *   (all Tq of them, no mask inside the chunk). s, w as for recache, taken
 *   from the layer's frame counter at call time: call it BEFORE ll_kv_append
 *   of the same chunk. bf16 operands, fp32 accumulation and softmax, the
 *   probabilities rounded to bf16 for the PV product, bf16 output.
 *   Quantised caches: the layer's held frames are first dequantised into the
 *   cache's bf16 view (FP8: E4M3 x power-of-two row scale; NVFP4: E2M1 x
 *   E4M3 block scale; both exact in bf16), then attended to like a bf16
 *   cache, so the attention sees exactly the dequantised values. The
 *   view is shared by all layers, so attention calls on one quantised cache
 *   must be ordered (one stream, or events).
 *   Pages: dpshk.com sec. 五/六; techwalker.com sec. 四/六; wmrh.cn sec. 6.  */
LL_API ll_status ll_attn_sink_window(const void *q, const void *k_cur, const void *v_cur,
                              ll_kv_cache *cache, int layer, void *out, ll_stream_t stream);

/* ll_attn_sink_window_append - ll_attn_sink_window followed by ll_kv_append of
 *   the same chunk, in one launch: the results (out, the cache bytes, the
 *   counters) are those of the two calls in that order. Two otherwise idle
 *   warps of each CTA store (and for FP8/NVFP4 quantise) that CTA's rows of
 *   k_cur/v_cur. Needs a cache made by ll_kv_cache_create_fused; any other
 *   cache returns LL_ERR_UNSUPPORTED. Arguments and errors as for
 *   ll_attn_sink_window. Pages: as for the two calls it fuses.               */
LL_API ll_status ll_attn_sink_window_append(const void *q, const void *k_cur, const void *v_cur,
                                            ll_kv_cache *cache, int layer, void *out, ll_stream_t stream);

/* ll_kv_cache_destroy - free all memory of the cache (NULL is a no-op).
 *   Synchronises the device first so that no enqueued work still uses it.  */
LL_API ll_status ll_kv_cache_destroy(ll_kv_cache *cache);

/* ---- sequence-parallel inference: the local steps around the exchange ---
 * LongLive-2.0 explainer (wmrh.cn), sec. 18.3: inference can run sequence
 * parallel across GPUs; sec. 15.2: a low-precision KV cache then also reduces
 * the traffic between them. Head-sharded form used here: P ranks each hold
 * N_s = N/P tokens of the chunk ([N_s][H][D] q, k_cur, v_cur) and a cache of
 * H/P heads (rank r: heads r*H/P .. (r+1)*H/P-1). The caller's all-to-all
 * (equal splits, e.g. NCCL) exchanges what ll_sp_pack_heads (or
 * ll_sp_pack_heads_fp8) prepared; what rank r receives, [P][N_s][H/P][D] from
 * ranks 0..P-1, is the whole chunk [N][H/P][D] for its heads: attention and
 * append take it as is. The outputs [N][H/P][D] go back through a second
 * all-to-all and ll_sp_unpack_heads. Heads never interact inside attention, so
 * each rank's results are those of an unsharded cache for the same heads.
 * Shared rules: head_dim 64 or 128; heads divisible by ranks (else
 * LL_ERR_INVALID_ARG); device pointers, 16-byte aligned, caller-owned; work is
 * only enqueued on `stream`; nothing is allocated.                          */

/* [tokens][heads][D] bf16 -> [ranks][tokens][heads/ranks][D] bf16: the block
 * for rank r holds heads r*heads/ranks.. of every token, contiguous. x and
 * packed must not overlap.                                                   */
LL_API ll_status ll_sp_pack_heads(const void *x, int tokens, int heads, int head_dim, int ranks, void *packed,
                                  ll_stream_t stream);

/* The inverse: [ranks][tokens][heads/ranks][D] -> [tokens][heads][D]. Used on
 * the outputs after the return all-to-all (block r = heads of rank r).       */
LL_API ll_status ll_sp_unpack_heads(const void *packed, int tokens, int heads, int head_dim, int ranks, void *x,
                                    ll_stream_t stream);

/* As ll_sp_pack_heads, but each (token, head) row is sent in the cache's FP8
 * row format: codes [ranks][tokens][heads/ranks][D] E4M3 bytes and scales
 * [ranks][tokens][heads/ranks] fp32, the scale the smallest power of two 2^k
 * >= max|row|/448 (k >= -124; 1 for a zero row), codes round to nearest even,
 * saturating - D + 4 bytes per row on the links instead of 2D. For K and V
 * (sec. 15.2's quantised-KV communication); the receiver restores bf16 rows
 * with ll_sp_dequant_fp8 before attention and append, which therefore see
 * the FP8-rounded chunk.                                                     */
LL_API ll_status ll_sp_pack_heads_fp8(const void *x, int tokens, int heads, int head_dim, int ranks, void *codes,
                                      void *scales, ll_stream_t stream);

/* FP8 rows [rows][D] codes + [rows] fp32 power-of-two scales -> [rows][D]
 * bf16, code x scale (exact in bf16).                                        */
LL_API ll_status ll_sp_dequant_fp8(const void *codes, const void *scales, long long rows, int head_dim, void *x,
                                   ll_stream_t stream);

/* ---- helpers --------------------------------------------------------- */

/* Static string for a status code. Never NULL.                              */
LL_API const char *ll_status_string(ll_status status);

/* Frames appended so far to `layer` (p) and the cache's total device bytes
 * (all layers, data + scales). Either output pointer may be NULL. Once an
 * append has been enqueued inside a stream capture, p is read from the device
 * after a device-wide synchronisation (do not call it while capturing).     */
LL_API ll_status ll_kv_cache_info(const ll_kv_cache *cache, int layer, long long *frames_seen,
                           size_t *device_bytes);

/* Frames of `layer` held now: global sink, current shot sink, window. Read
 * from the host's mirror, or, once an append or shot start has been enqueued
 * inside a stream capture, from the device after a device-wide
 * synchronisation (do not call it while capturing). Any output may be NULL.   */
LL_API ll_status ll_kv_cache_held(const ll_kv_cache *cache, int layer, int *global_frames, int *shot_frames,
                                  int *window_frames);

/* Number of device allocations the library currently holds (all caches).
 * Constant between create and destroy: the footprint check of a rollout.   */
LL_API long long ll_allocation_count(void);

/* Raw bytes of one layer, in the order: K data [H][(S+W)*T][...], V data,
 * then for quantised formats K scales, V scales (layouts as at create).
 * host_dst must hold `bytes` == ll_kv_export_bytes(cache); the call copies on
 * `stream` and synchronises that stream before returning.                  */
LL_API size_t ll_kv_export_bytes(const ll_kv_cache *cache);
LL_API ll_status ll_kv_cache_export(const ll_kv_cache *cache, int layer, void *host_dst, size_t bytes,
                             ll_stream_t stream);

/* ll_attn_sink_window_noalloc - the attention of ll_attn_sink_window over a
 *   quantised single-shot cache layer (FP8 or NVFP4) held in caller memory,
 *   performing no device allocation at all. The pages have no counterpart: this entry point
 *   exists for callers that cannot call cudaMalloc, for example code whose
 *   device memory is owned entirely by a host framework's pool (a serving
 *   engine that reserves all memory up front and forbids libraries from
 *   allocating), or code on a latency-critical path where cudaMalloc's implicit
 *   device synchronisation is not acceptable.
 *   Inputs (device pointers, caller-owned): q, k_cur, v_cur [F*T][H][D] bf16;
 *   layer_codes [2][H][(S+W)*T][row bytes] (K planes, then V planes; row bytes
 *   D for FP8, D/2 for NVFP4) and layer_scales [2][H][(S+W)*T][...] (fp32 per
 *   row for FP8, D/16 E4M3 bytes per row for NVFP4) - the layout that
 *   ll_kv_cache_export writes for one layer (data part, then scale part) of a
 *   cache made by ll_kv_cache_create (S + W slots per plane, the window ring
 *   starting at slot S) on which ll_kv_shot_begin was never called;
 *   frames_seen = that layer's own frame counter p (frames appended to it so
 *   far). Layers of multi-shot or fused caches, or of a cache after a shot
 *   start, have another slot layout and are not accepted (their results would
 *   be wrong). Output: out [F*T][H][D] bf16. Results equal those of
 *   ll_attn_sink_window on a cache holding the same bytes.
 *   Scratch: the dequantised bf16 view of the layer, 2*H*(S+W)*T*D*2 bytes,
 *   lives in a file-scope device array of LL_NOALLOC_SCRATCH_BYTES that every
 *   GPU loading the library holds until exit. Larger geometries are rejected
 *   with LL_ERR_INVALID_ARG before anything is enqueued. All calls share that
 *   array and it keeps the last call's contents, so calls that overlap on the
 *   GPU (different streams, or different host threads, on one device) race:
 *   order them. The first call on a device looks up the array's device
 *   address (once per device, with that device current); make that first call
 *   before any stream capture. A bounded in-kernel wait that gives up (the
 *   output is then incomplete) is recorded in this path's own device status
 *   word, read with ll_noalloc_debug_status.                                */
#define LL_NOALLOC_SCRATCH_BYTES (16u << 20)
LL_API ll_status ll_attn_sink_window_noalloc(const void *q, const void *k_cur, const void *v_cur,
                                             const void *layer_codes, const void *layer_scales,
                                             ll_kv_dtype kv_dtype, int heads, int head_dim,
                                             int tokens_per_frame, int frames_per_chunk, int sink_frames,
                                             int window_frames, long long frames_seen, void *out,
                                             ll_stream_t stream);

/* Status word of ll_attn_sink_window_noalloc's kernels on the current device
 * (one per device, shared by every call of that entry point): as for
 * ll_debug_status, reading synchronises `stream`, `clear` resets it to 0, and
 * the return value is LL_ERR_TIMEOUT if a bounded wait gave up, LL_OK for 0.
 * Allocates nothing.                                                        */
LL_API ll_status ll_noalloc_debug_status(unsigned int *word, int clear, ll_stream_t stream);

/* Device-side status word of the cache's kernels: 0 = fine; otherwise OR-ed
 * flags, reasons in the low byte (1 = a bounded in-kernel wait gave up,
 * 2 = a recache addressed frames a layer does not hold, 4 = an index check of
 * the bounds-checking build failed) and the reporting
 * kernels in the next (1 = attention, 2 = append/recache, 4 = self-test).
 * Reading synchronises `stream`; `clear` resets it to 0. The call returns
 * LL_ERR_TIMEOUT if reason 1 is set, LL_ERR_INVALID_ARG for any other
 * non-zero word, LL_OK for 0; *word is filled in all three cases.          */
LL_API ll_status ll_debug_status(ll_kv_cache *cache, unsigned int *word, int clear, ll_stream_t stream);

/* Stray-write check: every region of a cache's allocation (data, scales,
 * status word, counters, completion counts, view) is followed by a guard of
 * canary bytes, filled at create and touched by nothing afterwards. This
 * synchronises the cache's device, reads every guard back and returns LL_OK if
 * all are intact; otherwise LL_ERR_INVALID_ARG, with *bad_offset (may be NULL)
 * the allocation offset of the first changed byte. Not callable while
 * capturing a stream.                                                        */
LL_API ll_status ll_debug_check_canaries(const ll_kv_cache *cache, size_t *bad_offset);

/* Self-test of the in-kernel failure path: launches one thread that waits, with
 * the kernels' bounded mbarrier wait, on a barrier that nothing ever completes.
 * After the wait limit (about a second) the kernel records the timeout in the
 * cache's status word and returns; read it with ll_debug_status (expect
 * LL_ERR_TIMEOUT). The context stays usable. Faults nothing, hangs nothing.   */
LL_API ll_status ll_debug_wait_selftest(ll_kv_cache *cache, ll_stream_t stream);

/* Bounds-checking build. The library built with LL_BOUNDS_CHECK defined
 * (libll_kvattn_debug.so) checks, before each access, the slot rows, planes
 * and source vectors that the append/recache, dequantise and attention kernels
 * compute, and every cache tile a TMA load addresses; an index outside its
 * buffer sets reason 4 (with the kernel id) in the cache's status word and the
 * access is skipped (a cache tile is replaced by row 0). Nothing traps or
 * asserts. ll_bounds_checked() returns 1 in that build, 0 in the regular one.
 * ll_debug_bounds_selftest runs one failing check on the cache's status word
 * (kernel id 4, reason 4), in either build, to exercise the reporting path;
 * nothing is accessed.                                                        */
LL_API int ll_bounds_checked(void);
LL_API ll_status ll_debug_bounds_selftest(ll_kv_cache *cache, ll_stream_t stream);

/* Test hook: when the environment variable LL_KVATTN_TEST_FAIL_ALLOC is set to
 * a non-empty value other than "0", ll_kv_cache_create fails as if the device
 * allocation had failed (LL_ERR_OOM), before any CUDA call, releasing
 * everything it had set up.                                                   */

#ifdef __cplusplus
}
#endif

#endif /* LL_KVATTN_H */
