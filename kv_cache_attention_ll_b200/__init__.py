"""Python binding of libll_kvattn.so (the C ABI in include/ll_kvattn.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels. torch is used for device memory and streams; tensors passed in
must be CUDA, bf16, contiguous, 16-byte aligned, token-major [tokens][H][D].
Raw integer device pointers are accepted too.

Importing this module loads the in-tree library and fails loudly if it is
missing (build it with `python kv_cache_attention_ll_b200/build.py`); there is
no fallback path. With LL_KVATTN_LIB=debug in the environment it loads the
bounds-checking build instead (libll_kvattn_debug.so, built with --debug).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
_VARIANT = os.environ.get("LL_KVATTN_LIB", "")
if _VARIANT not in ("", "release", "debug"):
    raise ImportError(f"LL_KVATTN_LIB={_VARIANT!r}: expected 'debug' or 'release'")
LIB_PATH = os.path.join(_HERE, "libll_kvattn_debug.so" if _VARIANT == "debug" else "libll_kvattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build the CUDA library first "
                      "(python kv_cache_attention_ll_b200/build.py [--debug]); there is no fallback")
_lib = ctypes.CDLL(LIB_PATH)

LL_KV_BF16, LL_KV_FP8_E4M3, LL_KV_NVFP4 = 0, 1, 2
LL_OK, LL_ERR_INVALID_ARG, LL_ERR_OOM, LL_ERR_CUDA, LL_ERR_UNSUPPORTED, LL_ERR_TIMEOUT = range(6)
_DTYPES = {"bf16": LL_KV_BF16, "fp8": LL_KV_FP8_E4M3, "nvfp4": LL_KV_NVFP4}

_vp, _i, _ll, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
_sig = {
    "ll_kv_cache_create": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "ll_kv_append": (_i, [_vp, _i, _vp, _vp, _vp]),
    "ll_kv_recache_write": (_i, [_vp, _i, _vp, _vp, _i, _i, _vp]),
    "ll_attn_sink_window": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _vp]),
    "ll_kv_cache_destroy": (_i, [_vp]),
    "ll_status_string": (ctypes.c_char_p, [_i]),
    "ll_kv_cache_info": (_i, [_vp, _i, ctypes.POINTER(_ll), ctypes.POINTER(_sz)]),
    "ll_allocation_count": (_ll, []),
    "ll_kv_export_bytes": (_sz, [_vp]),
    "ll_kv_cache_export": (_i, [_vp, _i, _vp, _sz, _vp]),
    "ll_debug_status": (_i, [_vp, ctypes.POINTER(ctypes.c_uint), _i, _vp]),
    "ll_attn_sink_window_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _ll, _vp, _vp]),
    "ll_debug_wait_selftest": (_i, [_vp, _vp]),
    "ll_noalloc_debug_status": (_i, [ctypes.POINTER(ctypes.c_uint), _i, _vp]),
    "ll_debug_check_canaries": (_i, [_vp, ctypes.POINTER(_sz)]),
    "ll_bounds_checked": (_i, []),
    "ll_debug_bounds_selftest": (_i, [_vp, _vp]),
    "ll_sp_pack_heads": (_i, [_vp, _i, _i, _i, _i, _vp, _vp]),
    "ll_sp_unpack_heads": (_i, [_vp, _i, _i, _i, _i, _vp, _vp]),
    "ll_sp_pack_heads_fp8": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "ll_sp_dequant_fp8": (_i, [_vp, _vp, _ll, _i, _vp, _vp]),
    "ll_kv_cache_create_multishot": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "ll_kv_shot_begin": (_i, [_vp, _i, _i, _vp]),
    "ll_kv_cache_held": (_i, [_vp, _i, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "ll_kv_cache_create_fused": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "ll_attn_sink_window_append": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _vp]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class LLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {ll_status_string(status)} ({status})")


def ll_status_string(status: int) -> str:
    return _lib.ll_status_string(status).decode()


def _check(status: int, where: str):
    if status != LL_OK:
        raise LLError(status, where)


def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    import torch
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"expected a torch tensor or an int pointer, got {type(x)}")
    if not x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("tensors must be CUDA, bfloat16 and contiguous")
    return x.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class KVCache:
    """Owner of one ll_kv_cache handle (the device memory lives in the library)."""

    def __init__(self, handle: int, layers, heads, head_dim, tokens_per_frame, frames_per_chunk,
                 sink_frames, window_frames, kv_dtype):
        self.handle = handle
        self.layers, self.heads, self.head_dim = layers, heads, head_dim
        self.tokens_per_frame, self.frames_per_chunk = tokens_per_frame, frames_per_chunk
        self.sink_frames, self.window_frames, self.kv_dtype = sink_frames, window_frames, kv_dtype
        self.shot_sink_frames = 0

    @property
    def tq(self) -> int:
        return self.frames_per_chunk * self.tokens_per_frame

    def close(self):
        if self.handle:
            h, self.handle = self.handle, 0
            _check(_lib.ll_kv_cache_destroy(h), "ll_kv_cache_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def ll_kv_cache_create(layers: int, heads: int, head_dim: int, tokens_per_frame: int, frames_per_chunk: int,
                       sink_frames: int, window_frames: int, kv_dtype="bf16") -> KVCache:
    dt = _DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    h = _vp()
    _check(_lib.ll_kv_cache_create(layers, heads, head_dim, tokens_per_frame, frames_per_chunk, sink_frames,
                                   window_frames, dt, ctypes.byref(h)), "ll_kv_cache_create")
    return KVCache(h.value, layers, heads, head_dim, tokens_per_frame, frames_per_chunk, sink_frames,
                   window_frames, kv_dtype)


def ll_kv_cache_create_multishot(layers: int, heads: int, head_dim: int, tokens_per_frame: int,
                                 frames_per_chunk: int, global_sink_frames: int, shot_sink_frames: int,
                                 window_frames: int, kv_dtype="bf16") -> KVCache:
    dt = _DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    h = _vp()
    _check(_lib.ll_kv_cache_create_multishot(layers, heads, head_dim, tokens_per_frame, frames_per_chunk,
                                             global_sink_frames, shot_sink_frames, window_frames, dt,
                                             ctypes.byref(h)), "ll_kv_cache_create_multishot")
    cache = KVCache(h.value, layers, heads, head_dim, tokens_per_frame, frames_per_chunk, global_sink_frames,
                    window_frames, kv_dtype)
    cache.shot_sink_frames = shot_sink_frames
    return cache


def ll_kv_cache_create_fused(layers: int, heads: int, head_dim: int, tokens_per_frame: int, frames_per_chunk: int,
                             global_sink_frames: int, shot_sink_frames: int, window_frames: int,
                             kv_dtype="bf16") -> KVCache:
    """A cache with F spare ring slots, for ll_attn_sink_window_append."""
    dt = _DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    h = _vp()
    _check(_lib.ll_kv_cache_create_fused(layers, heads, head_dim, tokens_per_frame, frames_per_chunk,
                                         global_sink_frames, shot_sink_frames, window_frames, dt, ctypes.byref(h)),
           "ll_kv_cache_create_fused")
    cache = KVCache(h.value, layers, heads, head_dim, tokens_per_frame, frames_per_chunk, global_sink_frames,
                    window_frames, kv_dtype)
    cache.shot_sink_frames = shot_sink_frames
    return cache


def ll_attn_sink_window_append(q, k_cur, v_cur, cache: KVCache, layer: int, out, stream=None):
    """Attention of the chunk, then its append, in one launch (fused caches)."""
    _check(_lib.ll_attn_sink_window_append(_ptr(q), _ptr(k_cur), _ptr(v_cur), cache.handle, layer, _ptr(out),
                                           _stream(stream)), "ll_attn_sink_window_append")


def ll_kv_shot_begin(cache: KVCache, layer: int = -1, clear_window: bool = False, stream=None):
    _check(_lib.ll_kv_shot_begin(cache.handle, layer, int(clear_window), _stream(stream)), "ll_kv_shot_begin")


def ll_kv_cache_held(cache: KVCache, layer: int = 0):
    """(global-sink, shot-sink, window) frames the layer holds now."""
    g, sf, w = _i(), _i(), _i()
    _check(_lib.ll_kv_cache_held(cache.handle, layer, ctypes.byref(g), ctypes.byref(sf), ctypes.byref(w)),
           "ll_kv_cache_held")
    return g.value, sf.value, w.value


def ll_kv_append(cache: KVCache, layer: int, k_cur, v_cur, stream=None):
    _check(_lib.ll_kv_append(cache.handle, layer, _ptr(k_cur), _ptr(v_cur), _stream(stream)), "ll_kv_append")


def ll_kv_recache_write(cache: KVCache, layer: int, k_new, v_new, first_frame: int, num_frames: int, stream=None):
    _check(_lib.ll_kv_recache_write(cache.handle, layer, _ptr(k_new), _ptr(v_new), first_frame, num_frames,
                                    _stream(stream)), "ll_kv_recache_write")


def ll_attn_sink_window(q, k_cur, v_cur, cache: KVCache, layer: int, out, stream=None):
    _check(_lib.ll_attn_sink_window(_ptr(q), _ptr(k_cur), _ptr(v_cur), cache.handle, layer, _ptr(out),
                                    _stream(stream)), "ll_attn_sink_window")


def ll_kv_cache_destroy(cache: KVCache):
    cache.close()


def ll_kv_cache_info(cache: KVCache, layer: int = 0):
    p, b = _ll(), _sz()
    _check(_lib.ll_kv_cache_info(cache.handle, layer, ctypes.byref(p), ctypes.byref(b)), "ll_kv_cache_info")
    return p.value, b.value


def ll_allocation_count() -> int:
    return _lib.ll_allocation_count()


def ll_kv_export_bytes(cache: KVCache) -> int:
    return _lib.ll_kv_export_bytes(cache.handle)


def ll_kv_cache_export(cache: KVCache, layer: int, stream=None) -> bytes:
    n = ll_kv_export_bytes(cache)
    buf = ctypes.create_string_buffer(n)
    _check(_lib.ll_kv_cache_export(cache.handle, layer, ctypes.cast(buf, _vp), n, _stream(stream)),
           "ll_kv_cache_export")
    return buf.raw


def ll_debug_status(cache: KVCache, clear: bool = False, stream=None) -> int:
    """The cache's device status word (0 = fine); see ll_debug_status in the header."""
    if not cache.handle:
        raise ValueError("closed cache")
    w = ctypes.c_uint()
    st = _lib.ll_debug_status(cache.handle, ctypes.byref(w), int(clear), _stream(stream))
    if st not in (LL_OK, LL_ERR_TIMEOUT, LL_ERR_INVALID_ARG):   # the last two report a non-zero word
        _check(st, "ll_debug_status")
    return w.value


def ll_attn_sink_window_noalloc(q, k_cur, v_cur, layer_codes, layer_scales, kv_dtype, heads: int, head_dim: int,
                                tokens_per_frame: int, frames_per_chunk: int, sink_frames: int, window_frames: int,
                                frames_seen: int, out, stream=None):
    """Attention over one quantised cache layer held in caller memory, with no
    device allocation (the scratch is a static device array of the library).
    layer_codes / layer_scales: device buffers (uint8 tensors or pointers) in
    the layout ll_kv_cache_export writes for one layer of a single-shot cache
    (ll_kv_cache_create, no shot start); frames_seen: that layer's counter."""
    dt = _DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    _check(_lib.ll_attn_sink_window_noalloc(_ptr(q), _ptr(k_cur), _ptr(v_cur), _raw_ptr(layer_codes),
                                            _raw_ptr(layer_scales), dt, heads, head_dim, tokens_per_frame,
                                            frames_per_chunk, sink_frames, window_frames, frames_seen, _ptr(out),
                                            _stream(stream)), "ll_attn_sink_window_noalloc")


def ll_noalloc_debug_status(clear: bool = False, stream=None) -> int:
    """Status word of ll_attn_sink_window_noalloc's kernels on the current device (0 = fine)."""
    w = ctypes.c_uint()
    st = _lib.ll_noalloc_debug_status(ctypes.byref(w), int(clear), _stream(stream))
    if st not in (LL_OK, LL_ERR_TIMEOUT, LL_ERR_INVALID_ARG):
        _check(st, "ll_noalloc_debug_status")
    return w.value


def ll_sp_pack_heads(x, tokens: int, heads: int, head_dim: int, ranks: int, packed, stream=None):
    """[tokens][heads][D] -> [ranks][tokens][heads/ranks][D] (bf16)."""
    _check(_lib.ll_sp_pack_heads(_ptr(x), tokens, heads, head_dim, ranks, _ptr(packed), _stream(stream)),
           "ll_sp_pack_heads")


def ll_sp_unpack_heads(packed, tokens: int, heads: int, head_dim: int, ranks: int, x, stream=None):
    """[ranks][tokens][heads/ranks][D] -> [tokens][heads][D] (bf16)."""
    _check(_lib.ll_sp_unpack_heads(_ptr(packed), tokens, heads, head_dim, ranks, _ptr(x), _stream(stream)),
           "ll_sp_unpack_heads")


def ll_sp_pack_heads_fp8(x, tokens: int, heads: int, head_dim: int, ranks: int, codes, scales, stream=None):
    """As ll_sp_pack_heads, each row as E4M3 codes + an fp32 power-of-two scale."""
    _check(_lib.ll_sp_pack_heads_fp8(_ptr(x), tokens, heads, head_dim, ranks, _raw_ptr(codes), _raw_ptr(scales),
                                     _stream(stream)), "ll_sp_pack_heads_fp8")


def ll_sp_dequant_fp8(codes, scales, rows: int, head_dim: int, x, stream=None):
    """FP8 rows (codes, scales) -> bf16 rows [rows][D]."""
    _check(_lib.ll_sp_dequant_fp8(_raw_ptr(codes), _raw_ptr(scales), rows, head_dim, _ptr(x), _stream(stream)),
           "ll_sp_dequant_fp8")


def _raw_ptr(x) -> int:
    """Device pointer of a byte buffer (any dtype, contiguous CUDA tensor) or an int."""
    if isinstance(x, int):
        return x
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("buffers must be contiguous CUDA tensors")
    return x.data_ptr()


def ll_debug_check_canaries(cache: KVCache) -> int:
    """-1 if every guard byte around the cache's regions is intact, else the
    allocation offset of the first changed byte."""
    off = _sz()
    st = _lib.ll_debug_check_canaries(cache.handle, ctypes.byref(off))
    if st == LL_OK:
        return -1
    if st == LL_ERR_INVALID_ARG and off.value != ctypes.c_size_t(-1).value:
        return off.value
    _check(st, "ll_debug_check_canaries")
    return -1


def ll_bounds_checked() -> bool:
    """True for the bounds-checking build of the library."""
    return bool(_lib.ll_bounds_checked())


def ll_debug_bounds_selftest(cache: KVCache, stream=None):
    _check(_lib.ll_debug_bounds_selftest(cache.handle, _stream(stream)), "ll_debug_bounds_selftest")


def ll_debug_wait_selftest(cache: KVCache, stream=None):
    _check(_lib.ll_debug_wait_selftest(cache.handle, _stream(stream)), "ll_debug_wait_selftest")


def raw_lib():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib
