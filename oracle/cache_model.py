"""O2 - byte-exact host model of the sink + ring-window KV cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Behaviour fixed by the pages:
* KV cache = K/V of the sink frames + K/V of the recent window
  (LongLive explainer, dpshk.com, sec. 六); the sink frames are kept for the whole
  rollout; frames that fall out of the short window are evicted (sec. 五);
  memory stays constant as the video grows (techwalker.com LONGLIVE article, sec. 四).
* On a prompt switch the cache of the sink + recent-window context is recomputed
  and rewritten (dpshk.com sec. 三.3 and 三.5; techwalker.com sec. 六 names the
  window-only variant with the sink unchanged).

Readings taken where the pages are silent (the library follows the same ones):
* Layout per layer, per K and V:  [H][(S+W)*T][D]; slots 0..S-1 hold the sink
  frames, slots S..S+W-1 are a frame-granular ring holding the window.
* Append of chunk frames f = p .. p+F-1 (p = frames appended before):
    f < S                       -> slot f                  (sink)
    f >= S and f >= p + F - W   -> slot S + ((f - S) mod W) (ring; the oldest
                                   window frame is the one overwritten)
    otherwise (only when W < F) -> not stored
  then p += F.
* Recache: logical frame k of the held context (sink 0..s-1, then window frames
  oldest to newest), s = min(p, S), w = min(W, max(0, p - S)):
    k < s  -> slot k;   else absolute frame a = p - w + (k - s) -> slot S + ((a - S) mod W).
  p is unchanged.
* Inputs are token-major [tokens][H][D] bf16; the source of a recache is
  [layers'][n*T][H][D] with layers' = 1 for one layer, L for all layers.

Stored formats: "bf16" raw bits; "fp8" E4M3 codes + one fp32 scale per
(token, head) row; "nvfp4" packed E2M1 codes + one E4M3 scale per 16 values.
Export of a layer = data of K, data of V, then (quantised formats) scales of K,
scales of V, each C-contiguous [H][slots][...].
"""
from __future__ import annotations

import numpy as np

from . import quant


class CacheModel:
    def __init__(self, layers: int, heads: int, head_dim: int, tokens_per_frame: int,
                 frames_per_chunk: int, sink_frames: int, window_frames: int, kv_dtype: str = "bf16"):
        assert kv_dtype in ("bf16", "fp8", "nvfp4")
        self.L, self.H, self.D = layers, heads, head_dim
        self.T, self.F, self.S, self.W = tokens_per_frame, frames_per_chunk, sink_frames, window_frames
        self.kv_dtype = kv_dtype
        self.slots = (self.S + self.W) * self.T
        shape = (layers, 2, heads, self.slots)
        if kv_dtype == "bf16":
            self.data = np.zeros(shape + (head_dim,), dtype=np.uint16)
            self.scales = None
        elif kv_dtype == "fp8":
            self.data = np.zeros(shape + (head_dim,), dtype=np.uint8)
            self.scales = np.zeros(shape, dtype=np.float32)
        else:
            self.data = np.zeros(shape + (head_dim // 2,), dtype=np.uint8)
            self.scales = np.zeros(shape + (head_dim // 16,), dtype=np.uint8)
        self.p = [0] * layers

    # -- slot rules ---------------------------------------------------------
    def append_slot(self, f: int, p: int):
        """Physical frame slot of absolute frame f appended in a chunk that starts at p, or None."""
        if f < self.S:
            return f
        if self.W > 0 and f >= p + self.F - self.W:
            return self.S + (f - self.S) % self.W
        return None

    def held(self, layer: int):
        p = self.p[layer]
        s = min(p, self.S)
        w = min(self.W, max(0, p - self.S))
        return s, w

    def logical_slot(self, layer: int, k: int) -> int:
        p = self.p[layer]
        s, w = self.held(layer)
        assert 0 <= k < s + w
        if k < s:
            return k
        a = p - w + (k - s)
        return self.S + (a - self.S) % self.W

    # -- writes -------------------------------------------------------------
    def _store_frame(self, layer: int, kv: int, slot: int, src_bits: np.ndarray):
        """src_bits: [T][H][D] bf16 bits of one frame -> physical rows of `slot`."""
        rows = np.transpose(src_bits, (1, 0, 2))              # [H][T][D]
        sl = slice(slot * self.T, (slot + 1) * self.T)
        if self.kv_dtype == "bf16":
            self.data[layer, kv, :, sl, :] = rows
        elif self.kv_dtype == "fp8":
            codes, sc = quant.fp8_quantize_rows(rows)
            self.data[layer, kv, :, sl, :] = codes
            self.scales[layer, kv, :, sl] = sc
        else:
            codes, sb = quant.nvfp4_quantize_rows(rows)
            self.data[layer, kv, :, sl, :] = codes
            self.scales[layer, kv, :, sl, :] = sb

    def append(self, layer: int, k_cur: np.ndarray, v_cur: np.ndarray):
        """k_cur, v_cur: [F*T][H][D] bf16 bits of the chunk just generated."""
        p = self.p[layer]
        for fi in range(self.F):
            slot = self.append_slot(p + fi, p)
            if slot is None:
                continue
            tok = slice(fi * self.T, (fi + 1) * self.T)
            self._store_frame(layer, 0, slot, k_cur[tok])
            self._store_frame(layer, 1, slot, v_cur[tok])
        self.p[layer] = p + self.F

    def recache_write(self, layer: int, k_new: np.ndarray, v_new: np.ndarray, first: int, num: int):
        """layer -1 = all layers. k_new/v_new: [layers'][num*T][H][D] bf16 bits."""
        layers = range(self.L) if layer < 0 else [layer]
        for li, l in enumerate(layers):
            s, w = self.held(l)
            assert 0 <= first and first + num <= s + w
            for fi in range(num):
                slot = self.logical_slot(l, first + fi)
                tok = slice(fi * self.T, (fi + 1) * self.T)
                self._store_frame(l, 0, slot, k_new[li][tok])
                self._store_frame(l, 1, slot, v_new[li][tok])

    # -- reads --------------------------------------------------------------
    def export(self, layer: int) -> bytes:
        parts = [self.data[layer, 0].tobytes(), self.data[layer, 1].tobytes()]
        if self.scales is not None:
            parts += [self.scales[layer, 0].tobytes(), self.scales[layer, 1].tobytes()]
        return b"".join(parts)

    def export_nbytes(self) -> int:
        n = self.data[0].nbytes
        if self.scales is not None:
            n += self.scales[0].nbytes
        return n

    def logical_view(self, layer: int, kv: int) -> np.ndarray:
        """Stored rows of the held context in logical order, token-major:
        [(s+w)*T][H][...] (bf16 bits, or codes for the quantised formats)."""
        s, w = self.held(layer)
        frames = []
        for k in range(s + w):
            slot = self.logical_slot(layer, k)
            frames.append(np.transpose(self.data[layer, kv, :, slot * self.T:(slot + 1) * self.T], (1, 0, 2)))
        if not frames:
            return np.zeros((0, self.H) + self.data.shape[4:], dtype=self.data.dtype)
        return np.concatenate(frames, axis=0)

    def held_frames(self, layer: int, kv: int) -> dict:
        """Held context as {absolute frame number: fp64 values [T][H][D]}: the sink
        frames 0..s-1 and the window frames p-w..p-1, each dequantised exactly
        (bf16 bits, or E4M3 code x fp32 row scale, or E2M1 code x E4M3 block
        scale, in fp64)."""
        p = self.p[layer]
        s, w = self.held(layer)
        out = {}
        for k in range(s + w):
            frame = k if k < s else p - w + (k - s)
            slot = self.logical_slot(layer, k)
            sl = slice(slot * self.T, (slot + 1) * self.T)
            if self.kv_dtype == "bf16":
                rows = (self.data[layer, kv, :, sl].astype(np.uint32) << np.uint32(16)).view(np.float32) \
                    .astype(np.float64)
            elif self.kv_dtype == "fp8":
                rows = quant.fp8_dequantize_rows(self.data[layer, kv, :, sl], self.scales[layer, kv, :, sl])
            else:
                rows = quant.nvfp4_dequantize_rows(self.data[layer, kv, :, sl], self.scales[layer, kv, :, sl])
            out[frame] = np.transpose(rows, (1, 0, 2))
        return out
