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

Several shots (LongLive-2.0 explainer, wmrh.cn, sec. 16: a global-level sink
all shots attend to and a shot-level sink per shot). With Ss shot-sink frames
the layout per plane becomes [(S+Ss+W)*T]: slots 0..S-1 global sink,
S..S+Ss-1 shot sink, then the W-slot ring. Each appended frame goes to exactly
one region, in order: f < S -> global slot f; else, while the current shot's
sink holds fewer than Ss frames -> the next shot-sink slot; else -> the next
ring slot, S + Ss + (ring count mod W) (later frames of a chunk overwrite
earlier ones when W < F, so only the last W survive). shot_begin empties the
shot sink (and, if asked, starts the window afresh). Held context, in logical
order: global sink, shot sink (fill order), window (oldest to newest, at most
the last W ring frames since the last window restart). With Ss = 0 and no
shot_begin this is exactly the single-shot rule above.

Spare ring slots (ring_slots = R > W): the ring has R slots and ring frame
number i lives in slot S + Ss + (i mod R); the window is still its last W
frames. With R = W + F the F frames a chunk appends land in slots the window
no longer covers, so attention and append can share one launch. The held
frames are the same as with R = W; only the slots differ.

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
                 frames_per_chunk: int, sink_frames: int, window_frames: int, kv_dtype: str = "bf16",
                 shot_sink_frames: int = 0, ring_slots: int | None = None):
        assert kv_dtype in ("bf16", "fp8", "nvfp4")
        self.L, self.H, self.D = layers, heads, head_dim
        self.T, self.F, self.S, self.W = tokens_per_frame, frames_per_chunk, sink_frames, window_frames
        self.Ss = shot_sink_frames
        self.R = self.W if ring_slots is None else ring_slots
        assert self.R >= self.W
        self.kv_dtype = kv_dtype
        self.slots = (self.S + self.Ss + self.R) * self.T
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
        self.p = [0] * layers              # frames appended
        self.shot_fill = [0] * layers      # frames in the current shot's sink
        self.ring_count = [0] * layers     # frames that went to the ring
        self.ring_start = [0] * layers     # ring count at the last window restart
        self.slot_frame = [dict() for _ in range(layers)]   # frame slot -> absolute frame it holds

    # -- slot rules ---------------------------------------------------------
    def _route(self, layer: int, f: int):
        """Frame slot of absolute frame f, appended next to `layer`, or None;
        advances the shot-sink fill and the ring count."""
        if f < self.S:
            return f
        if self.shot_fill[layer] < self.Ss:
            slot = self.S + self.shot_fill[layer]
            self.shot_fill[layer] += 1
            return slot
        idx = self.ring_count[layer]
        self.ring_count[layer] += 1
        if self.R == 0:
            return None
        return self.S + self.Ss + idx % self.R

    def held(self, layer: int):
        """(global sink frames, window frames) held; see held3 for the shot sink."""
        g, sf, w = self.held3(layer)
        assert self.Ss == 0
        return g, w

    def held3(self, layer: int):
        g = min(self.p[layer], self.S)
        sf = self.shot_fill[layer]
        w = min(self.W, self.ring_count[layer] - self.ring_start[layer])
        return g, sf, w

    def n_held(self, layer: int) -> int:
        return sum(self.held3(layer))

    def logical_slot(self, layer: int, k: int) -> int:
        g, sf, w = self.held3(layer)
        assert 0 <= k < g + sf + w
        if k < g:
            return k
        if k < g + sf:
            return self.S + (k - g)
        idx = self.ring_count[layer] - w + (k - g - sf)
        return self.S + self.Ss + idx % self.R

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
            slot = self._route(layer, p + fi)
            if slot is None:
                continue
            tok = slice(fi * self.T, (fi + 1) * self.T)
            self._store_frame(layer, 0, slot, k_cur[tok])
            self._store_frame(layer, 1, slot, v_cur[tok])
            self.slot_frame[layer][slot] = p + fi
        self.p[layer] = p + self.F

    def shot_begin(self, layer: int, clear_window: bool = False):
        """A new shot starts with the next appended frame (layer -1 = all layers)."""
        for l in (range(self.L) if layer < 0 else [layer]):
            self.shot_fill[l] = 0
            if clear_window:
                self.ring_start[l] = self.ring_count[l]

    def recache_write(self, layer: int, k_new: np.ndarray, v_new: np.ndarray, first: int, num: int):
        """layer -1 = all layers. k_new/v_new: [layers'][num*T][H][D] bf16 bits."""
        layers = range(self.L) if layer < 0 else [layer]
        for li, l in enumerate(layers):
            assert 0 <= first and first + num <= self.n_held(l)
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
        [n_held*T][H][...] (bf16 bits, or codes for the quantised formats)."""
        frames = []
        for k in range(self.n_held(layer)):
            slot = self.logical_slot(layer, k)
            frames.append(np.transpose(self.data[layer, kv, :, slot * self.T:(slot + 1) * self.T], (1, 0, 2)))
        if not frames:
            return np.zeros((0, self.H) + self.data.shape[4:], dtype=self.data.dtype)
        return np.concatenate(frames, axis=0)

    def held_frames(self, layer: int, kv: int) -> dict:
        """Held context as {absolute frame number: fp64 values [T][H][D]}, each
        frame dequantised exactly (bf16 bits, or E4M3 code x fp32 row scale, or
        E2M1 code x E4M3 block scale, in fp64)."""
        out = {}
        for k in range(self.n_held(layer)):
            slot = self.logical_slot(layer, k)
            frame = self.slot_frame[layer][slot]
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
