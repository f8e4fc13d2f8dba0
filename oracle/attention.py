"""O1 - sink + window + own-chunk attention, written as its plain definition.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed, and where the pages fix it:

* Generation is chunk-level causal autoregression: chunk c is produced from the
  chunks before it, whose self-attention K/V sit in the KV cache
  (LongLive explainer, dpshk.com, sec. 二; LongLive-2.0 explainer, wmrh.cn, sec. 3).
* Keys visible to the queries of chunk c
    - the own chunk, with full attention inside it; nothing from a later chunk
      (LongLive-2.0 explainer, sec. 6: a noisy chunk sees the clean earlier
      chunks and itself, never the future);
    - the frame sink: the first S latent frames, kept for the whole rollout
      (dpshk.com sec. 六; techwalker.com LONGLIVE article, sec. 四 and 六);
    - the short window: the most recent W latent frames before the chunk, older
      ones evicted (dpshk.com sec. 五; techwalker.com sec. 四 and 六: chunk 3,
      window 9, sink = first 3 latent frames).
  A frame below S is a sink frame only; the window is the last W frames that
  precede the chunk and are not sink frames.
* Attention itself: o_i = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j over the
  visible keys j, per head. The 1/sqrt(D) scale is the standard scaled
  dot-product scale; the pages print no other.

The mask is built over the full token history (frame f_j = j // T of every key
token j), not over cache slots: the oracle knows nothing about the ring buffer.
"""
from __future__ import annotations

import numpy as np


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values; float arrays pass through
    (used for caches whose held values are dequantised products)."""
    a = np.asarray(bits)
    if np.issubdtype(a.dtype, np.floating):
        return a.astype(np.float64)
    return (a.astype(np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def frame_visible(query_frame: int, key_frame: int, S: int, W: int, F: int) -> bool:
    """Is key frame `key_frame` visible to a query in frame `query_frame`?"""
    cq = query_frame // F
    ck = key_frame // F
    if ck == cq:
        return True            # own chunk: full attention inside the chunk
    if ck > cq:
        return False           # a later chunk: never visible
    if key_frame < S:
        return True            # frame sink
    return key_frame >= cq * F - W   # one of the last W frames before the chunk


def visible_key_frames(chunk: int, S: int, W: int, F: int) -> list[int]:
    """Sorted list of the frames whose keys the queries of `chunk` see."""
    return [f for f in range((chunk + 1) * F) if frame_visible(chunk * F, f, S, W, F)]


def multishot_visible_frames(chunk: int, G: int, Ss: int, W: int, F: int, shots=()) -> list[int]:
    """Frames whose keys the queries of `chunk` see when the video has several shots.

    LongLive-2.0 explainer (wmrh.cn, sec. 16): a global-level sink that every
    shot attends to (identity, style, long-term context) and a shot-level sink
    that keeps the current shot's own early frames; the short recent window of
    LongLive (dpshk.com sec. 五) stays. Readings where the page is silent:
      * the global sink is the first G frames of the video;
      * the shot sink of a shot is its first Ss frames that are not global-sink
        frames; a new shot empties it (its old frames are no longer seen);
      * every other frame is a window frame; the window is the last W window
        frames before the chunk, across shots, counted from the last shot start
        that asked to clear it;
      * the chunk's own frames are fully visible.
    shots: (start_chunk, clear_window) of every shot after the first, which
    starts at chunk 0. With Ss = 0 and no shots this is visible_key_frames.
    """
    starts = sorted(shots)
    assert all(0 < c for c, _ in starts)

    def shot_start_frame(f):
        b = 0
        for c, _ in starts:
            if c * F <= f:
                b = c * F
        return b

    def is_shot_sink(f):
        lo = max(shot_start_frame(f), G)
        return f >= G and f - lo < Ss

    first = chunk * F
    cur_lo = max(shot_start_frame(first), G)
    clear_from = 0
    for c, clear in starts:
        if c <= chunk and clear:
            clear_from = c * F
    global_sink = [f for f in range(min(G, first))]
    shot_sink = [f for f in range(cur_lo, min(cur_lo + Ss, first))]
    window_frames = [f for f in range(max(G, clear_from), first) if not is_shot_sink(f)]
    window = window_frames[max(0, len(window_frames) - W):] if W > 0 else []
    own = list(range(first, first + F))
    return sorted(set(global_sink) | set(shot_sink) | set(window) | set(own))


def key_mask(chunk: int, query_rows: np.ndarray, n_key_tokens: int, S: int, W: int, F: int, T: int) -> np.ndarray:
    """Explicit boolean mask [len(query_rows)][n_key_tokens].

    query_rows are token indices inside the chunk (0..F*T-1); key token j belongs
    to frame j // T of the history.
    """
    q_frame = chunk * F + np.asarray(query_rows) // T           # [R]
    k_frame = np.arange(n_key_tokens) // T                        # [N]
    cq = (q_frame // F)[:, None]
    ck = (k_frame // F)[None, :]
    kf = k_frame[None, :]
    own = ck == cq
    past = ck < cq
    sink = kf < S
    window = kf >= cq * F - W
    return own | (past & (sink | window))


def sink_window_attention(q_bits: np.ndarray, k_hist_bits: np.ndarray, v_hist_bits: np.ndarray,
                          chunk: int, S: int, W: int, F: int, T: int,
                          rows=None, row_block: int = 256, visible_frames=None) -> np.ndarray:
    """Attention output of chunk `chunk` in fp64.

    q_bits       [F*T][H][D] bf16 bits, the chunk's queries
    k_hist_bits  [(chunk+1)*F*T][H][D] bf16 bits (or float values): K of every frame
                 generated so far, in generation order, the current chunk's K last
    v_hist_bits  same for V
    rows         optional subset of query rows (token index in the chunk)
    visible_frames  optional explicit set of visible frames (e.g. from
                 multishot_visible_frames), used instead of the S/W rule
    returns      [len(rows)][H][D] float64
    """
    Tq, H, D = q_bits.shape
    assert Tq == F * T
    n_keys = k_hist_bits.shape[0]
    assert n_keys == (chunk + 1) * F * T, "history must hold every frame up to the current chunk"
    rows = np.arange(Tq) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), H, D), dtype=np.float64)
    scale = 1.0 / np.sqrt(D)
    for h in range(H):
        k = _bf16_to_f64(k_hist_bits[:, h, :])                      # [N][D]
        v = _bf16_to_f64(v_hist_bits[:, h, :])
        for r0 in range(0, len(rows), row_block):
            rr = rows[r0:r0 + row_block]
            q = _bf16_to_f64(q_bits[rr, h, :])                      # [R][D]
            if visible_frames is None:
                mask = key_mask(chunk, rr, n_keys, S, W, F, T)      # [R][N]
            else:
                vis = np.zeros(n_keys // T, dtype=bool)
                vis[list(visible_frames)] = True
                mask = np.broadcast_to(vis[np.arange(n_keys) // T][None, :], (len(rr), n_keys))
            s = (q @ k.T) * scale
            s = np.where(mask, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            out[r0:r0 + len(rr), h, :] = p @ v
    return out
