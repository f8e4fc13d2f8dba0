// cache_layout.cuh - where frames live in the ring cache, shared by the
// kernels (device) and the host-side argument checks (host), so both apply one
// rule.
//
// Per layer and per K/V plane the cache holds (G + Ss + R) frame slots of T rows:
//   [0, G)            global sink: the first G frames of the video
//   [G, G + Ss)       shot sink: the first Ss non-global frames of the current shot
//   [G + Ss, +R)      ring: every other frame; the window is its last W entries
// R = W, or W + F for a cache whose attention call also appends: the F spare
// slots take the chunk's own frames while the same launch still reads the
// window, so the writes never touch a slot that launch reads.
// (LongLive explainer, dpshk.com, sec. 五 and 六: sink frames + recent window;
// LongLive-2.0 explainer, wmrh.cn, sec. 16: a global-level sink all shots
// attend to and a shot-level sink per shot). With Ss = 0 and a single shot the
// ring slot of frame f is G + ((f - G) mod W), the single-shot layout.
#pragma once
#include <cstdint>

namespace llk {

// Frame counters of one layer, in device memory (the host keeps a mirror).
struct LayerCtr {
  long long p;           // frames appended so far
  long long ring_count;  // frames that went to the ring
  long long ring_start;  // ring count when the window was last restarted
  int shot_fill;         // frames in the current shot's sink (0..Ss)
  int reserved;
};
static_assert(sizeof(LayerCtr) == 32, "counter record layout");

struct HeldFrames {
  int g, sf, w;          // held global-sink, shot-sink and window frames
};

__host__ __device__ inline HeldFrames held_frames(long long p, int shot_fill, long long ring_count,
                                                  long long ring_start, int G, int W) {
  HeldFrames h;
  h.g = static_cast<int>(p < G ? p : G);
  h.sf = shot_fill;
  const long long w = ring_count - ring_start;
  h.w = static_cast<int>(w < W ? w : W);
  return h;
}

// Up to three slot ranges (in frames) that hold the visible cache frames: the
// global + shot sink head, then the window's ring range, which wraps into two
// pieces when the window starts mid-ring. When everything up to the end of the
// window is held and the window starts at the ring's first slot (always so
// when the window fills the whole ring), the ranges are merged into one.
struct FrameRanges {
  int start[3], len[3];
  int n;
};

__host__ __device__ inline FrameRanges visible_ranges(const HeldFrames &h, long long ring_count, int G, int Ss,
                                                      int R) {
  // the ranges are built in scalars and stored with constant indices, so that
  // nothing here needs local memory on the device
  int s0 = 0, l0 = 0, s1 = 0, l1 = 0, s2 = 0, l2 = 0, n = 0;
  const int head = h.g < G ? h.g : G + h.sf;   // a shot sink exists only after the global sink is full
  int a = 0;                                    // ring slot of the oldest window frame
  if (h.w > 0 && h.w < R) a = static_cast<int>((ring_count - h.w) % R);
  if (h.w > 0 && h.g == G && h.sf == Ss && a == 0) {
    l0 = G + Ss + h.w;
    n = 1;
  } else {
    if (head > 0) {
      l0 = head;
      n = 1;
    }
    if (h.w > 0) {
      const int first = a + h.w <= R ? h.w : R - a;
      if (n == 0) { s0 = G + Ss + a; l0 = first; } else { s1 = G + Ss + a; l1 = first; }
      ++n;
      if (first < h.w) {
        if (n == 1) { s1 = G + Ss; l1 = h.w - first; } else { s2 = G + Ss; l2 = h.w - first; }
        ++n;
      }
    }
  }
  FrameRanges r;
  r.start[0] = s0; r.len[0] = l0;
  r.start[1] = s1; r.len[1] = l1;
  r.start[2] = s2; r.len[2] = l2;
  r.n = n;
  return r;
}

// Append of a chunk of F frames starting at frame p: frame fi of the chunk
// goes to the returned slot, or to none (-1) when R < F makes a later frame of
// the same chunk overwrite its ring slot, or when R = 0.
__host__ __device__ inline int append_slot(long long p, int shot_fill, long long ring_count, int G, int Ss, int R,
                                           int F, int fi) {
  const long long f = p + fi;
  if (f < G) return static_cast<int>(f);
  const long long global_in_chunk = G - p > 0 ? (G - p < F ? G - p : F) : 0;
  const int j = fi - static_cast<int>(global_in_chunk);     // index among the chunk's non-global frames
  const int room = Ss - shot_fill;
  if (j < room) return G + shot_fill + j;
  const int r = j - room;                                    // index among the chunk's ring frames
  const int n_ring = (F - static_cast<int>(global_in_chunk)) - room;
  if (R == 0 || r < n_ring - R) return -1;
  return G + Ss + static_cast<int>((ring_count + r) % R);
}

// Counter updates of that append: shot-sink fill and ring count after it.
__host__ __device__ inline void append_advance(long long p, int shot_fill, long long ring_count, int G, int Ss,
                                               int F, int *new_fill, long long *new_ring_count) {
  const long long global_in_chunk = G - p > 0 ? (G - p < F ? G - p : F) : 0;
  const int non_global = F - static_cast<int>(global_in_chunk);
  const int room = Ss - shot_fill;
  const int to_shot = non_global < room ? non_global : room;
  *new_fill = shot_fill + to_shot;
  *new_ring_count = ring_count + (non_global - to_shot);
}

// Recache: slot of logical frame k of the held context (global sink, shot
// sink in fill order, window oldest to newest); k < g + sf + w.
__host__ __device__ inline int logical_slot(const HeldFrames &h, long long ring_count, int G, int Ss, int R, int k) {
  if (k < h.g) return k;
  if (k < h.g + h.sf) return G + (k - h.g);
  const long long idx = ring_count - h.w + (k - h.g - h.sf);
  return G + Ss + static_cast<int>(idx % R);
}

}  // namespace llk
