"""The frame-slot rules of cache_layout.cuh, compiled for the host, against the
oracle's cache model, with no GPU.

The kernels take every slot decision from cache_layout.cuh: the slot of each
appended frame (append_slot) and the counter update after it (append_advance),
the held frames (held_frames), the slot of each held frame in logical order
(logical_slot, used by the recache), and the visible slot ranges the attention
walks (visible_ranges). A small host program built from that header with g++
replays seeded sequences of appends and shot starts (with and without a window
restart) for many cache geometries, and its answers are compared with
oracle.CacheModel after every step: the same slots for every stored frame (-1
for a frame a later frame of the same chunk overwrites), the same held
frames, the same logical slots, and visible ranges that cover exactly the held
slots, each once."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import CacheModel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_attention_ll_b200", "csrc")

HARNESS = r"""
#define __host__
#define __device__
#include "cache_layout.cuh"
#include <cstdio>
using namespace llk;
int main() {
  int G, Ss, W, R, F, n_ops;
  if (scanf("%d %d %d %d %d %d", &G, &Ss, &W, &R, &F, &n_ops) != 6) return 1;
  long long p = 0, rc = 0, rs = 0;
  int fill = 0;
  for (int i = 0; i < n_ops; ++i) {
    char op[8];
    int arg;
    if (scanf("%7s %d", op, &arg) != 2) return 1;
    if (op[0] == 'A') {
      printf("A");
      for (int fi = 0; fi < F; ++fi) printf(" %d", append_slot(p, fill, rc, G, Ss, R, F, fi));
      printf("\n");
      int nf;
      long long nrc;
      append_advance(p, fill, rc, G, Ss, F, &nf, &nrc);
      p += F;
      fill = nf;
      rc = nrc;
    } else {
      fill = 0;
      if (arg) rs = rc;
      printf("S\n");
    }
    const HeldFrames h = held_frames(p, fill, rc, rs, G, W);
    printf("H %d %d %d", h.g, h.sf, h.w);
    for (int k = 0; k < h.g + h.sf + h.w; ++k) printf(" %d", logical_slot(h, rc, G, Ss, R, k));
    printf("\n");
    const FrameRanges r = visible_ranges(h, rc, G, Ss, R);
    printf("V %d", r.n);
    for (int j = 0; j < r.n; ++j) printf(" %d %d", r.start[j], r.len[j]);
    printf("\n");
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not available")
    d = tmp_path_factory.mktemp("layout")
    src = d / "harness.cpp"
    src.write_text(HARNESS)
    exe = d / "harness"
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)], check=True)
    return str(exe)


def _ops(seed: int, n: int, shots: bool):
    rng = np.random.default_rng(seed)
    ops = []
    for _ in range(n):
        if shots and rng.random() < 0.15:
            ops.append(("S", int(rng.random() < 0.5)))
        else:
            ops.append(("A", 0))
    return ops


def _run(harness, G, Ss, W, R, F, ops):
    text = f"{G} {Ss} {W} {R} {F} {len(ops)}\n" + "".join(f"{o} {a}\n" for o, a in ops)
    out = subprocess.run([harness], input=text, capture_output=True, text=True, check=True).stdout
    return [line.split() for line in out.splitlines()]


GEOMETRIES = [
    # G (global sink), Ss (shot sink), W (window), F (chunk frames), spare ring slots
    (3, 0, 9, 3, False),       # the Wan configuration
    (3, 0, 9, 3, True),        # with the fused call's F spare ring slots
    (3, 0, 6, 3, False),
    (0, 0, 4, 2, False),       # no sink
    (3, 0, 0, 2, False),       # sink only
    (1, 0, 2, 3, False),       # window shorter than a chunk
    (2, 0, 5, 1, True),
    (1, 2, 3, 1, False),       # multi-shot
    (2, 3, 6, 3, False),
    (3, 3, 6, 3, True),
    (1, 1, 2, 3, False),       # multi-shot, window shorter than a chunk
    (0, 2, 4, 2, False),       # shot sink without a global sink
]


@pytest.mark.parametrize("G,Ss,W,F,spare", GEOMETRIES)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_slot_rules_match_the_oracle(harness, G, Ss, W, F, spare, seed):
    R = W + F if spare else W
    ops = _ops(seed * 100 + G * 10 + W, 60, shots=Ss > 0 or seed == 2)
    lines = _run(harness, G, Ss, W, R, F, ops)
    model = CacheModel(1, 1, 16, 1, F, G, W, "bf16", shot_sink_frames=Ss, ring_slots=R)
    zeros = np.zeros((F, 1, 16), np.uint16)
    li = 0
    for op, arg in ops:
        line = lines[li]
        li += 1
        if op == "A":
            p = model.p[0]
            model.append(0, zeros, zeros)
            where = {frame: slot for slot, frame in model.slot_frame[0].items()}
            want = [where.get(p + fi, -1) for fi in range(F)]
            assert line[0] == "A" and [int(x) for x in line[1:]] == want, (op, p, line, want)
        else:
            model.shot_begin(0, bool(arg))
            assert line == ["S"]
        held = lines[li]
        vis = lines[li + 1]
        li += 2
        g, sf, w = model.held3(0)
        n = g + sf + w
        assert held[0] == "H" and [int(x) for x in held[1:4]] == [g, sf, w]
        slots = [model.logical_slot(0, k) for k in range(n)]
        assert [int(x) for x in held[4:]] == slots
        assert vis[0] == "V"
        covered = []
        for j in range(int(vis[1])):
            s0, ln = int(vis[2 + 2 * j]), int(vis[3 + 2 * j])
            covered += list(range(s0, s0 + ln))
        assert sorted(covered) == sorted(slots), "the visible ranges cover exactly the held slots, once each"
