"""CPU oracle for the LongLive sink + window chunk attention and its KV cache.

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, obviously-correct
restatement of what the library computes. Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it. The
CUDA library never calls it, and it shares no code, header, table or helper with
the CUDA path; it never imports the product package.

Precision: attention in fp64 (inputs are exact bf16 values); the quantisers in
IEEE fp32 with round-to-nearest-even, as the cache formats fix them.

Modules
  attention   O1  explicit sink + window + block-causal mask, naive softmax
  cache_model O2  byte-exact replay of create / append / recache on the
                  physical cache layout
  quant       O3  FP8 E4M3 (per-row fp32 scale) and NVFP4 (E2M1, 16-element
                  blocks, E4M3 block scale) encoders and decoders

Parity pins (what each function is checked against, in tests/test_oracle_*.py):
  attention   brute force with Python loops on tiny shapes; textbook block-causal
              attention (torch SDPA, fp64) when the window covers all history;
              closed forms (zero queries -> mean of visible V; one visible key ->
              that key's V); hand-derived visible-frame sets for the pages'
              configuration (tests/golden/).
  cache_model a list/deque simulation of "sink frames + last W frames";
              recache equivalence; constant footprint.
  multi-shot  reduction to the single-shot rule; a hand-derived two-shot
              example (tests/golden/); the cache model's held frames against
              the frame-classification definition; recache equivalence.
  quant       exhaustive code tables; ml_dtypes' round-to-nearest-even casts;
              hand-listed ties and saturation cases (tests/golden/).
"""
from .attention import visible_key_frames, key_mask, sink_window_attention, multishot_visible_frames  # noqa: F401
from .cache_model import CacheModel  # noqa: F401
from . import quant  # noqa: F401
