"""Build step of the CUDA library: compiles csrc/ into libll_kvattn.so for
sm_100a, in-tree, next to this file, and the bounds-checking build
libll_kvattn_debug.so (LL_BOUNDS_CHECK: every computed slot, plane and tile
index is checked before its access and a bad one is reported in the status
word). Run `python kv_cache_attention_ll_b200/build.py [--debug]` or call
build(); the Python binding loads the result and refuses to run without it."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libll_kvattn.so")
LIB_DEBUG = os.path.join(HERE, "libll_kvattn_debug.so")
SOURCES = [os.path.join(HERE, "csrc", "ll_kvattn.cu"), os.path.join(HERE, "csrc", "sp_exchange.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in ("attn_sink_window.cuh", "kv_scatter.cuh", "kv_codec.cuh",
                                                           "sm100_ptx.cuh", "cache_layout.cuh")] + [
    os.path.abspath(__file__),
    os.path.join(ROOT, "include", "ll_kvattn.h")]


def nvcc_cmd(out: str = LIB, extra=()) -> list[str]:
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), "-o", out, *SOURCES, *extra]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if force or not up_to_date(lib):
        extra = (("-Xptxas", "-v") if verbose else ()) + (("-DLL_BOUNDS_CHECK",) if debug else ())
        subprocess.run(nvcc_cmd(out=lib, extra=extra), check=True)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
