"""Build step of the CUDA library: compiles csrc/ into libll_kvattn.so for
sm_100a, in-tree, next to this file. Run `python kv_cache_attention_ll_b200/build.py`
or call build(); the Python binding loads the result and refuses to run
without it."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libll_kvattn.so")
SOURCES = [os.path.join(HERE, "csrc", "ll_kvattn.cu"), os.path.join(HERE, "csrc", "sp_exchange.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in ("attn_sink_window.cuh", "kv_scatter.cuh",
                                                           "sm100_ptx.cuh", "cache_layout.cuh")] + [
    os.path.join(ROOT, "include", "ll_kvattn.h")]


def nvcc_cmd(out: str = LIB, extra=()) -> list[str]:
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), "-o", out, *SOURCES, *extra]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        cmd = nvcc_cmd(extra=("-Xptxas", "-v") if verbose else ())
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
