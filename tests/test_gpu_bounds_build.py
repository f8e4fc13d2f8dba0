"""The bounds-checking build (libll_kvattn_debug.so, LL_BOUNDS_CHECK).

Compute-sanitizer cannot be run here, so a second build of the library checks,
before each access, the slot rows, planes and source vectors that the
append/recache, dequantise and attention kernels compute, and every cache tile
a TMA load addresses; a bad index is recorded in the cache's status word and
the access is skipped. The cache tests, the randomised operation sequences,
the multi-shot, fused, graph and sequence-parallel tests then run against that
build in a child process: every status word they check must stay 0. The
reporting path itself is exercised by a self-test check that fails on purpose
and accesses nothing."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_failed_check_is_reported_in_the_status_word():
    import kv_cache_attention_ll_b200 as ll
    cache = ll.ll_kv_cache_create(1, 1, 64, 4, 1, 1, 1)
    try:
        ll.ll_debug_bounds_selftest(cache)
        assert ll.ll_debug_status(cache, clear=True) == (4 << 8) | 4      # self-test kernel, index check
        assert ll.ll_debug_status(cache) == 0
    finally:
        cache.close()


def test_gpu_suites_pass_under_the_bounds_checking_build():
    env = dict(os.environ, LL_KVATTN_LIB="debug")
    probe = subprocess.run([sys.executable, "-c", "import kv_cache_attention_ll_b200 as ll; "
                            "assert ll.ll_bounds_checked() and ll.LIB_PATH.endswith('libll_kvattn_debug.so')"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert probe.returncode == 0, probe.stderr[-2000:]
    suites = ["tests/test_gpu_cache.py", "tests/test_gpu_random_ops.py", "tests/test_gpu_multishot.py",
              "tests/test_gpu_fused.py", "tests/test_gpu_graph.py", "tests/test_gpu_sp.py",
              "tests/test_gpu_attention.py::test_odd_shapes_all_chunks"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider", *suites],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-2000:])
