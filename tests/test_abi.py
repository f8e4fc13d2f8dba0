"""CPU checks of the boundary: the library loads, exports every symbol that
include/ll_kvattn.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ll_kvattn.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LL_API\s+[\w\s\*]+?\b(ll_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("ll_kv_cache_create", "ll_kv_append", "ll_kv_recache_write", "ll_attn_sink_window",
              "ll_kv_cache_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import kv_cache_attention_ll_b200 as ll
    lib = ctypes.CDLL(ll.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings():
    import kv_cache_attention_ll_b200 as ll
    assert ll.ll_status_string(ll.LL_OK) == "ok"
    assert ll.ll_status_string(ll.LL_ERR_TIMEOUT).startswith("in-kernel")
    assert ll.ll_status_string(99) == "unknown status"


@pytest.mark.parametrize("args", [
    (0, 2, 64, 16, 3, 3, 6, 0),      # no layers
    (1, 0, 64, 16, 3, 3, 6, 0),      # no heads
    (1, 2, 96, 16, 3, 3, 6, 0),      # unsupported head_dim
    (1, 2, 64, 0, 3, 3, 6, 0),       # no tokens per frame
    (1, 2, 64, 16, 0, 3, 6, 0),      # no frames per chunk
    (1, 2, 64, 16, 3, -1, 6, 0),     # negative sink
    (1, 2, 64, 16, 3, 0, 0, 0),      # neither sink nor window
    (1, 2, 64, 16, 3, 3, 6, 7),      # unknown dtype
    (1, 2, 64, 1 << 30, 3, 3, 6, 0),  # too many slots
])
def test_create_rejects_bad_arguments_before_cuda(args):
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    h = ctypes.c_void_p(1234)
    assert lib.ll_kv_cache_create(*args, ctypes.byref(h)) == ll.LL_ERR_INVALID_ARG
    assert h.value is None


def test_calls_reject_null_cache():
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    assert lib.ll_kv_append(None, 0, 16, 16, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_kv_recache_write(None, -1, 16, 16, 0, 1, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_attn_sink_window(16, 16, 16, None, 0, 32, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_kv_cache_destroy(None) == ll.LL_OK
    assert lib.ll_kv_export_bytes(None) == 0
    assert lib.ll_allocation_count() == 0


def test_allocation_failure_hook_reports_oom_and_leaks_nothing():
    """Host-side fault injection: the test hook makes create fail as if the
    device allocation had failed; nothing is held afterwards."""
    import os
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    before = lib.ll_allocation_count()
    os.environ["LL_KVATTN_TEST_FAIL_ALLOC"] = "1"
    try:
        h = ctypes.c_void_p(1234)
        assert lib.ll_kv_cache_create(1, 2, 64, 16, 3, 3, 6, 0, ctypes.byref(h)) == ll.LL_ERR_OOM
        assert h.value is None
        with pytest.raises(ll.LLError) as e:
            ll.ll_kv_cache_create(1, 2, 64, 16, 3, 3, 6)
        assert e.value.status == ll.LL_ERR_OOM
    finally:
        del os.environ["LL_KVATTN_TEST_FAIL_ALLOC"]
    assert lib.ll_allocation_count() == before


@pytest.mark.parametrize("args", [
    (1, 2, 64, 16, 3, 3, -1, 6, 0),          # negative shot sink
    (1, 2, 64, 16, 3, 0, 0, 0, 0),           # no frame slots at all
    (1, 32768, 64, 16, 3, 3, 3, 6, 0),       # too many heads for the dequantise grid
    (1, 1, 128, 1 << 25, 1, 3, 3, 2, 0),     # a plane of 2^30 or more vectors
    (1, 2, 64, 16, 3, 3, 3, 6, 3),           # unknown dtype
])
def test_multishot_create_rejects_bad_arguments_before_cuda(args):
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    h = ctypes.c_void_p(1234)
    assert lib.ll_kv_cache_create_multishot(*args, ctypes.byref(h)) == ll.LL_ERR_INVALID_ARG
    assert h.value is None


def test_multishot_calls_reject_null_cache():
    import kv_cache_attention_ll_b200 as ll
    lib = ll.raw_lib()
    g = ctypes.c_int()
    assert lib.ll_kv_shot_begin(None, -1, 0, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_kv_cache_held(None, 0, ctypes.byref(g), None, None) == ll.LL_ERR_INVALID_ARG
    assert lib.ll_debug_wait_selftest(None, None) == ll.LL_ERR_INVALID_ARG


def test_header_is_plain_c_and_links(tmp_path):
    """The boundary is a C ABI: a C99 program that includes the header, takes
    the address of every entry point and calls the ones that need no device
    links against the library and runs."""
    import shutil
    import subprocess
    import kv_cache_attention_ll_b200 as ll
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = _declared()
    src = tmp_path / "use_abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"ll_kvattn.h\"\n"
        "int main(void) {\n"
        "  const void *fns[] = {" + ", ".join(f"(const void *)&{n}" for n in names) + "};\n"
        "  ll_kv_cache *c = (ll_kv_cache *)0;\n"
        "  if (ll_kv_cache_create(0, 1, 64, 1, 1, 1, 1, LL_KV_BF16, &c) != LL_ERR_INVALID_ARG || c) return 1;\n"
        "  if (ll_kv_cache_destroy((ll_kv_cache *)0) != LL_OK) return 2;\n"
        "  if (ll_allocation_count() != 0) return 3;\n"
        "  printf(\"%s %d\\n\", ll_status_string(LL_ERR_TIMEOUT), (int)(sizeof(fns) / sizeof(fns[0])));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(ll.LIB_PATH)
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-lll_kvattn", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.split() == ["in-kernel", "wait", "timed", "out", str(len(names))]


def test_bounds_checking_build_loads_and_exports_every_symbol():
    """The bounds-checking build is a second, complete copy of the library."""
    import kv_cache_attention_ll_b200 as ll
    path = os.path.join(os.path.dirname(ll.LIB_PATH), "libll_kvattn_debug.so")
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n
    assert lib.ll_bounds_checked() == 1
    assert ll.raw_lib().ll_bounds_checked() == 0
