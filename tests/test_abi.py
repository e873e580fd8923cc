"""The C-ABI library loads, exports every function include/dkv.h declares, and
rejects bad configurations on the host before touching the GPU.  CPU only:
no call here launches a kernel."""
import ctypes
import subprocess

import pytest

import quantized_kv_cache_dkv_b200 as dkv


def _check_exports(path):
    names = dkv.header_symbols()
    assert "dkv_commit_block" in names and "dkv_block_attention" in names
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(path)
    for n in names:
        assert getattr(lib, n) is not None


def test_library_exports_every_header_symbol():
    _check_exports(dkv.LIB_PATH)


def test_bounds_checking_library_exports_every_header_symbol():
    """libdkv_bc.so (the DKV_BOUNDS_CHECK build) has the same boundary."""
    import os
    path = os.path.join(os.path.dirname(dkv.__file__), "libdkv_bc.so")
    if not os.path.exists(path):
        pytest.skip("libdkv_bc.so not built (build.py --bounds-check)")
    _check_exports(path)


def _alloc_rc(**over):
    cfg = dict(B=1, Hq=4, Hkv=1, d=128, blk=32, k_bits=4, v_bits=4, k_group=32, v_group=32,
               max_protected=0, max_tokens=256)
    cfg.update(over)
    c = dkv.make_config(**cfg)
    h = ctypes.c_void_p()
    return dkv._alloc(ctypes.byref(c), None, ctypes.byref(h)), dkv._lib.dkv_last_error().decode()


@pytest.mark.parametrize("over,code", [
    (dict(d=64), dkv.DKV_ERR_UNSUPPORTED),
    (dict(k_bits=5), dkv.DKV_ERR_UNSUPPORTED),
    (dict(B=513), dkv.DKV_ERR_UNSUPPORTED),
    (dict(v_bits=8), dkv.DKV_ERR_UNSUPPORTED),
    (dict(k_group=48), dkv.DKV_ERR_UNSUPPORTED),
    (dict(v_group=16), dkv.DKV_ERR_UNSUPPORTED),
    (dict(blk=48), dkv.DKV_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=4), dkv.DKV_ERR_INVALID_ARG),
    (dict(Hq=16, Hkv=1, blk=32), dkv.DKV_ERR_UNSUPPORTED),     # 512 query rows per kv-head
    (dict(max_tokens=100), dkv.DKV_ERR_INVALID_ARG),
    (dict(k_group=64, max_tokens=96), dkv.DKV_ERR_INVALID_ARG),
    (dict(B=0), dkv.DKV_ERR_INVALID_ARG),
    (dict(max_protected=-1), dkv.DKV_ERR_INVALID_ARG),
    (dict(sink_tokens=-1), dkv.DKV_ERR_INVALID_ARG),
    (dict(sink_tokens=257), dkv.DKV_ERR_INVALID_ARG),
    (dict(sink_tokens=64, max_tokens=32, blk=32), dkv.DKV_ERR_INVALID_ARG),
])
def test_bad_config_rejected_on_host(over, code):
    rc, msg = _alloc_rc(**over)
    assert rc == code
    assert msg


def test_valid_config_without_a_device_fails_cleanly():
    """On a machine without a usable CUDA device a valid configuration passes
    the host checks and then fails with DKV_ERR_CUDA and a message; no handle
    is returned."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    c = dkv.make_config(1, 4, 1, 128, 32, 4, 4, 32, 32, 0, 256)
    h = ctypes.c_void_p(12345)
    rc = dkv._alloc(ctypes.byref(c), None, ctypes.byref(h))
    assert rc == dkv.DKV_ERR_CUDA
    assert h.value is None
    assert dkv._lib.dkv_last_error().decode()


def test_null_arguments_rejected():
    P = ctypes.c_void_p
    assert dkv._commit(None, P(16), P(16), None, None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv._attn(None, P(16), P(16), P(16), ctypes.c_float(1.0), P(16), None) == \
        dkv.DKV_ERR_INVALID_ARG
    n = ctypes.c_int64()
    assert dkv._len(None, ctypes.byref(n)) == dkv.DKV_ERR_INVALID_ARG
    assert dkv._free(None) == dkv.DKV_ERR_INVALID_ARG
    assert dkv._setopt(None, 1, 0) == dkv.DKV_ERR_INVALID_ARG
    assert dkv._setrot(None, None, None, 32) == dkv.DKV_ERR_INVALID_ARG
    assert dkv._attn_dual(None, None, P(16), P(16), P(16), ctypes.c_float(1.0), P(16), None) == \
        dkv.DKV_ERR_INVALID_ARG
    assert "NULL" in dkv._lib.dkv_last_error().decode()


def test_package_refuses_to_load_without_library(tmp_path):
    """The binding has no fallback: a copy of the package without the .so
    fails at import."""
    import shutil
    import sys
    pkg = tmp_path / "quantized_kv_cache_dkv_b200"
    shutil.copytree(dkv.__path__[0], pkg, ignore=shutil.ignore_patterns("*.so", "_build"))
    r = subprocess.run([sys.executable, "-c", "import quantized_kv_cache_dkv_b200"],
                       cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "libdkv.so is missing" in r.stderr


def test_header_is_plain_c_and_links_from_c(tmp_path):
    """include/dkv.h compiles as strict C99, and a C program links against
    libdkv.so and gets the documented host-side error codes (no GPU call)."""
    import os
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "abi_check.c"
    src.write_text(
        '#include <stdio.h>\n#include <string.h>\n#include "dkv.h"\n'
        "int main(void) {\n"
        "  int64_t n = 0;\n"
        "  if (dkv_cache_len(0, &n) != DKV_ERR_INVALID_ARG) return 1;\n"
        "  if (strlen(dkv_last_error()) == 0) return 2;\n"
        "  if (dkv_cache_free(0) != DKV_ERR_INVALID_ARG) return 3;\n"
        "  dkv_config c; memset(&c, 0, sizeof c);\n"
        "  dkv_cache* h = 0;\n"
        "  if (dkv_cache_alloc(&c, 0, &h) != DKV_ERR_INVALID_ARG || h != 0) return 4;\n"
        '  printf("ok\\n");\n  return 0;\n}\n')
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(dkv.LIB_PATH)
    libname = os.path.basename(dkv.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(root, "include"), str(src), "-o", str(exe),
                        os.path.join(libdir, libname), "-Wl,-rpath," + libdir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
