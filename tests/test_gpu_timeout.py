"""Failure detection in the tcgen05 attention kernel: its bounded waits run
out (a test hook of the bounds-checking build withholds one tile's copies) and
the call returns with DKV_FLAG_TIMEOUT instead of hanging; later calls are
correct.  Runs tests/timeout_check.py in its own process on libdkv_bc.so (the
library is chosen when the package is imported).  The normal build refuses
the hook."""
import importlib.util
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bc_library() -> str:
    spec = importlib.util.spec_from_file_location(
        "_dkv_build", os.path.join(ROOT, "quantized_kv_cache_dkv_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build(bounds_check=True)


def test_bounded_wait_timeout_path():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _bc_library()
    env = dict(os.environ, DKV_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "timeout_check.py")],
                       env=env, capture_output=True, text=True, timeout=300)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert "library: libdkv_bc.so" in out
    assert "OK timeout path" in out


def test_normal_build_refuses_the_stall_hook():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as dkv
    if os.path.basename(dkv.LIB_PATH) != "libdkv.so":
        pytest.skip("runs on the normal build")
    cache = dkv.dkv_cache_alloc(dkv.make_config(1, 4, 1, 128, 32, 4, 4, 32, 32, 0, 64))
    with pytest.raises(dkv.DkvError) as ei:
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_TEST_STALL, 0)
    assert ei.value.code == dkv.DKV_ERR_UNSUPPORTED
    dkv.dkv_cache_free(cache)
