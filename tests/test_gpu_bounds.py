"""The bounds-checking build (libdkv_bc.so, DKV_BOUNDS_CHECK): every copy
range, side-table index and segment bound the kernels use is checked on the
device, and a failed check records DKV_FLAG_BOUNDS and skips the access.  A
seeded sweep of small random shapes runs on it in a separate process (the
library is chosen when the package is imported) and must match the oracle
with the flag never set."""
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


@pytest.mark.parametrize("seed,n", [(7, 32), (11, 16)])
def test_bounds_checked_sweep(seed, n):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _bc_library()
    env = dict(os.environ, DKV_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bounds_sweep.py"), str(n),
                        str(seed)], env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert r.returncode == 0, out[-4000:]
    assert "library: libdkv_bc.so" in out
    assert f"OK {n} cases" in out
