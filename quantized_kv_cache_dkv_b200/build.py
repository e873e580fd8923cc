"""Build libdkv.so in-tree for sm_100a with nvcc.

    python quantized_kv_cache_dkv_b200/build.py [--force] [-v] [--bounds-check | --trace]

Objects go to quantized_kv_cache_dkv_b200/_build/, the library to
quantized_kv_cache_dkv_b200/libdkv.so.  --bounds-check builds the
bounds-checking variant instead (DKV_BOUNDS_CHECK: kernels check their index
arithmetic and copy ranges, record DKV_FLAG_BOUNDS and skip the access) into
_build_bc/ and libdkv_bc.so; --trace the pipeline-trace variant (DKV_TRACE:
the tcgen05 kernels stamp the clock at each hand-off of CTA 0, read by
pipeline_trace.py) into _build_trace/ and libdkv_trace.so.  A source is
recompiled when it or any header is newer than its object.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdkv.so")
BUILD_BC = os.path.join(HERE, "_build_bc")
LIB_BC = os.path.join(HERE, "libdkv_bc.so")
BUILD_TRACE = os.path.join(HERE, "_build_trace")
LIB_TRACE = os.path.join(HERE, "libdkv_trace.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
          "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
# the quantizer's fp32 steps must not be contracted into fused multiply-adds
PER_FILE = {"commit.cu": ["-fmad=false"]}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers_mtime() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def _compile(src: str, obj: str, verbose: bool, extra=()) -> None:
    cmd = [nvcc(), *ARCH, *COMMON, *PER_FILE.get(os.path.basename(src), []), *extra, "-c", src,
           "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or r.returncode:
        sys.stdout.write(r.stdout)
        sys.stderr.write(r.stderr)
    if r.returncode:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False,
          trace: bool = False) -> str:
    if bounds_check:
        build_dir, lib, extra = BUILD_BC, LIB_BC, ["-DDKV_BOUNDS_CHECK"]
    elif trace:
        build_dir, lib, extra = BUILD_TRACE, LIB_TRACE, ["-DDKV_TRACE"]
    else:
        build_dir, lib, extra = BUILD, LIB, []
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_t = _headers_mtime()
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(build_dir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_t):
            jobs.append((s, o))
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            for f in [ex.submit(_compile, s, o, verbose, extra) for s, o in jobs]:
                f.result()
    if jobs or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-lcuda"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"link of {os.path.basename(lib)} failed")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                bounds_check="--bounds-check" in sys.argv, trace="--trace" in sys.argv))
