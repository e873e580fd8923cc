"""Pipeline trace of the tcgen05 attention kernels: clock64 stamps of CTA 0
(unit 0, first split) at every hand-off of its tile pipeline, from the
trace build of the library (libdkv_trace.so, DKV_TRACE).

    python quantized_kv_cache_dkv_b200/build.py --trace
    python quantized_kv_cache_dkv_b200/pipeline_trace.py [workload] [kernel] [B] [L] [splits]

One attention call on a cache of the workload's shape (seeded synthetic
inputs), then one line per tile with the cycles since the CTA started of:
the loader issuing the tile's copies (load), the K producer starting and
ending the tile (k_beg, k_end), the V producer getting its buffer, starting
and ending (v_wt, v_beg, v_end), the QK MMAs' issue starting and ending
(qk, qk_end), the softmax
holding the scores (sm_beg), after its first pass / vote (sm_mid), P
written (p_out), the PV MMAs' issue starting and ending (pv, pv_end); and
the steady-state period (pv
issue to pv issue over the last two thirds of the tiles).  The stamps cost
a few instructions in CTA 0 only; times of a trace-build call are not
benchmark figures."""
import ctypes
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
os.environ["DKV_LIB"] = os.path.join(HERE, "libdkv_trace.so")
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

EVENTS = [(0, "load"), (1, "k_beg"), (2, "k_end"), (11, "v_wt"), (3, "v_beg"), (4, "v_end"),
          (5, "qk"), (14, "qk_end"), (6, "sm_beg"), (12, "sm_mid"), (7, "p_out"), (8, "pv"),
          (13, "pv_end")]


def trace(workload="batch32", kernel=2, B=0, L=0, splits=1):
    import torch
    import synth
    import quantized_kv_cache_dkv_b200 as dkv
    lib = dkv._lib
    lib.dkv_trace_read.argtypes = [ctypes.c_void_p]
    w = synth.WORKLOADS[workload]
    if B:
        w = w.with_(B=B)
    if L:
        w = w.with_(L=L)

    def dev(bits, dt=torch.bfloat16):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(dt)

    unit = max(w.k_group, w.blk)
    cap = ((w.L + 2 * w.blk + unit - 1) // unit) * unit
    P = int(round(w.prot_frac * cap)) * 2 + 64
    cache = dkv.dkv_cache_alloc(dkv.make_config(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits,
                                                w.k_group, w.v_group, P, cap))
    for i in range(w.L // w.blk):
        K, V, M = synth.block_inputs(w, i)
        dkv.dkv_commit_block(cache, dev(K), dev(V),
                             torch.from_numpy(np.ascontiguousarray(M).view(np.int32)).cuda())
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, splits)
    Q = dev(synth.queries_bits(w, 0))
    Ka, Va = [dev(x) for x in synth.active_block_bits(w, 0)]
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, out)
    torch.cuda.synchronize()
    lib.dkv_trace_clear()
    dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, out)
    torch.cuda.synchronize()
    tr = np.zeros((16, 64), np.uint64)
    lib.dkv_trace_read(tr.ctypes.data)
    dkv.dkv_cache_free(cache)
    t0 = int(tr[9, 0])
    nt = int((tr[5] > 0).sum())
    a_, b_ = nt // 3, nt - 1
    period = (int(tr[8, b_]) - int(tr[8, a_])) / max(b_ - a_, 1)
    print(f"{workload} B={w.B} L={w.L} kernel {kernel} splits {splits}: CTA 0 ran "
          f"{int(tr[10, 0]) - t0} cycles, {nt} tiles, steady-state period {period:.0f} cycles/tile")
    print("tile " + " ".join(f"{n:>7s}" for _, n in EVENTS))
    for j in range(nt):
        print(f"{j:4d} " + " ".join(f"{int(tr[e, j]) - t0 if tr[e, j] else -1:7d}" for e, _ in EVENTS))
    return period


if __name__ == "__main__":
    a = sys.argv[1:]
    trace(a[0] if a else "batch32", int(a[1]) if len(a) > 1 else 2, int(a[2]) if len(a) > 2 else 0,
          int(a[3]) if len(a) > 3 else 0, int(a[4]) if len(a) > 4 else 1)
