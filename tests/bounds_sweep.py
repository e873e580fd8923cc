"""Seeded sweep of small random cache shapes against the oracle, run in its
own process on the library named by DKV_LIB (the bounds-checking build,
libdkv_bc.so, whose kernels check every copy range and index they use and
record DKV_FLAG_BOUNDS instead of making an out-of-range access).

    DKV_LIB=.../libdkv_bc.so python tests/bounds_sweep.py [n_cases] [seed]

Each case draws bit widths, group sizes, block, heads, fill level (empty up
to a full cache), side-table size (some too small, so the capacity path
runs), sink length, a roll-back and recommit (bit widths 2, 3, 4 and 16);
commits through the library and
the oracle, compares the exported state bit for bit and the status flags
exactly (the oracle never sets DKV_FLAG_BOUNDS), and the block attention of
both attention kernels, with and without splits, within the output bound.
Prints one line per case and exits non-zero on the first mismatch."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import synth  # noqa: E402
from gpu_util import (assert_close, commit_both, compare_exports, dev_bf16,  # noqa: E402
                      gpu_config, host_bits, oracle_cache)


def draw_case(r: np.random.Generator, i: int):
    kb, vb = (int(x) for x in r.choice([2, 3, 4, 16], 2))
    gk, gv = (int(x) for x in r.choice([32, 64, 128], 2))
    blk = int(r.choice([32, 64, 128]))
    g = int(r.choice([g for g in (1, 2, 4, 8) if g * blk <= 256]))
    Hkv = int(r.integers(1, 3))
    B = int(r.integers(1, 3))
    unit = max(blk, gk)
    n_blocks = int(r.integers(0, max(2, 640 // blk)))
    full = r.random() < 0.3
    cap = -(-max(n_blocks * blk, 1) // unit) * unit
    if not full:
        cap += unit * int(r.integers(1, 3))
    n_blocks = min(n_blocks, cap // blk)
    prot_frac = float(r.choice([0.0, 0.01, 0.05]))
    P = int(r.choice([0, 4, 16, int(prot_frac * cap) * 2 + 16]))
    sink = 0
    if r.random() < 0.35:
        sink = int(min(r.integers(1, 257), cap))
        P += sink
    w = synth.WORKLOADS["tiny"].with_(B=B, Hq=g * Hkv, Hkv=Hkv, blk=blk, k_bits=kb, v_bits=vb,
                                      k_group=gk, v_group=gv, prot_frac=prot_frac,
                                      L=n_blocks * blk, seed=1000 + i)
    trunc = None
    if n_blocks >= 2 and r.random() < 0.4:
        trunc = int(r.integers(0, n_blocks * blk // unit + 1)) * unit
    return w, n_blocks, cap, P, sink, trunc


def run_case(dkv, torch, w, n_blocks, cap, P, sink, trunc):
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P, sink))
    oc = oracle_cache(w, cap, P, sink=sink)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    if trunc is not None:
        dkv.dkv_cache_truncate(cache, trunc)
        oc.truncate(trunc)
        more = min(2, (cap - trunc) // w.blk)
        commit_both(dkv, cache, oc, w, range(n_blocks, n_blocks + more))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    st = dkv.dkv_cache_status(cache)
    assert st & dkv.DKV_FLAG_BOUNDS == 0, f"bounds flag after commit: {st:#x}"
    assert st == oc.flags, (st, oc.flags)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
    for kernel in (1, 2):
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
        for sp in (0, 2):
            dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, sp)
            out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
            dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                    w.softmax_scale, out)
            torch.cuda.synchronize()
            st = dkv.dkv_cache_status(cache)
            assert st & dkv.DKV_FLAG_BOUNDS == 0, f"bounds flag, kernel {kernel}: {st:#x}"
            assert_close(host_bits(out), ref, f"kernel {kernel} splits {sp}")
    dkv.dkv_cache_free(cache)


def main(n_cases: int, seed: int) -> int:
    import torch
    import quantized_kv_cache_dkv_b200 as dkv
    print("library:", os.path.basename(dkv.LIB_PATH), flush=True)
    r = np.random.default_rng(seed)
    for i in range(n_cases):
        w, n_blocks, cap, P, sink, trunc = draw_case(r, i)
        desc = (f"case {i}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} blk={w.blk} k{w.k_bits}/g{w.k_group} "
                f"v{w.v_bits}/g{w.v_group} blocks={n_blocks} cap={cap} P={P} sink={sink} "
                f"trunc={trunc}")
        print(desc, flush=True)
        run_case(dkv, torch, w, n_blocks, cap, P, sink, trunc)
    print(f"OK {n_cases} cases", flush=True)
    return 0


if __name__ == "__main__":
    a = sys.argv[1:]
    sys.exit(main(int(a[0]) if a else 24, int(a[1]) if len(a) > 1 else 7))
