"""The bounded waits of the tcgen05 attention kernel, run out on purpose, in
its own process on the library named by DKV_LIB (the bounds-checking build,
libdkv_bc.so, the only build with the DKV_OPT_TEST_STALL hook).

    DKV_LIB=.../libdkv_bc.so python tests/timeout_check.py

The hook makes the kernel's loader withhold the copies of one tile, so the
producers' waits on that pipeline stage run out (2 ms limit while the hook is
set).  Nothing faults, traps or spins without a limit: every wait in the
kernel is bounded, and on expiry every role leaves its loop, the CTA waits for
its own copies and MMAs in flight and frees its tensor memory.  Checked: the
call returns, the status reports DKV_FLAG_TIMEOUT, and the next calls -- on
the same handle with the hook off, and on a fresh handle -- match the
oracle with a clean status.  Prints OK and exits 0, else raises."""
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import synth  # noqa: E402
from gpu_util import (assert_close, commit_both, default_P, default_cap, dev_bf16,  # noqa: E402
                      gpu_config, host_bits, oracle_cache)


def main():
    import quantized_kv_cache_dkv_b200 as dkv
    print("library:", os.path.basename(dkv.LIB_PATH), flush=True)
    # 128-row query groups (4 query heads x 32-token blocks) and 32-row groups
    # (one query head per kv-head) on the row-block kernel; 32-row groups with
    # the tokens on the TMEM lanes
    check(dkv, synth.WORKLOADS["tiny"].with_(B=2, Hq=8, Hkv=2, L=1024, prot_frac=0.02), 2)
    check(dkv, synth.WORKLOADS["tiny"].with_(B=2, Hq=2, Hkv=2, L=1024, prot_frac=0.02), 2)
    check(dkv, synth.WORKLOADS["tiny"].with_(B=2, Hq=2, Hkv=2, L=1024, prot_frac=0.02), 3)
    print("OK timeout path", flush=True)


def check(dkv, w, kernel):
    import torch
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)

    def built():
        cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
        return cache

    cache = built()
    oc = oracle_cache(w, cap, P)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    assert dkv.dkv_cache_status(cache) == 0
    Qh = synth.queries_bits(w, 0)
    Kah, Vah = synth.active_block_bits(w, 0)
    Q, Ka, Va = dev_bf16(Qh), dev_bf16(Kah), dev_bf16(Vah)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    ref = oc.block_attention(Qh, Kah, Vah, w.softmax_scale)

    # (splits, stalled tile): the first tile of every CTA; a later tile of a
    # single-split CTA, after some tiles went through the whole pipeline
    for splits, tile in ((0, 0), (1, 3)):
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, splits)
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_TEST_STALL, tile)
        t0 = time.time()
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, out)
        torch.cuda.synchronize()
        dt = time.time() - t0
        flags = dkv.dkv_cache_status(cache)
        print(f"stall tile {tile}, splits {splits}: flags {flags:#x}, {dt * 1e3:.1f} ms",
              flush=True)
        assert flags & dkv.DKV_FLAG_TIMEOUT, flags
        assert not flags & dkv.DKV_FLAG_BOUNDS, flags
        assert dt < 5.0, dt
        # the hook off: the same handle attends correctly again
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_TEST_STALL, -1)
        out.zero_()
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, out)
        torch.cuda.synchronize()
        assert_close(host_bits(out), ref, f"after the stall of tile {tile}")
        assert dkv.dkv_cache_status(cache) == 0

    # a fresh handle after the timeouts
    cache2 = built()
    commit_both(dkv, cache2, None, w, range(n_blocks))
    out.zero_()
    dkv.dkv_block_attention(cache2, Q, Ka, Va, w.softmax_scale, out)
    torch.cuda.synchronize()
    assert_close(host_bits(out), ref, "fresh handle")
    assert dkv.dkv_cache_status(cache2) == 0
    dkv.dkv_cache_free(cache2)
    dkv.dkv_cache_free(cache)


if __name__ == "__main__":
    main()
