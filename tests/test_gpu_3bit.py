"""3-bit K and V (SoloQ summary: KV-only results near 3 bits, and the KV2 sink
ablation): commit codes, scales and zero points bit for bit against the
oracle -- 32 codes fill three words, codes 10 and 21 straddle two -- and
attention within the output bound on every attention kernel: mma.sync,
tcgen05 with query-row blocks, and tcgen05 with the tokens on the TMEM lanes
for 32-row query groups.  The tcgen05 producers extract the 32 codes of three
words one by one and keep the natural token / channel order."""
import pytest

import synth
from gpu_util import (assert_close, commit_both, compare_exports, default_P, default_cap,
                      dev_bf16, gpu_config, host_bits, oracle_cache)
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


CASES = [
    ("batch32", dict(k_bits=3, v_bits=3, k_group=64, v_group=64), 0),
    ("gqa7b", dict(k_bits=3, v_bits=3, k_group=32, v_group=32), 0),
    ("mha8b", dict(k_bits=3, v_bits=4, k_group=128, v_group=32), 0),
    ("tiny", dict(k_bits=2, v_bits=3, k_group=32, v_group=128, prot_frac=0.05), 0),
    ("longprompt", dict(k_bits=3, v_bits=3, L=640), 0),
    ("batch32", dict(k_bits=3, v_bits=3, k_group=32, v_group=32), 40),   # with a sink
]


@pytest.mark.parametrize("name,over,sink", CASES)
def test_three_bit_commit_and_attention(dkv, name, over, sink):
    import torch
    w = SHRUNK[name].with_(**over)
    n_blocks = w.L // w.blk + 1          # an odd count: a tail with k_group 64 / 128
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap) + sink
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P, sink))
    oc = oracle_cache(w, cap, P, sink=sink)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    assert dkv.dkv_cache_status(cache) == oc.flags
    rows = (w.Hq // w.Hkv) * w.blk
    kernels = (1, 2, 3) if rows == 32 else (1, 2)
    for step in (0, 1):
        Q = synth.queries_bits(w, step)
        Ka, Va = synth.active_block_bits(w, step)
        ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
        for kernel in kernels:
            dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
            for sp in (0, 1, 3):
                dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, sp)
                out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
                dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                        w.softmax_scale, out)
                torch.cuda.synchronize()
                assert_close(host_bits(out), ref,
                             f"{name} {over} step {step} kernel {kernel} splits {sp}")
                assert dkv.dkv_last_attention_plan(cache)[0] == kernel
    assert dkv.dkv_cache_status(cache) == oc.flags
    # the default plan of a 3-bit cache is the row-block tcgen05 kernel
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, 0)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    torch.cuda.synchronize()
    assert dkv.dkv_last_attention_plan(cache)[0] == 2
