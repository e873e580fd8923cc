"""Attention sink (the first sink_tokens positions kept in full precision:
K protected, V in bf16) on both attention kernels against the oracle."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, compare_exports, default_cap, dev_bf16,
                      gpu_config, host_bits, oracle_cache)
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _attend(dkv, cache, oc, w, step):
    import torch
    Q = synth.queries_bits(w, step)
    Ka, Va = synth.active_block_bits(w, step)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    torch.cuda.synchronize()
    assert_close(host_bits(out), oc.block_attention(Q, Ka, Va, w.softmax_scale))


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("name,sink", [("batch32", 1), ("batch32", 40), ("mha8b", 4),
                                       ("mha8b", 160), ("gqa7b", 64)])
def test_sink_commit_and_attention(dkv, kernel, name, sink):
    w = SHRUNK[name]
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = 64 + sink
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P, sink))
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
    oc = oracle_cache(w, cap, P, sink=sink)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    exp = dkv.dkv_cache_export(cache)
    assert "v_sink" in exp
    compare_exports(exp, oc.snapshot())
    assert dkv.dkv_cache_status(cache) == oc.flags
    for sp in (0, 2):
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, sp)
        _attend(dkv, cache, oc, w, 1)


def test_sink_truncate_below_and_recommit(dkv):
    w = SHRUNK["batch32"].with_(k_group=32)
    cap = default_cap(w, 12)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 96, 48))
    oc = oracle_cache(w, cap, 96, sink=48)
    commit_both(dkv, cache, oc, w, range(5))
    dkv.dkv_cache_truncate(cache, 32)
    oc.truncate(32)
    commit_both(dkv, cache, oc, w, (7, 8))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    _attend(dkv, cache, oc, w, 2)


def test_sink_config_limits(dkv):
    w = SHRUNK["tiny"]
    for bad in (-1, 257):
        with pytest.raises(dkv.DkvError):
            dkv.dkv_cache_alloc(gpu_config(dkv, w, 512, 8, bad))
