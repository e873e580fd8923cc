"""dkv_block_attention_noalloc -- the attention entry point for callers that
cannot call cudaMalloc (code running under CUDA stream capture, plugins whose
host application owns all device memory) -- against dkv_block_attention on the
same cache and inputs, on two calls in a row, through the C-ABI.  Collected
last, and self-contained so it also passes alone in a fresh process."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, default_P, default_cap, dev_bf16, gpu_config,
                      host_bits, output_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


CASES = {
    # 128-row query groups (tcgen05 kernel), several splits
    "groups128": synth.WORKLOADS["batch32"].with_(B=2, Hq=8, Hkv=2, L=1216),
    # 32-row query groups (mma.sync kernel), several splits
    "groups32": synth.WORKLOADS["mha8b"].with_(Hq=8, Hkv=8, L=1024),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_block_attention(dkv, name):
    import torch
    w = CASES[name]
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, default_P(w, cap)))
    commit_both(dkv, cache, None, w, range(n_blocks))
    for step in (0, 1):            # two calls in a row, different inputs
        Q = dev_bf16(synth.queries_bits(w, step))
        Ka, Va = [dev_bf16(x) for x in synth.active_block_bits(w, step)]
        ref = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        got = torch.empty_like(ref)
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, ref)
        _, splits, _ = dkv.dkv_last_attention_plan(cache)
        dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, got)
        torch.cuda.synchronize()
        assert splits > 1              # the scratch buffer is in use
        r = synth.bf16_bits_to_f32(host_bits(ref)).astype(np.float64)
        g = host_bits(got)
        assert_close(g, r, f"{name} call {step}")
        assert np.all(np.abs(synth.bf16_bits_to_f32(g) - r) <= output_bound(r))
    assert dkv.dkv_cache_status(cache) == 0


def test_noalloc_rejects_scratch_beyond_buffer(dkv):
    import torch
    w = CASES["groups128"].with_(B=8, Hkv=8, Hq=32, L=2048)
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, default_P(w, cap)))
    commit_both(dkv, cache, None, w, range(n_blocks))
    # 64 units x 8 splits x 128 rows x 520 bytes = 34 MB > 16 MiB
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, 8)
    Q = dev_bf16(synth.queries_bits(w, 0))
    Ka, Va = [dev_bf16(x) for x in synth.active_block_bits(w, 0)]
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dkv.DkvError) as ei:
        dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, out)
    assert ei.value.code == dkv.DKV_ERR_UNSUPPORTED
    assert "scratch" in str(ei.value)
    # one split needs no scratch at all
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, 1)
    dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, out)
    torch.cuda.synchronize()
