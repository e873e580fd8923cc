"""dkv_block_attention_noalloc -- the attention entry point for callers that
cannot call cudaMalloc (code running under CUDA stream capture, where an
allocation is a prohibited call that invalidates the capture, and plugins
whose host application owns all device memory) -- through the C-ABI.

Checked against the oracle and against dkv_block_attention on the same cache
and inputs, on two calls in a row; captured in a CUDA graph and replayed with
new queries and active blocks; on a rotated-V cache.  Collected last, and
self-contained so it also passes alone in a fresh process."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, default_P, default_cap, dev_bf16, gpu_config,
                      host_bits, oracle_cache, output_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


CASES = {
    # 128-row query groups, several splits
    "groups128": synth.WORKLOADS["batch32"].with_(B=2, Hq=8, Hkv=2, L=1216),
    # 32-row query groups (one query head per kv-head), several splits
    "groups32": synth.WORKLOADS["mha8b"].with_(Hq=8, Hkv=8, L=1024),
}


def _built(dkv, w, with_oracle=True):
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = oracle_cache(w, cap, P) if with_oracle else None
    commit_both(dkv, cache, oc, w, range(n_blocks))
    return cache, oc


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_oracle_and_block_attention(dkv, name):
    import torch
    w = CASES[name]
    cache, oc = _built(dkv, w)
    for step in (0, 1):            # two calls in a row, different inputs
        Qh = synth.queries_bits(w, step)
        Kah, Vah = synth.active_block_bits(w, step)
        Q, Ka, Va = dev_bf16(Qh), dev_bf16(Kah), dev_bf16(Vah)
        ref = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        got = torch.empty_like(ref)
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, ref)
        _, splits, _ = dkv.dkv_last_attention_plan(cache)
        dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, got)
        torch.cuda.synchronize()
        assert splits > 1              # the scratch buffer is in use
        exact = oc.block_attention(Qh, Kah, Vah, w.softmax_scale)
        g = host_bits(got)
        assert_close(g, exact, f"{name} call {step} (no-allocation vs oracle)")
        assert_close(host_bits(ref), exact, f"{name} call {step} (with allocation vs oracle)")
        r = synth.bf16_bits_to_f32(host_bits(ref)).astype(np.float64)
        assert np.all(np.abs(synth.bf16_bits_to_f32(g) - r) <= output_bound(r))
    assert dkv.dkv_cache_status(cache) == 0


def test_noalloc_under_graph_capture(dkv):
    """One eager call (looks the buffer up), then the call captured in a CUDA
    graph -- the capture would fail on any allocation -- and replayed twice
    with new queries and active blocks copied into the captured inputs; each
    replay matches dkv_block_attention, and the device's free memory is the
    same before and after the replays."""
    import torch
    w = CASES["groups128"]
    cache, _ = _built(dkv, w, with_oracle=False)
    Q = dev_bf16(synth.queries_bits(w, 0))
    Ka, Va = [dev_bf16(x) for x in synth.active_block_bits(w, 0)]
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    ref = torch.empty_like(out)
    # eager calls of both entry points first (buffer look-up, module loading)
    dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, out)
    dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, ref)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dkv.dkv_block_attention_noalloc(cache, Q, Ka, Va, w.softmax_scale, out)
    g.replay()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for step in (1, 2):
        Q.copy_(dev_bf16(synth.queries_bits(w, step)))
        ka, va = synth.active_block_bits(w, step)
        Ka.copy_(dev_bf16(ka))
        Va.copy_(dev_bf16(va))
        out.zero_()
        g.replay()
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, ref)
        torch.cuda.synchronize()
        r = synth.bf16_bits_to_f32(host_bits(ref)).astype(np.float64)
        o = synth.bf16_bits_to_f32(host_bits(out)).astype(np.float64)
        assert np.all(np.abs(o - r) <= output_bound(r)), f"replay {step}"
        assert not np.array_equal(o, 0 * o)
    assert torch.cuda.mem_get_info()[0] == free0
    del g
    assert dkv.dkv_cache_status(cache) == 0


def test_noalloc_rotated_v(dkv):
    """A rotated-V cache always runs the combine kernel (inverse rotation), so
    the call takes its partials from the static buffer; its output matches
    the oracle."""
    import torch
    from oracle import OracleCache
    w = CASES["groups32"].with_(L=512)
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    perm, mix = synth.krpbh_params(5, 32)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    dkv.dkv_cache_set_v_rotation(cache, perm, mix, 32)
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group, P,
                     cap, v_rotation=(perm, mix, 32))
    commit_both(dkv, cache, oc, w, range(n_blocks))
    for step in (0, 1):
        Qh = synth.queries_bits(w, step)
        Kah, Vah = synth.active_block_bits(w, step)
        out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        dkv.dkv_block_attention_noalloc(cache, dev_bf16(Qh), dev_bf16(Kah), dev_bf16(Vah),
                                        w.softmax_scale, out)
        torch.cuda.synchronize()
        assert_close(host_bits(out), oc.block_attention(Qh, Kah, Vah, w.softmax_scale),
                     f"rotated V call {step}")
    assert dkv.dkv_cache_status(cache) == 0


def test_noalloc_rejects_scratch_beyond_buffer(dkv):
    import torch
    w = CASES["groups128"].with_(B=16, Hkv=8, Hq=32, L=2048)
    cache, _ = _built(dkv, w, with_oracle=False)
    # 17 tiles in splits of 3: 128 units x 6 splits x 128 rows x 264 bytes
    # (fp16 partial + (max, sum)) = 26 MB > 16 MiB
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
