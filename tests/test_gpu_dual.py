"""Dual-cache attention (prefix cache + active block + suffix cache) on both
attention kernels against the oracle."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, default_cap, default_P, dev_bf16, gpu_config,
                      host_bits, oracle_cache)
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _out(w):
    import torch
    return torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")


def _dual(dkv, pre, suf, w, Q, Ka, Va):
    import torch
    out = _out(w)
    dkv.dkv_block_attention_dual(pre, suf, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                 w.softmax_scale, out)
    torch.cuda.synchronize()
    return host_bits(out)


def _pair(dkv, w, ws, n_pre, n_suf):
    """Prefix cache of w with n_pre blocks, suffix cache of ws (same heads and
    block, its own bits and groups) with n_suf blocks, and their oracles."""
    cap = default_cap(w, n_pre + 1)
    caps = default_cap(ws, n_suf + 1)
    P, Ps = default_P(w, cap), default_P(ws, caps)
    pre = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    suf = dkv.dkv_cache_alloc(gpu_config(dkv, ws, caps, Ps))
    op, osf = oracle_cache(w, cap, P), oracle_cache(ws, caps, Ps)
    commit_both(dkv, pre, op, w, range(n_pre))
    commit_both(dkv, suf, osf, ws, range(100, 100 + n_suf))
    return pre, suf, op, osf


CASES = [("batch32", {}, 6), ("mha8b", {"k_bits": 2, "v_bits": 2, "k_group": 64}, 4),
         ("gqa7b", {"k_bits": 16, "v_bits": 16}, 3), ("longprompt", {"v_group": 128}, 9),
         ("tiny", {}, 1)]


@pytest.mark.parametrize("name,sover,n_suf", CASES)
def test_dual_attention_matches_oracle(dkv, name, sover, n_suf):
    w = SHRUNK[name]
    ws = w.with_(**sover)
    n_pre = min(w.L // w.blk, 12)
    pre, suf, op, osf = _pair(dkv, w, ws, n_pre, n_suf)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    ref = op.block_attention_dual(osf, Q, Ka, Va, w.softmax_scale)
    for k1 in (1, 2):
        for k2 in (1, 2):
            dkv.dkv_cache_set_option(pre, dkv.DKV_OPT_ATTN_KERNEL, k1)
            dkv.dkv_cache_set_option(suf, dkv.DKV_OPT_ATTN_KERNEL, k2)
            for sp1, sp2 in ((0, 0), (1, 1), (2, 3)):
                dkv.dkv_cache_set_option(pre, dkv.DKV_OPT_SPLITS, sp1)
                dkv.dkv_cache_set_option(suf, dkv.DKV_OPT_SPLITS, sp2)
                got = _dual(dkv, pre, suf, w, Q, Ka, Va)
                assert_close(got, ref, f"{name} kernels {k1}/{k2} splits {sp1}/{sp2}")
                assert dkv.dkv_last_attention_plan(pre)[2] == 3
    assert dkv.dkv_cache_status(pre) == op.flags
    assert dkv.dkv_cache_status(suf) == osf.flags


def test_dual_empty_suffix_is_single_call(dkv):
    import torch
    w = SHRUNK["batch32"]
    pre, suf, op, osf = _pair(dkv, w, w, 5, 0)
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    one = _out(w)
    dkv.dkv_block_attention(pre, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, one)
    torch.cuda.synchronize()
    assert np.array_equal(_dual(dkv, pre, suf, w, Q, Ka, Va), host_bits(one))


def test_dual_roles_swap_and_suffix_refresh(dkv):
    """Prefix/suffix roles swap within fp32 rounding; a suffix rebuilt with
    truncate(0) + new commits (the per-block refresh) matches the oracle."""
    from gpu_util import bf16_to_f64
    w = SHRUNK["gqa7b"].with_(L=256)
    a, b, oa, ob = _pair(dkv, w, w, 8, 8)
    Q = synth.queries_bits(w, 2)
    Ka, Va = synth.active_block_bits(w, 2)
    ab = bf16_to_f64(_dual(dkv, a, b, w, Q, Ka, Va))
    ba = bf16_to_f64(_dual(dkv, b, a, w, Q, Ka, Va))
    assert np.abs(ab - ba).max() <= 2.0 ** -7 * max(1.0, np.abs(ab).max())
    dkv.dkv_cache_truncate(b, 0)
    ob.truncate(0)
    commit_both(dkv, b, ob, w, range(200, 203))
    assert_close(_dual(dkv, a, b, w, Q, Ka, Va), oa.block_attention_dual(ob, Q, Ka, Va,
                                                                          w.softmax_scale))


def test_dual_rejections(dkv):
    w = SHRUNK["tiny"]
    cap = default_cap(w, 4)
    pre = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 16))
    other = dkv.dkv_cache_alloc(gpu_config(dkv, w.with_(Hq=8), cap, 16))
    sink = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 16, sink=4))
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    out = _out(w)
    for suf, code in ((other, dkv.DKV_ERR_INVALID_ARG), (sink, dkv.DKV_ERR_UNSUPPORTED)):
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_block_attention_dual(pre, suf, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                         w.softmax_scale, out)
        assert e.value.code == code
    rot = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 16))
    perm, mix = synth.krpbh_params(0, 32)
    dkv.dkv_cache_set_v_rotation(rot, perm, mix, 32)
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_block_attention_dual(rot, pre, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                     w.softmax_scale, out)
    assert e.value.code == dkv.DKV_ERR_UNSUPPORTED
