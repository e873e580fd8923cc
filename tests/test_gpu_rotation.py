"""Rotated V (K-RPBH before per-token V quantization, output rotated back) on
both attention kernels against the oracle, at 2, 3 and 4 bits: codes, scales
and zero points bit for bit (the rotation runs in the same fp32 order on both
sides), attention within the output bound."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, compare_exports, default_cap, default_P,
                      dev_bf16, gpu_config, host_bits)
from oracle import OracleCache, krpbh
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _caches(dkv, w, cap, P, b, seed=0):
    perm, mix = synth.krpbh_params(seed, b)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    dkv.dkv_cache_set_v_rotation(cache, perm, mix, b)
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group, P,
                     cap, v_rotation=(perm, mix, b))
    return cache, oc


def _attend(dkv, cache, Q, Ka, Va, w, noalloc=False):
    import torch
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    f = dkv.dkv_block_attention_noalloc if noalloc else dkv.dkv_block_attention
    f(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    torch.cuda.synchronize()
    return host_bits(out)


CASES = [("mha8b", 16, {}), ("mha8b", 128, {}), ("batch32", 32, {}), ("gqa7b", 64, {}),
         ("tiny", 32, {"v_group": 128}), ("tiny", 16, {"v_bits": 2, "v_group": 64}),
         ("longprompt", 32, {"L": 320}),
         # 3-bit V: a lane's 12 code bits straddle words in lanes 2 and 5 of each 8
         ("batch32", 64, {"k_bits": 3, "v_bits": 3, "v_group": 32}),
         ("tiny", 128, {"v_bits": 3, "v_group": 128}), ("mha8b", 32, {"v_bits": 3, "v_group": 64})]


@pytest.mark.parametrize("name,b,over", CASES)
def test_rotated_v_commit_and_attention(dkv, name, b, over):
    w = SHRUNK[name].with_(**over)
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache, oc = _caches(dkv, w, cap, P, b)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    assert dkv.dkv_cache_status(cache) == oc.flags
    for step in (0, 1):
        Q = synth.queries_bits(w, step)
        Ka, Va = synth.active_block_bits(w, step)
        ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
        for kernel in (1, 2):
            dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
            for sp in (0, 1, 2):
                dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, sp)
                got = _attend(dkv, cache, Q, Ka, Va, w)
                assert_close(got, ref, f"{name} b={b} kernel {kernel} splits {sp}")
                k, s, n = dkv.dkv_last_attention_plan(cache)
                assert k == kernel and n == 3  # rotation + attention + combine


def test_rotated_v_empty_cache_and_noalloc(dkv):
    """len = 0: one split, still through the combine (inverse rotation); the
    no-allocation entry point gives the same bytes."""
    w = SHRUNK["batch32"]
    cap = default_cap(w, 4)
    cache, oc = _caches(dkv, w, cap, 16, 32, seed=3)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
    got = _attend(dkv, cache, Q, Ka, Va, w)
    assert_close(got, ref, "empty cache")
    assert np.array_equal(_attend(dkv, cache, Q, Ka, Va, w, noalloc=True), got)
    commit_both(dkv, cache, oc, w, range(3))
    ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
    got = _attend(dkv, cache, Q, Ka, Va, w)
    assert_close(got, ref, "three blocks")
    assert np.array_equal(_attend(dkv, cache, Q, Ka, Va, w, noalloc=True), got)


def test_rotated_v_truncate_and_recommit(dkv):
    w = SHRUNK["mha8b"].with_(L=256)
    cap = default_cap(w, 12)
    P = default_P(w, cap)
    cache, oc = _caches(dkv, w, cap, P, 64, seed=5)
    commit_both(dkv, cache, oc, w, range(8))
    dkv.dkv_cache_truncate(cache, 96)
    oc.truncate(96)
    commit_both(dkv, cache, oc, w, range(20, 24))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    Q = synth.queries_bits(w, 2)
    Ka, Va = synth.active_block_bits(w, 2)
    assert_close(_attend(dkv, cache, Q, Ka, Va, w), oc.block_attention(Q, Ka, Va, w.softmax_scale))


@pytest.mark.parametrize("vb,GV", [(4, 32), (2, 64)])
def test_rotated_v_grid_exact_rows(dkv, vb, GV):
    """Rows whose rotation lands exactly on the quantization grid (exact zeros
    included): codes bit for bit, and the output equal to dense attention over
    the unrotated V within the output bound."""
    b, d, blk = 16, 128, 32
    r = np.random.default_rng(40 + vb)
    perm = r.permutation(d).astype(np.int32)
    mix = np.roll(np.eye(d // b, dtype=np.float32), 1, axis=1)
    levels = 2 ** vb - 1

    def rows(n):
        wr = np.zeros((n, d))
        for t in range(n):
            s = 2.0 ** int(r.integers(-3, 2))
            for g in range(d // GV):
                vals = r.integers(0, levels + 1, GV // b).astype(np.float64)
                vals[0] = levels
                wr[t, g * GV:(g + 1) * GV:b] = vals * s
        return krpbh.f32_to_bf16_bits(krpbh.unrotate_f64(wr, perm, mix, b).astype(np.float32))

    w = SHRUNK["tiny"].with_(k_bits=16, v_bits=vb, v_group=GV, Hq=4, Hkv=2)
    cap = 6 * blk
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 0))
    dkv.dkv_cache_set_v_rotation(cache, perm, mix, b)
    oc = OracleCache(w.B, w.Hq, w.Hkv, d, blk, 16, vb, w.k_group, GV, 0, cap,
                     v_rotation=(perm, mix, b))
    import torch
    for i in range(5):
        K = synth.f32_to_bf16_bits(r.standard_normal((1, 2, blk, d)).astype(np.float32))
        V = np.stack([rows(blk), rows(blk)])[None]
        dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), None)
        oc.commit(K, V)
    torch.cuda.synchronize()
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    Q = synth.queries_bits(w, 0)
    Ka = synth.f32_to_bf16_bits(r.standard_normal((1, 2, blk, d)).astype(np.float32))
    Va = np.stack([rows(blk), rows(blk)])[None]
    ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
    for kernel in (1, 2):
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
        assert_close(_attend(dkv, cache, Q, Ka, Va, w), ref, f"grid kernel {kernel}")


def test_rotation_rejections_and_switch_off(dkv):
    w = SHRUNK["tiny"]
    cap = default_cap(w, 4)
    perm, mix = synth.krpbh_params(0, 32)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 16))

    def rc(p, m, b):
        with pytest.raises(dkv.DkvError) as e:
            dkv.dkv_cache_set_v_rotation(cache, p, m, b)
        return e.value.code

    bad = perm.copy()
    bad[3] = bad[4]
    assert rc(bad, mix, 32) == dkv.DKV_ERR_INVALID_ARG
    assert rc(perm, mix * 1.01, 32) == dkv.DKV_ERR_INVALID_ARG
    nan = mix.copy()
    nan[0, 0] = np.nan
    assert rc(perm, nan, 32) == dkv.DKV_ERR_INVALID_ARG
    assert rc(perm, np.eye(16, dtype=np.float32), 8) == dkv.DKV_ERR_UNSUPPORTED
    # switched on, then off again: the plain path (two launches at most)
    dkv.dkv_cache_set_v_rotation(cache, perm, mix, 32)
    dkv.dkv_cache_set_v_rotation(cache, None, None, 0)
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group, 16,
                     cap)
    commit_both(dkv, cache, oc, w, range(2))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    # after the first commit the rotation can no longer change
    assert rc(perm, mix, 32) == dkv.DKV_ERR_INVALID_ARG
    # bf16 V and a sink: not supported
    c16 = dkv.dkv_cache_alloc(gpu_config(dkv, w.with_(v_bits=16), cap, 16))
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_cache_set_v_rotation(c16, perm, mix, 32)
    assert e.value.code == dkv.DKV_ERR_UNSUPPORTED
    cs = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 16, sink=4))
    with pytest.raises(dkv.DkvError) as e:
        dkv.dkv_cache_set_v_rotation(cs, perm, mix, 32)
    assert e.value.code == dkv.DKV_ERR_UNSUPPORTED
