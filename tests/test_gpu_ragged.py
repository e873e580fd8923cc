"""Per-sequence committed lengths (sequences of one batch commit their blocks
at different steps; SoloQ's block-diffusion paragraph quantizes each block
when it is committed) through the C-ABI against the oracle's ragged cache:
every sequence's export bit for bit at its own length, attention of every
sequence over its own tokens within the output bound, on both attention
kernels and several split counts (splits past a shorter sequence's end are
empty), through a per-sequence roll-back and recommit, and in the dual-cache
call."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, compare_exports, default_P, dev_bf16, dev_words,
                      gpu_config, host_bits)
from oracle import OracleRaggedCache
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _schedule(B, n_steps):
    """Which sequences commit at each step: sequence b skips every (b + 2)-th
    step, so the lengths drift apart (and sequence 0 commits least)."""
    return [[b for b in range(B) if (i + 1) % (b + 2) != 0 or b == B - 1] for i in range(n_steps)]


def _build(dkv, w, n_steps, cap):
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = OracleRaggedCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group,
                           w.v_group, P, cap)
    for i, seqs in enumerate(_schedule(w.B, n_steps)):
        _commit(dkv, cache, oc, w, i, seqs)
    return cache, oc


def _commit(dkv, cache, oc, w, i, seqs):
    K, V, M = synth.block_inputs(w, i)
    dkv.dkv_commit_block_seqs(cache, dev_bf16(K), dev_bf16(V), dev_words(M), seqs)
    oc.commit(K, V, M, seqs)


def _check_state(dkv, cache, oc):
    assert dkv.dkv_cache_seq_lens(cache) == oc.lens
    assert dkv.dkv_cache_len(cache) == max(oc.lens)
    for b in range(oc.B):
        compare_exports(dkv.dkv_cache_export_seq(cache, b), oc.seqs[b].snapshot())


def _attend(dkv, cache, w, step, kernel, splits):
    import torch
    Q = synth.queries_bits(w, step)
    Ka, Va = synth.active_block_bits(w, step)
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, splits)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    torch.cuda.synchronize()
    return host_bits(out), (Q, Ka, Va)


@pytest.mark.parametrize("name", ["batch32", "gqa7b", "mha8b", "tiny"])
def test_ragged_commit_and_attention(dkv, name):
    w = SHRUNK[name].with_(B=3, prot_frac=0.03)
    n_steps = max(12, min(w.L // w.blk, 20))
    unit = max(w.k_group, w.blk)
    cap = ((n_steps + 4) * w.blk + unit - 1) // unit * unit + unit
    cache, oc = _build(dkv, w, n_steps, cap)
    assert len(set(oc.lens)) > 1
    _check_state(dkv, cache, oc)
    assert dkv.dkv_cache_status(cache) == 0
    with pytest.raises(dkv.DkvError):
        dkv.dkv_cache_export(cache)  # lengths differ: per-sequence export only
    for kernel in (1, 2):
        for splits in (0, 1, 4):
            got, (Q, Ka, Va) = _attend(dkv, cache, w, kernel, kernel, splits)
            ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
            assert_close(got, ref, f"{name} kernel {kernel} splits {splits}")
    # one sequence rolled back to a group boundary, then new commits to a subset
    b = 1
    new_len = (oc.lens[b] // (2 * unit)) * unit
    dkv.dkv_cache_truncate_seq(cache, b, new_len)
    oc.truncate(b, new_len)
    for i in range(n_steps, n_steps + 3):
        _commit(dkv, cache, oc, w, i, [b, 2] if i % 2 else [b])
    _check_state(dkv, cache, oc)
    got, (Q, Ka, Va) = _attend(dkv, cache, w, 7, 2, 0)
    assert_close(got, oc.block_attention(Q, Ka, Va, w.softmax_scale), f"{name} after roll-back")
    assert dkv.dkv_cache_status(cache) == 0


def test_ragged_argument_checks_and_uniform_equivalence(dkv):
    """A commit listing every sequence equals dkv_commit_block; an empty list
    changes nothing; bad lists are refused without a change."""
    w = SHRUNK["batch32"].with_(B=2)
    cap = 512
    P = default_P(w, cap)
    a = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    c = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    for i in range(5):
        K, V, M = synth.block_inputs(w, i)
        dkv.dkv_commit_block(a, dev_bf16(K), dev_bf16(V), dev_words(M))
        dkv.dkv_commit_block_seqs(c, dev_bf16(K), dev_bf16(V), dev_words(M), [1, 0])
        dkv.dkv_commit_block_seqs(c, dev_bf16(K), dev_bf16(V), dev_words(M), [])
    ea, ec = dkv.dkv_cache_export(a), dkv.dkv_cache_export(c)
    for key, arr in ea.items():
        if isinstance(arr, np.ndarray):
            assert np.array_equal(arr.view(np.uint8), ec[key].view(np.uint8)), key
    K, V, M = synth.block_inputs(w, 9)
    for bad in ([0, 0], [2], [-1]):
        with pytest.raises(dkv.DkvError) as ei:
            dkv.dkv_commit_block_seqs(c, dev_bf16(K), dev_bf16(V), dev_words(M), bad)
        assert ei.value.code == dkv.DKV_ERR_INVALID_ARG
    assert dkv.dkv_cache_seq_lens(c) == [160, 160]
    with pytest.raises(dkv.DkvError):
        dkv.dkv_cache_truncate_seq(c, 0, 32)   # not a multiple of the K group (64)
    dkv.dkv_cache_truncate_seq(c, 0, 64)
    assert dkv.dkv_cache_seq_lens(c) == [64, 160]
    with pytest.raises(dkv.DkvError):
        dkv.dkv_cache_truncate(c, 128)         # beyond sequence 0's length
    dkv.dkv_cache_truncate(c, 64)
    assert dkv.dkv_cache_seq_lens(c) == [64, 64]


def test_ragged_dual_cache(dkv):
    """Both caches ragged: every sequence attends over its own prefix, the
    active block and its own suffix."""
    import torch
    w = SHRUNK["batch32"].with_(B=3, prot_frac=0.03)
    cap = 1024
    pre, opre = _build(dkv, w, 14, cap)
    P = default_P(w, cap)
    suf = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    osuf = OracleRaggedCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group,
                             w.v_group, P, cap)
    for i, seqs in enumerate(_schedule(w.B, 6)):
        _commit(dkv, suf, osuf, w, 500 + i, seqs[::-1])
    Q = synth.queries_bits(w, 3)
    Ka, Va = synth.active_block_bits(w, 3)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    for kernel in (1, 2):
        for c in (pre, suf):
            dkv.dkv_cache_set_option(c, dkv.DKV_OPT_ATTN_KERNEL, kernel)
        dkv.dkv_block_attention_dual(pre, suf, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                     w.softmax_scale, out)
        torch.cuda.synchronize()
        ref = np.concatenate([opre.seqs[b].block_attention_dual(
            osuf.seqs[b], Q[b:b + 1], Ka[b:b + 1], Va[b:b + 1], w.softmax_scale)
            for b in range(w.B)])
        assert_close(host_bits(out), ref, f"dual kernel {kernel}")
