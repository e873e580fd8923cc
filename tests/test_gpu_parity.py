"""CUDA path (through the C-ABI) against the CPU oracle on the same seeded
inputs: packed codes, scales, zero-points, tail and side table bit-exact;
attention within max-abs 1e-2 / mean-abs 1e-3 of the oracle rounded to bf16."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, compare_exports, default_P, default_cap,
                      dev_bf16, dev_words, gpu_config, host_bits, oracle_cache)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _torch():
    import torch
    return torch


# the five workload recipes at sizes the oracle finishes in seconds; every
# case spans several 64- and 128-token tiles and ends on a ragged tile
SHRUNK = {
    "tiny": synth.WORKLOADS["tiny"],
    "mha8b": synth.WORKLOADS["mha8b"].with_(Hq=8, Hkv=8, L=544),
    "gqa7b": synth.WORKLOADS["gqa7b"].with_(B=2, L=608),
    "batch32": synth.WORKLOADS["batch32"].with_(B=2, Hq=8, Hkv=2, L=608),
    "longprompt": synth.WORKLOADS["longprompt"].with_(Hq=8, Hkv=2, L=1184),
}


def _run_case(dkv, w, n_blocks, steps=(0,), splits=(0,), kernel=0, check_export=True):
    torch = _torch()
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    if kernel:
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
    oc = oracle_cache(w, cap, P)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    assert dkv.dkv_cache_len(cache) == oc.len
    if check_export:
        compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    assert dkv.dkv_cache_status(cache) == oc.flags
    results = []
    for st in steps:
        Q = synth.queries_bits(w, st)
        Ka, Va = synth.active_block_bits(w, st)
        ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
        for sp in splits:
            dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, sp)
            out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
            dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                    w.softmax_scale, out)
            torch.cuda.synchronize()
            got = host_bits(out)
            results.append(got)
            assert_close(got, ref, f"{w.name} step {st} splits {sp}")
    return cache, results


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("name", list(SHRUNK))
def test_commit_and_attention_parity(dkv, name, kernel):
    """kernel 1 = warp-level mma.sync, 2 = tcgen05 (the default)."""
    w = SHRUNK[name]
    cache, _ = _run_case(dkv, w, w.L // w.blk, steps=(0, 1), splits=(0, 1, 3), kernel=kernel)
    assert dkv.dkv_last_attention_plan(cache)[0] == kernel


@pytest.mark.parametrize("name", ["batch32", "tiny"])
def test_odd_commit_count_leaves_tail(dkv, name):
    w = SHRUNK[name].with_(k_group=64)
    _run_case(dkv, w, 7, steps=(2,), splits=(0, 2))


@pytest.mark.parametrize("kb,vb,gk,gv", [(16, 16, 32, 32), (16, 4, 32, 32), (4, 16, 64, 32),
                                         (2, 16, 128, 32), (4, 2, 128, 128), (2, 4, 32, 128)])
def test_bit_width_and_group_mix(dkv, kb, vb, gk, gv):
    w = SHRUNK["gqa7b"].with_(k_bits=kb, v_bits=vb, k_group=gk, v_group=gv, L=416)
    _run_case(dkv, w, 13, steps=(3,), splits=(0, 1))


def test_passthrough_equals_dense_attention(dkv):
    """bits = 16: the cache stores bf16, and the result is dense softmax
    attention over the committed + active K/V (checked by the oracle, which
    pins this case against exact arithmetic)."""
    w = SHRUNK["mha8b"].with_(k_bits=16, v_bits=16, L=320)
    _run_case(dkv, w, 10, steps=(0, 5), splits=(0, 1))


def test_empty_cache_attends_active_block_only(dkv):
    w = SHRUNK["gqa7b"]
    _run_case(dkv, w, 0, steps=(0,), splits=(0,))


def test_single_block_cache(dkv):
    w = SHRUNK["batch32"]
    _run_case(dkv, w, 1, steps=(0,), splits=(0,))


def test_split_count_does_not_change_result(dkv):
    torch = _torch()
    w = SHRUNK["longprompt"]
    _, outs = _run_case(dkv, w, 37, steps=(1,), splits=(1, 2, 5, 9, 0))
    base = synth.bf16_bits_to_f32(outs[0]).astype(np.float64)
    # split counts change only fp32 rounding: at most one bf16 ulp apart
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(base), 2.0 ** -126))) - 7)
    for o in outs[1:]:
        x = synth.bf16_bits_to_f32(o).astype(np.float64)
        assert np.all(np.abs(x - base) <= ulp + 1e-3)
    del torch


def test_repeat_runs_are_bit_identical(dkv):
    torch = _torch()
    w = SHRUNK["gqa7b"]
    cache, _ = _run_case(dkv, w, 9, steps=(), splits=())
    Q = dev_bf16(synth.queries_bits(w, 0))
    Ka, Va = [dev_bf16(x) for x in synth.active_block_bits(w, 0)]
    outs = []
    for _ in range(3):
        out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        dkv.dkv_block_attention(cache, Q, Ka, Va, w.softmax_scale, out)
        outs.append(host_bits(out))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_gqa_equals_mha_with_replicated_kv(dkv):
    torch = _torch()
    w = SHRUNK["batch32"].with_(B=1, Hq=8, Hkv=2)
    wm = w.with_(Hkv=8)
    cap = default_cap(w, 6)
    c1 = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 64))
    c2 = dkv.dkv_cache_alloc(gpu_config(dkv, wm, cap, 64))
    rep = [0, 0, 0, 0, 1, 1, 1, 1]
    for i in range(5):
        K, V, M = synth.block_inputs(w, i)
        dkv.dkv_commit_block(c1, dev_bf16(K), dev_bf16(V), dev_words(M))
        dkv.dkv_commit_block(c2, dev_bf16(K[:, rep]), dev_bf16(V[:, rep]), dev_words(M[:, rep]))
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    o1 = torch.empty((1, 8, 32, 128), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    dkv.dkv_block_attention(c1, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), 0.1, o1)
    dkv.dkv_block_attention(c2, dev_bf16(Q), dev_bf16(Ka[:, rep]), dev_bf16(Va[:, rep]), 0.1, o2)
    a = synth.bf16_bits_to_f32(host_bits(o1)).astype(np.float64)
    b = synth.bf16_bits_to_f32(host_bits(o2)).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    assert np.all(np.abs(a - b) <= ulp + 1e-3)


@pytest.mark.parametrize("kernel", [1, 2])
def test_permuting_whole_groups_leaves_output(dkv, kernel):
    """Committing whole K groups (here one block each) in another order gives
    the same attention: both orders are within the output bound of the
    oracle's value for the original order (the oracle's own invariance is a
    CPU pin)."""
    torch = _torch()
    w = SHRUNK["batch32"].with_(k_group=32)
    order = [5, 0, 3, 1, 4, 2]
    cap = default_cap(w, len(order) + 1)
    P = default_P(w, cap)
    oc = oracle_cache(w, cap, P)
    outs = []
    Q = synth.queries_bits(w, 3)
    Ka, Va = synth.active_block_bits(w, 3)
    for blocks in (sorted(order), order):
        cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
        dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
        commit_both(dkv, cache, oc if blocks is not order else None, w, blocks)
        out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale,
                                out)
        torch.cuda.synchronize()
        outs.append(host_bits(out))
        dkv.dkv_cache_free(cache)
    ref = oc.block_attention(Q, Ka, Va, w.softmax_scale)
    for o in outs:
        assert_close(o, ref, f"kernel {kernel}")


def test_all_protected_group_and_side_table_overflow(dkv):
    w = SHRUNK["tiny"].with_(prot_frac=0.0)
    cap, P = 256, 40
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = oracle_cache(w, cap, P)
    for i in range(4):
        K, V, _ = synth.block_inputs(w, i)
        M = np.zeros((1, 1, 1), np.uint32)
        M[0, 0, 0] = 0xFFFFFFFF if i in (1, 2) else 0x00010001
        dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), dev_words(M))
        oc.commit(K, V, M)
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    flags = dkv.dkv_cache_status(cache)
    assert flags == oc.flags and flags & dkv.DKV_FLAG_CAPACITY
    assert dkv.dkv_cache_status(cache) == 0   # read-and-clear
    torch = _torch()
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    out = torch.empty((1, 4, 32, 128), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    assert_close(host_bits(out), oc.block_attention(Q, Ka, Va, w.softmax_scale))


@pytest.mark.parametrize("bits,group", [(2, 32), (4, 32), (2, 64), (4, 64)])
def test_commit_codes_at_rounding_ties(dkv, bits, group):
    """Grid inputs put many (x - z) / s quotients exactly on k + 1/2 or within
    an ulp of it: the codes must still be those of the correctly rounded
    division with round-half-even."""
    w = SHRUNK["tiny"].with_(k_bits=bits, v_bits=bits, k_group=group, v_group=group,
                             prot_frac=0.0)
    levels = (1 << bits) - 1
    cap = 256
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 8))
    oc = oracle_cache(w, cap, 8)
    for i in range(6):
        K, V = synth.grid_block_bits(w, i, levels)
        dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), None)
        oc.commit(K, V, None)
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())


def test_range_flag_and_clamp(dkv):
    w = SHRUNK["tiny"]
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, 128, 8))
    oc = oracle_cache(w, 128, 8)
    K, V, M = synth.block_inputs(w, 0)
    V = V.copy()
    K = K.copy()
    V[0, 0, 3, 7] = 0x7F80           # +inf
    K[0, 0, 5, 9] = 0x4780           # 65536 > fp16 max
    V[0, 0, 4, 1] = 0x7FC1           # NaN
    dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), dev_words(M))
    oc.commit(K, V, M)
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    assert dkv.dkv_cache_status(cache) == oc.flags == dkv.DKV_FLAG_RANGE


def test_capacity_error_leaves_state(dkv):
    w = SHRUNK["tiny"]
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, 64, 8))
    commit_both(dkv, cache, None, w, range(2))
    K, V, M = synth.block_inputs(w, 2)
    with pytest.raises(dkv.DkvError) as ei:
        dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), dev_words(M))
    assert ei.value.code == dkv.DKV_ERR_CAPACITY
    assert dkv.dkv_cache_len(cache) == 64


@pytest.mark.parametrize("gk", [32, 64])
def test_truncate_then_recommit(dkv, gk):
    torch = _torch()
    w = SHRUNK["batch32"].with_(k_group=gk, prot_frac=0.1)
    cap = default_cap(w, 12)
    P = 64
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = oracle_cache(w, cap, P)
    commit_both(dkv, cache, oc, w, range(7))
    dkv.dkv_cache_truncate(cache, 128)
    oc.truncate(128)
    commit_both(dkv, cache, oc, w, (9, 10, 11))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    assert_close(host_bits(out), oc.block_attention(Q, Ka, Va, w.softmax_scale))
    with pytest.raises(dkv.DkvError):
        dkv.dkv_cache_truncate(cache, 32 if gk == 64 else 33)


@pytest.mark.parametrize("gk", [32, 64])
def test_truncate_recorded_then_attention_export_commit(dkv, gk):
    """Truncation only records the new length: attention right after it, two
    truncations in a row, export applying it, and a later commit must all
    agree with the oracle."""
    torch = _torch()
    w = SHRUNK["batch32"].with_(k_group=gk, prot_frac=0.1)
    cap = default_cap(w, 12)
    P = 64
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = oracle_cache(w, cap, P)
    commit_both(dkv, cache, oc, w, range(7))
    for n in (192, 128):
        dkv.dkv_cache_truncate(cache, n)
        oc.truncate(n)
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    assert_close(host_bits(out), oc.block_attention(Q, Ka, Va, w.softmax_scale))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())
    commit_both(dkv, cache, oc, w, (8, 9, 10))
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())


def test_null_protect_mask_means_none(dkv):
    w = SHRUNK["batch32"]
    cap = default_cap(w, 4)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, 8))
    oc = oracle_cache(w, cap, 8)
    commit_both(dkv, cache, oc, w, range(4), protect=False)
    compare_exports(dkv.dkv_cache_export(cache), oc.snapshot())


# ------------------------------------------------------------- full sizes

def _unit_oracle(w, b, h, n_blocks, cap, P):
    oc = oracle_cache(w, cap, P, B=1, Hkv=1, Hq=w.g)
    for i in range(n_blocks):
        K, V = synth.kv_block_bits(w, b, h, i)
        M = synth.block_protect_words(w, b, h, i)
        oc.commit(K[None, None], V[None, None], M[None, None])
    return oc


@pytest.mark.parametrize("name", ["mha8b", "gqa7b", "batch32", "longprompt"])
def test_full_size_sampled_units(dkv, name):
    """The workloads at their full sizes, in the launch configuration the
    benchmark uses (automatic kernel and split choice): the whole cache is
    built through dkv_commit_block, then sampled units are checked against a
    single-unit oracle fed the same blocks (codes bit-exact, attention within
    tolerance)."""
    torch = _torch()
    w = synth.WORKLOADS[name]
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    commit_both(dkv, cache, None, w, range(n_blocks))
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), w.softmax_scale, out)
    got = host_bits(out)
    assert dkv.dkv_cache_status(cache) == 0
    exp = dkv.dkv_cache_export(cache)
    rng = np.random.default_rng(0)
    units = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(2)}
                   | {(w.B - 1, w.Hkv - 1)})
    for (b, h) in units:
        oc = _unit_oracle(w, b, h, n_blocks, cap, P)
        u = b * w.Hkv + h
        compare_exports({k: (v if k == "len" else v[u:u + 1]) for k, v in exp.items()},
                        oc.snapshot())
        ref = oc.block_attention(Q[b:b + 1, h * w.g:(h + 1) * w.g], Ka[b:b + 1, h:h + 1],
                                 Va[b:b + 1, h:h + 1], w.softmax_scale)
        assert_close(got[b:b + 1, h * w.g:(h + 1) * w.g], ref, f"{name} unit {(b, h)}")
    # every output finite and bounded by the largest |V| of the cache
    allv = synth.bf16_bits_to_f32(got)
    assert np.all(np.isfinite(allv))


@pytest.mark.parametrize("kernel,splits", [(2, 1), (2, 4), (2, 0), (1, 0)])
def test_repeat_bit_identical_mha8b(dkv, kernel, splits):
    """The attention of a fixed plan is deterministic: repeated calls give the
    same bits in every unit.  The 32-row query groups of the 8B MHA workload
    leave three of the four warps of each softmax warpgroup with padding rows
    only; a hand-off that lets those warps run a tile ahead of the row warps
    shows up as rows that change from call to call."""
    torch = _torch()
    w = synth.WORKLOADS["mha8b"]
    n_blocks = w.L // w.blk
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    commit_both(dkv, cache, None, w, range(n_blocks))
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_ATTN_KERNEL, kernel)
    dkv.dkv_cache_set_option(cache, dkv.DKV_OPT_SPLITS, splits)
    q, ka, va = (dev_bf16(x) for x in (synth.queries_bits(w, 0), *synth.active_block_bits(w, 0)))
    outs = []
    for _ in range(8):
        out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
        dkv.dkv_block_attention(cache, q, ka, va, w.softmax_scale, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dkv.dkv_cache_status(cache) == 0
    first = host_bits(outs[0])
    for i, o in enumerate(outs[1:], 1):
        diff = np.argwhere(host_bits(o) != first)
        assert diff.size == 0, f"call {i} differs from call 0 at (b, head, row, ch) {diff[:4].tolist()}"
