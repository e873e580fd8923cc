"""The tcgen05 (tensor-memory) attention kernels against the CPU oracle:
query groups of 32 rows (a row block zero-padded to M = 128, and, on
request, with the tokens on the TMEM lanes), 128 rows, and 224 rows (two
row blocks of 112)."""
import pytest

import synth
from test_gpu_parity import SHRUNK, _run_case

pytestmark = pytest.mark.gpu

TC_CASES = {
    "tiny": SHRUNK["tiny"],
    "batch32": SHRUNK["batch32"],
    "longprompt": SHRUNK["longprompt"],
    "mha8b": SHRUNK["mha8b"],
    "gqa7b": SHRUNK["gqa7b"],
    "rows64": SHRUNK["batch32"].with_(Hq=4, Hkv=2),
    "rows256": SHRUNK["gqa7b"].with_(Hq=32, Hkv=4, B=1),
}


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


@pytest.mark.parametrize("name", list(TC_CASES))
def test_tc_parity(dkv, name):
    w = TC_CASES[name]
    cache, _ = _run_case(dkv, w, w.L // w.blk, steps=(0, 1), splits=(0, 1, 3), kernel=2)
    assert dkv.dkv_last_attention_plan(cache)[0] == 2
    assert dkv.dkv_cache_status(cache) == 0


# 32-row query groups: the row-block kernel (2, the default) and the
# tokens-on-lanes kernel (3), each against the oracle, and against each other
TL_CASES = {
    "mha8b": SHRUNK["mha8b"],
    "mha8b_2bit_g64": SHRUNK["mha8b"].with_(k_bits=2, v_bits=2, k_group=64, v_group=64),
    "mha8b_bf16": SHRUNK["mha8b"].with_(k_bits=16, v_bits=16),
    "mha8b_mixed": SHRUNK["mha8b"].with_(k_bits=4, v_bits=16, k_group=128),
    "mha8b_long": SHRUNK["mha8b"].with_(Hq=2, Hkv=2, L=4096, prot_frac=0.03),
    "gqa_g1_b32": SHRUNK["gqa7b"].with_(Hq=4, Hkv=4),
}


@pytest.mark.parametrize("name", list(TL_CASES))
def test_tokens_on_lanes_kernel(dkv, name):
    import numpy as np
    from oracle import bf16_to_f64
    w = TL_CASES[name]
    assert w.rows == 32
    n = w.L // w.blk
    c2, r2 = _run_case(dkv, w, n, steps=(0, 1), splits=(0, 1, 3), kernel=2, check_export=False)
    assert dkv.dkv_last_attention_plan(c2)[0] == 2
    c3, r3 = _run_case(dkv, w, n, steps=(0, 1), splits=(0, 1, 3), kernel=3, check_export=False)
    assert dkv.dkv_last_attention_plan(c3)[0] == 3
    for a_, b_ in zip(r2, r3):  # the same inputs: fp32 rounding order apart, one bf16 ulp
        x, y = bf16_to_f64(a_), bf16_to_f64(b_)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126))) - 7)
        assert np.all(np.abs(x - y) <= ulp + 1e-3)
    assert dkv.dkv_cache_status(c2) == 0 and dkv.dkv_cache_status(c3) == 0


@pytest.mark.parametrize("kb,vb,gk,gv", [(16, 16, 32, 32), (4, 2, 128, 64), (2, 4, 64, 128),
                                         (16, 2, 32, 32), (2, 16, 128, 32)])
def test_tc_bit_width_mix(dkv, kb, vb, gk, gv):
    w = SHRUNK["batch32"].with_(k_bits=kb, v_bits=vb, k_group=gk, v_group=gv, L=416)
    _run_case(dkv, w, 13, steps=(3,), splits=(0, 1), kernel=2)


def test_tc_empty_and_ragged(dkv):
    w = SHRUNK["longprompt"]
    _run_case(dkv, w, 0, steps=(0,), splits=(0,), kernel=2)
    _run_case(dkv, w, 1, steps=(0,), splits=(0,), kernel=2)
    _run_case(dkv, w, 5, steps=(1,), splits=(0, 2), kernel=2)


def test_tc_many_splits_long_cache(dkv):
    w = SHRUNK["longprompt"].with_(L=4096, Hq=4, Hkv=1)
    _run_case(dkv, w, 128, steps=(2,), splits=(1, 7, 0), kernel=2, check_export=False)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("blk,hq,hkv,gk", [(64, 4, 2, 32), (96, 2, 2, 32), (128, 2, 1, 128),
                                           (32, 5, 1, 64), (64, 2, 1, 128)])
def test_block_sizes_and_row_counts(dkv, kernel, blk, hq, hkv, gk):
    """Blocks of 64, 96 and 128 tokens and query groups of 96, 128, 160 and
    256 rows (padding warps, two row blocks, K groups longer and shorter than
    the block)."""
    w = SHRUNK["batch32"].with_(blk=blk, Hq=hq, Hkv=hkv, k_group=gk, v_group=32,
                                L=(640 // blk) * blk)
    _run_case(dkv, w, w.L // w.blk, steps=(0,), splits=(0, 2), kernel=kernel)


@pytest.mark.parametrize("name", ["gqa7b", "mha8b"])
@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("scale_mul", [-1.0, 0.0, 3.0])
def test_softmax_scale_sign_zero_and_large(dkv, name, kernel, scale_mul):
    """A negative scale (folded into Q on the tcgen05 path), zero (uniform
    weights: the mean of V) and three times the workload's (peaked weights,
    frequent reference rises; the fp16-operand score error grows with the
    scale, so the bound does too)."""
    import torch
    from gpu_util import assert_close, default_P, default_cap, dev_bf16, host_bits, oracle_cache
    w = SHRUNK[name]
    if kernel == 3 and w.rows != 32:
        pytest.skip("tokens on the TMEM lanes: 32-row query groups only")
    cache, _ = _run_case(dkv, w, w.L // w.blk, steps=(), kernel=kernel)
    cap = default_cap(w, w.L // w.blk + 1)
    ref_cache = oracle_cache(w, cap, default_P(w, cap))
    for i in range(w.L // w.blk):
        K, V, M = synth.block_inputs(w, i)
        ref_cache.commit(K, V, M)
    Q = synth.queries_bits(w, 4)
    Ka, Va = synth.active_block_bits(w, 4)
    scale = w.softmax_scale * scale_mul
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    dkv.dkv_block_attention(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va), scale, out)
    torch.cuda.synchronize()
    assert_close(host_bits(out), ref_cache.block_attention(Q, Ka, Va, scale),
                 scale_mul=abs(scale_mul))
