"""The tcgen05 (tensor-memory) attention kernel against the CPU oracle:
query groups of 32 rows (zero-padded to M = 128), 128 rows, and 224 rows (two
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
