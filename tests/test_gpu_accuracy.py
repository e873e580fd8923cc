"""The accuracy figures of the five workloads as the target states them:
max |gpu - bf16(oracle)| and mean |gpu - bf16(oracle)| on bf16 attention
outputs, next to max |gpu - oracle| against the unrounded fp64 value.  Each
is printed (run with -s to see the lines) and checked:

* mean |gpu - bf16(oracle)| <= 1e-3;
* every element with |gpu - bf16(oracle)| > 1e-2 is one bf16 ulp from the
  rounded oracle value, with the exact value within 1e-2 + half an ulp of
  the GPU's: two bf16 roundings of values closer than 1e-2 can land an ulp
  apart (0.0156 at |o| in [2, 4)), which no implementation avoids;
* max |gpu - oracle| <= 1e-2 + half an ulp (the tests' output bound)."""
import numpy as np
import pytest

import synth
from gpu_util import bf16_round, output_bound
from oracle import bf16_to_f64
from test_gpu_parity import SHRUNK, _run_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


@pytest.mark.parametrize("kernel", [2, 1])
@pytest.mark.parametrize("name", list(SHRUNK))
def test_accuracy_figures(dkv, name, kernel):
    from oracle import OracleCache
    from gpu_util import default_P, default_cap
    w = SHRUNK[name]
    n = w.L // w.blk
    cache, outs = _run_case(dkv, w, n, steps=(0, 1, 2), splits=(0,), kernel=kernel,
                            check_export=False)
    cap = default_cap(w, n + 1)
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group,
                     default_P(w, cap), cap)
    for i in range(n):
        K, V, M = synth.block_inputs(w, i)
        oc.commit(K, V, M)
    mx_b, mean_b, mx_e = 0.0, [], 0.0
    for st, got_bits in zip((0, 1, 2), outs):
        Q = synth.queries_bits(w, st)
        Ka, Va = synth.active_block_bits(w, st)
        exact = oc.block_attention(Q, Ka, Va, w.softmax_scale)
        got = bf16_to_f64(got_bits)
        rb = bf16_round(exact)
        d_b = np.abs(got - rb)
        d_e = np.abs(got - exact)
        big = d_b > 1e-2
        if big.any():
            a = np.maximum(np.abs(rb[big]), 2.0 ** -126)
            ulp = np.exp2(np.floor(np.log2(a)) - 7)
            assert np.all(d_b[big] <= ulp * (1 + 1e-9)), (name, float(d_b.max()))
        assert np.all(d_e <= output_bound(exact))
        mx_b = max(mx_b, float(d_b.max()))
        mx_e = max(mx_e, float(d_e.max()))
        mean_b.append(float(d_b.mean()))
    mean = float(np.mean(mean_b))
    assert mean <= 1e-3
    print(f"ACCURACY {name} kernel {kernel}: max|gpu-bf16(oracle)| {mx_b:.3e}  "
          f"mean|gpu-bf16(oracle)| {mean:.3e}  max|gpu-oracle| {mx_e:.3e}")
