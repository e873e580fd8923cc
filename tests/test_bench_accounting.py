"""The benchmark's algorithmic byte count (the numerator of its roofline
figures) against the sizes of the arrays one attention call must read, taken
from the oracle's canonical cache.  CPU only."""
import numpy as np
import pytest

import bench
import synth
from oracle import OracleCache


def _cache_bytes(oc: OracleCache) -> int:
    """Bytes of the committed state an attention call reads: codes and
    (scale, zero) pairs, the group index, the bf16 tail, raw rows, and the
    protected rows with their positions."""
    snap = oc.snapshot()
    n = 0
    for key in ("k_codes", "k_sz", "k_tail", "k_raw", "v_codes", "v_sz", "v_raw"):
        if key in snap:
            n += snap[key].nbytes
    if oc.kb < 16:
        n += snap["prot_gstart"].nbytes
        cnt = int(snap["prot_gstart"][:, -1].sum())
        n += cnt * (oc.d * 2 + 4)
    return n


@pytest.mark.parametrize("kb,vb,gk,gv,n_blocks", [(4, 4, 32, 32, 8), (2, 2, 64, 64, 9),
                                                  (2, 4, 32, 128, 5), (16, 4, 32, 32, 4),
                                                  (4, 16, 128, 32, 7), (16, 16, 32, 32, 3),
                                                  (3, 3, 64, 64, 9), (3, 4, 32, 32, 6),
                                                  (2, 3, 128, 32, 5)])
def test_attention_bytes_match_the_cache_arrays(kb, vb, gk, gv, n_blocks):
    """No protected tokens: bench.attn_bytes equals the cache arrays plus Q,
    the active block and the output, exactly."""
    w = synth.WORKLOADS["tiny"].with_(B=2, Hq=4, Hkv=2, k_bits=kb, v_bits=vb, k_group=gk,
                                      v_group=gv, prot_frac=0.0)
    cap = ((n_blocks * w.blk + 127) // 128 + 1) * 128
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, kb, vb, gk, gv, 0, cap)
    for i in range(n_blocks):
        K, V, _ = synth.block_inputs(w, i)
        oc.commit(K, V)
    io = w.B * w.Hq * w.blk * w.d * 2 * 2 + 2 * w.B * w.Hkv * w.blk * w.d * 2
    assert bench.io_bytes(w) == io
    assert bench.attn_bytes(w, oc.len) == _cache_bytes(oc) + io


def test_protected_rows_counted_at_the_expected_rate():
    """With protection the benchmark counts prot_frac of the quantized
    positions; the oracle cache built from the same generator holds a count
    within a few percent of that."""
    w = synth.WORKLOADS["tiny"].with_(B=4, Hq=8, Hkv=4, prot_frac=0.05)
    n_blocks = 24
    cap = n_blocks * w.blk + 128
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group, w.v_group,
                     cap, cap)
    for i in range(n_blocks):
        K, V, M = synth.block_inputs(w, i)
        oc.commit(K, V, M)
    got = bench.attn_bytes(w, oc.len)
    io = bench.io_bytes(w)
    want = _cache_bytes(oc) + io
    assert abs(got - want) / want < 0.02, (got, want)


def test_attention_flops_definition():
    """4 * rows * d multiply-add flops per (token, kv-head) over committed +
    active tokens (QK^T and PV, 2 flops per multiply-add)."""
    w = synth.WORKLOADS["batch32"]
    L = 1000
    assert bench.attn_flops(w, L) == 2 * 2 * w.rows * w.d * (L + w.blk) * w.B * w.Hkv
