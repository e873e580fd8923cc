"""Q-MaskAhead selection (MaskAhead / Q-MaskAhead abstract) through the C-ABI
against the oracle's block_attention_selected:

* the contribution scores c_j of every committed token agree with the
  oracle's (fp16 tensor-core scores against fp64: a relative bound);
* the kept positions are exactly the top `budget` of the library's own
  scores, equal scores going to the lower position (checked bit for bit on
  the host), and they differ from the oracle's selection only among tokens
  whose oracle score ties the budget's boundary within that bound;
* the output equals the oracle's attention over the library's own selection
  plus the active block, within the output bound;
* budget 0 attends to the active block alone, a budget covering the cache
  gives the full attention."""
import numpy as np
import pytest

import synth
from gpu_util import (assert_close, commit_both, default_P, default_cap, dev_bf16, gpu_config,
                      host_bits, oracle_cache)
from test_gpu_parity import SHRUNK

pytestmark = pytest.mark.gpu

REL = 3e-2   # relative bound on a score
ABS = 1e-3   # ... plus this fraction of the unit's largest score


@pytest.fixture(scope="module")
def dkv():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_kv_cache_dkv_b200 as m
    return m


def _setup(dkv, w):
    n_blocks = w.L // w.blk + 1          # an odd count: a K tail with groups of 64
    cap = default_cap(w, n_blocks + 1)
    P = default_P(w, cap)
    cache = dkv.dkv_cache_alloc(gpu_config(dkv, w, cap, P))
    oc = oracle_cache(w, cap, P)
    commit_both(dkv, cache, oc, w, range(n_blocks))
    return cache, oc, cap


def _run(dkv, cache, w, cap, step, budget):
    import torch
    Q = synth.queries_bits(w, step)
    Ka, Va = synth.active_block_bits(w, step)
    out = torch.empty((w.B, w.Hq, w.blk, w.d), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((w.B, w.Hkv, budget), -7, dtype=torch.int32, device="cuda")
    scores = torch.zeros((w.B, w.Hkv, cap), dtype=torch.float32, device="cuda")
    dkv.dkv_block_attention_selected(cache, dev_bf16(Q), dev_bf16(Ka), dev_bf16(Va),
                                     w.softmax_scale, budget, out, sel, scores)
    torch.cuda.synchronize()
    U = w.B * w.Hkv
    return (Q, Ka, Va), host_bits(out), sel.cpu().numpy().reshape(U, budget), \
        scores.cpu().numpy().reshape(U, cap)


def _check_selection(gsel, gsc, contribs, L, budget):
    k = min(budget, L)
    for u, c_ref in enumerate(contribs):
        s = gsc[u, :L].astype(np.float64)
        # scores against the oracle's contributions
        tol = REL * np.abs(c_ref) + ABS * c_ref.max()
        bad = np.nonzero(np.abs(s - c_ref) > tol)[0]
        assert bad.size == 0, (u, bad[:5], s[bad[:5]], c_ref[bad[:5]])
        # the selection is the top k of the library's own scores, ties low
        order = np.lexsort((np.arange(L), -gsc[u, :L].astype(np.float32)))
        want = np.sort(order[:k])
        assert np.array_equal(gsel[u, :k], want), u
        assert np.all(gsel[u, k:] == -1)
        # against the oracle's own selection: only boundary ties may differ
        ref_sel = np.sort(np.lexsort((np.arange(L), -c_ref))[:k])
        kth = np.sort(c_ref)[::-1][k - 1] if 0 < k < L else None
        for j in np.setxor1d(want, ref_sel):
            assert kth is not None and abs(c_ref[j] - kth) <= 2 * (REL * kth + ABS * c_ref.max()), \
                (u, j, c_ref[j], kth)


CASES = [("batch32", 96), ("gqa7b", 128), ("mha8b", 64), ("tiny", 40), ("longprompt", 300)]


@pytest.mark.parametrize("name,budget", CASES)
def test_selected_attention(dkv, name, budget):
    w = SHRUNK[name]
    cache, oc, cap = _setup(dkv, w)
    for step in (0, 1):
        (Q, Ka, Va), got, gsel, gsc = _run(dkv, cache, w, cap, step, budget)
        _, _, contribs = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, budget)
        _check_selection(gsel, gsc, contribs, oc.len, budget)
        k = min(budget, oc.len)
        ref, _, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, budget,
                                                selection=[gsel[u, :k] for u in range(oc.U)])
        assert_close(got, ref, f"{name} budget {budget} step {step}")
        assert dkv.dkv_last_attention_plan(cache)[0] == 1
    assert dkv.dkv_cache_status(cache) == 0


def test_selection_extremes(dkv):
    """Budget 0: the active block alone; a budget of the whole cache: the full
    attention (every token kept)."""
    w = SHRUNK["batch32"]
    cache, oc, cap = _setup(dkv, w)
    (Q, Ka, Va), got, gsel, _ = _run(dkv, cache, w, cap, 2, 0)
    ref, sel, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 0)
    assert gsel.size == 0 and all(len(s) == 0 for s in sel)
    assert_close(got, ref, "budget 0")
    (Q, Ka, Va), got, gsel, _ = _run(dkv, cache, w, cap, 3, cap)
    assert np.array_equal(gsel[:, :oc.len], np.tile(np.arange(oc.len), (oc.U, 1)))
    assert np.all(gsel[:, oc.len:] == -1)
    assert_close(got, oc.block_attention(Q, Ka, Va, w.softmax_scale), "budget = capacity")
    assert dkv.dkv_cache_status(cache) == 0
