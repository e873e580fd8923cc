"""Helpers shared by the GPU tests: move synth inputs to the device, drive the
library and the oracle over the same blocks, compare results."""
import numpy as np

import synth
from oracle import OracleCache, bf16_to_f64

# tolerance on bf16 attention outputs against the oracle rounded to bf16
ATOL_MAX = 1e-2
ATOL_MEAN = 1e-3


def torch_mod():
    import torch
    return torch


def dev_bf16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_words(words: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).cuda()


def host_bits(t) -> np.ndarray:
    torch = torch_mod()
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_config(dkv, w: synth.Workload, cap: int, P: int, sink: int = 0):
    return dkv.make_config(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, w.k_group,
                           w.v_group, P, cap, sink)


def oracle_cache(w: synth.Workload, cap: int, P: int, B=None, Hkv=None, Hq=None, sink=0):
    return OracleCache(B or w.B, Hq or w.Hq, Hkv or w.Hkv, w.d, w.blk, w.k_bits, w.v_bits,
                       w.k_group, w.v_group, P, cap, sink)


def default_cap(w: synth.Workload, n_blocks: int) -> int:
    unit = max(w.k_group, w.blk)
    return ((n_blocks * w.blk + unit - 1) // unit + 1) * unit


def default_P(w: synth.Workload, cap: int) -> int:
    return int(round(w.prot_frac * cap)) * 2 + 16


def commit_both(dkv, cache, oc, w, blocks, protect=True):
    """Commit blocks (ids) to the GPU cache and, if given, the oracle cache."""
    for i in blocks:
        K, V, M = synth.block_inputs(w, i)
        dkv.dkv_commit_block(cache, dev_bf16(K), dev_bf16(V), dev_words(M) if protect else None)
        if oc is not None:
            oc.commit(K, V, M if protect else None)


def compare_exports(gpu: dict, ref: dict, units=None):
    """Bit-exact comparison of the canonical arrays (optionally a unit subset
    of the GPU export against a single-unit oracle, in order)."""
    sel = (lambda a: a) if units is None else (lambda a: a[units])
    assert gpu["len"] == ref["len"]
    for key in ("k_codes", "k_tail", "tail_mask", "v_codes", "prot_count", "prot_gstart",
                "k_raw", "v_raw", "v_sink"):
        if key in ref:
            g = sel(gpu[key])
            assert g.shape == ref[key].shape, (key, g.shape, ref[key].shape)
            bad = np.nonzero(g != ref[key])
            assert bad[0].size == 0, (key, [b[:5] for b in bad])
    for key in ("k_sz", "v_sz"):
        if key in ref:
            g = sel(gpu[key]).view(np.uint16)
            assert np.array_equal(g, ref[key].view(np.uint16)), key
    if "prot_pos" in ref and "prot_pos" in gpu:
        n = ref["prot_count"]
        gp, gk = sel(gpu["prot_pos"]), sel(gpu["prot_k"])
        for i in range(len(n)):
            assert np.array_equal(gp[i, :n[i]], ref["prot_pos"][i, :n[i]])
            assert np.array_equal(gk[i, :n[i]], ref["prot_k"][i, :n[i]])


def output_bound(ref64: np.ndarray, arith: float = ATOL_MAX) -> np.ndarray:
    """Per-element max-abs bound on a bf16 output against the exact (fp64)
    oracle value: `arith` (1e-2) for the arithmetic, plus the bf16 output
    format's own rounding (half an ulp of |o|, 8 significant bits), which no
    implementation can avoid (it alone is 0.0156 at |o| >= 4)."""
    a = np.maximum(np.abs(np.asarray(ref64, np.float64)), 2.0 ** -126)
    half_ulp = np.exp2(np.floor(np.log2(a)) - 8)
    return arith + half_ulp


def bf16_round(ref64: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 (nearest even, through fp32) -> fp64."""
    return bf16_to_f64(synth.f32_to_bf16_bits(np.asarray(ref64, np.float64).astype(np.float32)))


def assert_close(got_bits: np.ndarray, ref64: np.ndarray, what="", scale_mul: float = 1.0):
    """GPU bf16 output vs the fp64 oracle: every element within output_bound
    of the exact value; mean absolute difference to the oracle rounded to
    bf16 <= 1e-3 (the mean of bf16's own rounding alone is ulp/4, about 1e-3
    at |o| ~ 0.5-1, so the mean is taken between two bf16 results).
    scale_mul > 1: the softmax scale is that multiple of the workload's;
    score errors from fp16 operands grow with the scale, so both arithmetic
    bounds are multiplied by it."""
    got = bf16_to_f64(got_bits)
    ref = np.asarray(ref64, np.float64)
    assert np.all(np.isfinite(got)), what
    m = max(1.0, float(scale_mul))
    err = np.abs(got - ref)
    ratio = err / output_bound(ref, ATOL_MAX * m)
    assert ratio.max() <= 1.0, (what, float(err.max()), float(ratio.max()))
    mean = float(np.abs(got - bf16_round(ref)).mean())
    assert mean <= ATOL_MEAN * m, (what, mean)
    return float(err.max()), mean
