"""Seeded synthetic workloads for the quantize-on-commit / block-attention path.

This module only draws random numbers and formats them (fp32 -> bf16 bit
patterns, bit masks).  It holds none of the method's arithmetic: no
quantizer, no dequantizer, no attention.  Both the CPU oracle's tests and the
CUDA path's tests and benchmark take their inputs from here, so the two sides
see identical bytes.

Workload shapes follow the five synthetic configurations the pages' setting
implies (8B-class dLLM heads, 32-token blocks, long prompts; the block
diffusion description in "SoloQ: Calibration-Free Quantization for Diffusion
Language Models", and MaskAhead's batch-32 systems profile).  The pages print
no head counts or distributions; those are fixed here, in WORKLOADS below.

Every random draw is addressable by position: the K/V of one 32-token block of
one (batch, kv-head) unit comes from its own PCG64 stream keyed by
(seed, unit, block), so a test can regenerate any unit alone.
"""
from __future__ import annotations

import math
import functools
from dataclasses import dataclass, replace

import numpy as np

# stream tags keep independent draws apart
_TAG_OUTLIER = 1
_TAG_QUERY = 2
_TAG_KV_BLOCK = 3
_TAG_PROT_PREFILL = 4
_TAG_PROT_LATE = 5
_TAG_ACTIVE = 6
_TAG_GRID = 7
_TAG_ROTATION = 8


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int               # committed tokens per sequence before the timed steps
    blk: int
    k_bits: int
    v_bits: int
    k_group: int
    v_group: int
    prot_frac: float     # fraction of token positions per (b, kv-head) protected
    n_outlier: int       # K channels per kv-head scaled by outlier_scale
    outlier_scale: float
    k_dist: str          # "normal" or "student_t3"
    q_std: float         # Q ~ N(0, q_std^2)
    softmax_scale: float
    seed: int = 0
    attn_steps: int = 1  # denoising-step attentions the workload runs per block

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def rows(self) -> int:
        return self.g * self.blk

    @property
    def n_prot_prefill(self) -> int:
        return int(round(self.prot_frac * self.L))

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _five_pct(d: int) -> int:
    return int(round(0.05 * d))


WORKLOADS = {
    # 1 tiny: 4 of 128 K channels x10, 4-bit K/V, groups of 32, no protection
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=128, L=256, blk=32,
                     k_bits=4, v_bits=4, k_group=32, v_group=32,
                     prot_frac=0.0, n_outlier=4, outlier_scale=10.0,
                     k_dist="normal", q_std=1.0,
                     softmax_scale=1.0 / math.sqrt(128), seed=0),
    # 2 8B MHA-like layer: Q ~ N(0,1)/sqrt(d) already carries 1/sqrt(d)
    "mha8b": Workload("mha8b", B=1, Hq=32, Hkv=32, d=128, L=4096, blk=32,
                      k_bits=4, v_bits=4, k_group=32, v_group=32,
                      prot_frac=0.01, n_outlier=_five_pct(128), outlier_scale=10.0,
                      k_dist="normal", q_std=1.0 / math.sqrt(128),
                      softmax_scale=1.0, seed=0),
    # 3 7B GQA-like layer: 2-bit, groups of 32
    "gqa7b": Workload("gqa7b", B=8, Hq=28, Hkv=4, d=128, L=8192, blk=32,
                      k_bits=2, v_bits=2, k_group=32, v_group=32,
                      prot_frac=0.01, n_outlier=_five_pct(128), outlier_scale=10.0,
                      k_dist="normal", q_std=1.0,
                      softmax_scale=1.0 / math.sqrt(128), seed=0),
    # 4 batch-32 decode profile: 2-bit, groups of 64 (K tail of 32 between commits)
    "batch32": Workload("batch32", B=32, Hq=32, Hkv=8, d=128, L=16384, blk=32,
                        k_bits=2, v_bits=2, k_group=64, v_group=64,
                        prot_frac=0.02, n_outlier=_five_pct(128), outlier_scale=10.0,
                        k_dist="normal", q_std=1.0,
                        softmax_scale=1.0 / math.sqrt(128), seed=0),
    # 5 long prompt: 4096 commits of 32 tokens, then 64 attentions; Student-t K
    "longprompt": Workload("longprompt", B=1, Hq=32, Hkv=8, d=128, L=131072, blk=32,
                           k_bits=4, v_bits=4, k_group=32, v_group=32,
                           prot_frac=0.005, n_outlier=0, outlier_scale=1.0,
                           k_dist="student_t3", q_std=1.0,
                           softmax_scale=1.0 / math.sqrt(128), seed=0,
                           attn_steps=64),
}

WORKLOAD_ORDER = ["tiny", "mha8b", "gqa7b", "batch32", "longprompt"]


# ---------------------------------------------------------------- formatting

def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the uint16
    bit patterns.  Inputs here are finite, so no NaN handling is needed."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + (((u >> 16) & 1) + 0x7FFF)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def positions_to_mask(pos_in_block, blk: int) -> np.ndarray:
    """Bit t of word t//32 is set for each block-relative position t."""
    words = np.zeros((blk + 31) // 32, dtype=np.uint32)
    for t in pos_in_block:
        words[t // 32] |= np.uint32(1) << np.uint32(t % 32)
    return words


# ---------------------------------------------------------------- draws

def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


@functools.lru_cache(maxsize=4096)
def outlier_channels(w: Workload, h: int) -> np.ndarray:
    """K channels of kv-head h scaled by the outlier factor (same for every b)."""
    if w.n_outlier == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(w.seed, _TAG_OUTLIER, h).choice(w.d, w.n_outlier, replace=False))


def kv_block_f32(w: Workload, b: int, h: int, block: int):
    """fp32 K and V [blk, d] of token block `block` of unit (b, h), before
    bf16 rounding."""
    r = _rng(w.seed, _TAG_KV_BLOCK, b, h, block)
    if w.k_dist == "normal":
        k = r.standard_normal((w.blk, w.d), dtype=np.float32)
    elif w.k_dist == "student_t3":
        k = r.standard_t(3.0, (w.blk, w.d)).astype(np.float32)
    else:
        raise ValueError(w.k_dist)
    v = r.standard_normal((w.blk, w.d), dtype=np.float32)
    oc = outlier_channels(w, h)
    if oc.size:
        k[:, oc] *= np.float32(w.outlier_scale)
    return k, v


def kv_block_bits(w: Workload, b: int, h: int, block: int):
    k, v = kv_block_f32(w, b, h, block)
    return f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def unit_kv_bits(w: Workload, b: int, h: int, n_tokens: int):
    """bf16 bits of K and V [n_tokens, d] for positions [0, n_tokens) of one
    unit (n_tokens a multiple of blk)."""
    assert n_tokens % w.blk == 0
    ks, vs = [], []
    for blk_i in range(n_tokens // w.blk):
        k, v = kv_block_bits(w, b, h, blk_i)
        ks.append(k)
        vs.append(v)
    if not ks:
        return (np.zeros((0, w.d), np.uint16), np.zeros((0, w.d), np.uint16))
    return np.concatenate(ks), np.concatenate(vs)


@functools.lru_cache(maxsize=4096)
def prefill_protected_positions(w: Workload, b: int, h: int) -> np.ndarray:
    """round(prot_frac * L) distinct positions of [0, L), uniform, sorted."""
    n = w.n_prot_prefill
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(w.seed, _TAG_PROT_PREFILL, b, h).choice(w.L, n, replace=False))


def block_protect_words(w: Workload, b: int, h: int, block: int) -> np.ndarray:
    """Protect mask words of one block of unit (b, h).  Inside the prefill
    [0, L) they come from the uniform pick; past it each position is
    protected with probability prot_frac."""
    start = block * w.blk
    if start + w.blk <= w.L:
        pos = prefill_protected_positions(w, b, h)
        sel = pos[(pos >= start) & (pos < start + w.blk)] - start
    else:
        if w.prot_frac == 0.0:
            sel = np.zeros(0, dtype=np.int64)
        else:
            u = _rng(w.seed, _TAG_PROT_LATE, b, h, block).random(w.blk)
            sel = np.nonzero(u < w.prot_frac)[0]
    return positions_to_mask(sel, w.blk)


def block_inputs(w: Workload, block: int, units=None):
    """K, V bf16 bits [B, Hkv, blk, d] and protect words [B, Hkv, nw] of one
    block for all units (or only `units`, a list of (b, h); others zero)."""
    nw = (w.blk + 31) // 32
    K = np.zeros((w.B, w.Hkv, w.blk, w.d), np.uint16)
    V = np.zeros_like(K)
    M = np.zeros((w.B, w.Hkv, nw), np.uint32)
    todo = units if units is not None else [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    for (b, h) in todo:
        K[b, h], V[b, h] = kv_block_bits(w, b, h, block)
        M[b, h] = block_protect_words(w, b, h, block)
    return K, V, M


def grid_block_bits(w: Workload, block: int, levels: int):
    """K, V bf16 bits [B, Hkv, blk, d] on a grid of multiples of 1/64 in
    [0, levels], each (token, 32-channel) row of V and each (channel, 32-token)
    column of K holding both ends 0 and levels.  With group min 0 and max
    `levels` the scale is 1 or close to it, so many (x - z) / s quotients land
    exactly on or next to a rounding tie k + 1/2.  Seeded like the others."""
    r = _rng(w.seed, _TAG_GRID, block, levels)
    shape = (w.B, w.Hkv, w.blk, w.d)
    x = r.integers(0, 64 * levels + 1, size=(2,) + shape).astype(np.float32) / np.float32(64)
    K, V = x[0], x[1]
    V[..., 0::32] = 0.0
    V[..., 1::32] = float(levels)
    K[..., 0, :] = 0.0
    K[..., 1, :] = float(levels)
    # every other token row of V and channel of K slightly stretched, so that
    # its scale is not exactly 1 and quotients fall next to the ties
    f = np.array([1.0, 1.0 - 1.0 / 256, 1.0 + 1.0 / 256, 1.0 - 3.0 / 512], np.float32)
    V[:, :, 1::2, :] *= f[r.integers(0, 4, size=V[:, :, 1::2, :1].shape)]
    K[..., 1::2] *= f[r.integers(0, 4, size=K[..., :1, 1::2].shape)]
    return f32_to_bf16_bits(K), f32_to_bf16_bits(V)


def queries_bits(w: Workload, step: int) -> np.ndarray:
    """Q [B, Hq, blk, d] bf16 bits of denoising step `step`."""
    r = _rng(w.seed, _TAG_QUERY, step)
    q = r.standard_normal((w.B, w.Hq, w.blk, w.d), dtype=np.float32) * np.float32(w.q_std)
    return f32_to_bf16_bits(q)


def active_block_bits(w: Workload, step: int):
    """Active-block K, V [B, Hkv, blk, d] bf16 bits of denoising step `step`:
    drawn like committed K/V (same outlier channels and K distribution)."""
    K = np.zeros((w.B, w.Hkv, w.blk, w.d), np.uint16)
    V = np.zeros_like(K)
    for b in range(w.B):
        for h in range(w.Hkv):
            r = _rng(w.seed, _TAG_ACTIVE, step, b, h)
            if w.k_dist == "normal":
                k = r.standard_normal((w.blk, w.d), dtype=np.float32)
            else:
                k = r.standard_t(3.0, (w.blk, w.d)).astype(np.float32)
            v = r.standard_normal((w.blk, w.d), dtype=np.float32)
            oc = outlier_channels(w, h)
            if oc.size:
                k[:, oc] *= np.float32(w.outlier_scale)
            K[b, h] = f32_to_bf16_bits(k)
            V[b, h] = f32_to_bf16_bits(v)
    return K, V


def shrink(w: Workload, **kw) -> Workload:
    """A smaller case of the same recipe (for tests the oracle finishes in
    seconds): overrides sizes, keeps the distributions."""
    return w.with_(**kw)


def krpbh_params(seed: int, b: int, d: int = 128):
    """Random draws of a K-RPBH rotation with blocks of b coordinates: a
    permutation of [0, d) (int32) and a Haar-random (d/b) x (d/b) orthogonal
    mix (QR of a Gaussian matrix, column signs fixed by R's diagonal),
    rounded to fp32 -- the form the library takes them in."""
    k = d // b
    r = _rng(seed, _TAG_ROTATION, b)
    perm = r.permutation(d).astype(np.int32)
    q, rr = np.linalg.qr(r.standard_normal((k, k)))
    mix = (q * np.sign(np.diag(rr))[None, :]).astype(np.float32)
    return perm, mix
