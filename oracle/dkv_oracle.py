"""CPU oracle for quantize-on-commit and bidirectional block attention over a
low-bit block-diffusion KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may.  It shares no code with the CUDA library (no headers, no helpers, no
tables); the two meet only through the seeded inputs of the `synth` module and
the canonical cache layout written out below.

What it follows (the pages print no formula, kernel or bit layout; the
textbook meaning of the names they use is taken, and each reading of a step
the pages leave open is stated beside the function that takes it):

* "SoloQ: Calibration-Free Quantization for Diffusion Language Models"
  (block-diffusion paragraph): the cache is quantized at commit time and
  never earlier; the block under denoising keeps full precision; K is
  quantized per channel on an asymmetric grid, as in KIVI.
* "KV Cache Quantization for Diffusion Language Models" (Tai et al., Findings
  of EMNLP 2026, abstract): KIVI carried over to prefix-cache reuse; KProtect
  holds a chosen set of K entries in high precision, and V is stored at low
  bit width in the usual way.
* MaskAhead / Q-MaskAhead abstract: each denoising step of a block model
  reads the whole committed cache; the quantized variant does so on the
  low-bit cache itself.

Asymmetric quantizer of one group (b bits, 2^b - 1 levels), in fp32 with
round-to-nearest-even and no fused multiply-add:
    mn, mx = min, max over the group's non-protected members
    s = fp16(fp32(mx - mn) / (2^b - 1)),  z = fp16(mn)
    q = clamp(rint((x - z) / s), 0, 2^b - 1)    (q = 0 when s == 0)
Dequantization: x_hat = q * s + z (evaluated here in fp64).

Attention (fp64): O = softmax(scale * Q K_hat^T) V_hat over committed
(quantized) tokens, the bf16 K tail, and the bf16 active block; no mask;
query head h reads kv-head h // (Hq / Hkv).

Pins: every function here is checked in tests/test_oracle_pins.py against
closed forms, brute force, invariants and an exact-arithmetic softmax; none
is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

from . import krpbh

FLAG_CAPACITY = 0x1   # protected side table full: extra protected tokens quantized normally
FLAG_RANGE = 0x2      # a committed K/V value was non-finite or beyond fp16 range

FP16_MAX = np.float32(65504.0)


class CapacityError(Exception):
    """len + blk would exceed the cache capacity (state unchanged)."""


# ------------------------------------------------------------ number formats

def bf16_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32, exact: bf16 is the top half of fp32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def bf16_to_f64(bits) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def to_fp16(x) -> np.ndarray:
    """fp32 -> IEEE binary16, round to nearest, ties to even (subnormals kept,
    overflow to inf).  numpy's cast implements this rounding; the pins check
    it against a brute-force nearest search over all 2^16 patterns."""
    return np.asarray(x, dtype=np.float32).astype(np.float16)


def sanitize(x: np.ndarray):
    """Values the quantizer sees: NaN -> 0, others clamped to the fp16 range.
    Returns (values, range_flag)."""
    bad = ~np.isfinite(x) | (np.abs(x) > FP16_MAX)
    if not bad.any():
        return x, 0
    y = np.where(np.isnan(x), np.float32(0), x)
    y = np.clip(y, -FP16_MAX, FP16_MAX).astype(np.float32)
    return y, FLAG_RANGE


# ------------------------------------------------------------ quantizer

def quantize_groups(x: np.ndarray, keep: np.ndarray, bits: int):
    """Asymmetric min/max quantization of G independent groups.

    x    : fp32 [G, n]   the group members
    keep : bool [G, n]   members that take part (False = protected slot)
    returns codes uint8 [G, n], s float16 [G], z float16 [G]

    Protected members are left out of min/max and get code 0; a group with
    no member taking part gets s = z = 0.
    """
    x = np.asarray(x, dtype=np.float32)
    keep = np.broadcast_to(np.asarray(keep, dtype=bool), x.shape)
    levels = np.float32(2 ** bits - 1)
    anyk = keep.any(axis=1)
    mn = np.where(keep, x, np.float32(np.inf)).min(axis=1)
    mx = np.where(keep, x, np.float32(-np.inf)).max(axis=1)
    mn = np.where(anyk, mn, np.float32(0)).astype(np.float32)
    mx = np.where(anyk, mx, np.float32(0)).astype(np.float32)
    s_f = (mx - mn) / levels                      # fp32 subtract, fp32 divide
    s = to_fp16(s_f)
    z = to_fp16(mn)
    s32 = s.astype(np.float32)[:, None]
    z32 = z.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (x - z32) / np.where(s32 > 0, s32, np.float32(1))
    q = np.clip(np.rint(t), 0, levels)
    q = np.where((s32 > 0) & keep, q, 0).astype(np.uint8)
    return q, s, z


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Little-endian packing along the last axis: element e occupies bits
    [bits*e, bits*e + bits) of the bit stream formed by the words, where bit i
    of the stream is bit (i mod 32) of word floor(i / 32).  For bits 2 and 4
    no element crosses a word (element e sits at bits [bits*e mod 32, +bits)
    of word floor(bits*e / 32)); 3-bit elements do (32 of them fill 3 words)."""
    c = np.asarray(codes, dtype=np.uint32)
    n = c.shape[-1]
    assert (n * bits) % 32 == 0
    if 32 % bits == 0:
        per = 32 // bits
        c = c.reshape(c.shape[:-1] + (n // per, per))
        shifts = (np.arange(per, dtype=np.uint32) * np.uint32(bits))
        return np.bitwise_or.reduce(c << shifts, axis=-1).astype(np.uint32)
    c = c.astype(np.uint64)
    words = np.zeros(c.shape[:-1] + (n * bits // 32,), np.uint64)
    for e in range(n):
        w, off = divmod(bits * e, 32)
        words[..., w] |= (c[..., e] << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:                      # the high bits go to the next word
            words[..., w + 1] |= c[..., e] >> np.uint64(32 - off)
    return words.astype(np.uint32)


def unpack_codes(words: np.ndarray, bits: int, n: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint32)
    if 32 % bits == 0:
        per = 32 // bits
        shifts = (np.arange(per, dtype=np.uint32) * np.uint32(bits))
        c = (w[..., None] >> shifts) & np.uint32(2 ** bits - 1)
        c = c.reshape(w.shape[:-1] + (w.shape[-1] * per,))
        return c[..., :n].astype(np.uint8)
    w = w.astype(np.uint64)
    out = np.zeros(w.shape[:-1] + (n,), np.uint64)
    for e in range(n):
        i, off = divmod(bits * e, 32)
        v = w[..., i] >> np.uint64(off)
        if off + bits > 32:
            v = v | (w[..., i + 1] << np.uint64(32 - off))
        out[..., e] = v & np.uint64(2 ** bits - 1)
    return out.astype(np.uint8)


def mask_words_to_bool(words: np.ndarray, n: int) -> np.ndarray:
    """Bit t of word t // 32 -> bool [..., n]."""
    w = np.asarray(words, dtype=np.uint32)
    bits = (w[..., None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return bits.reshape(w.shape[:-1] + (w.shape[-1] * 32,))[..., :n].astype(bool)


def bool_to_mask_words(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=bool)
    n = b.shape[-1]
    nw = (n + 31) // 32
    pad = np.zeros(b.shape[:-1] + (nw * 32,), dtype=np.uint32)
    pad[..., :n] = b
    pad = pad.reshape(b.shape[:-1] + (nw, 32))
    return np.bitwise_or.reduce(pad << np.arange(32, dtype=np.uint32), axis=-1).astype(np.uint32)


# ------------------------------------------------------------ the cache

class OracleCache:
    """Committed low-bit KV cache of B sequences x Hkv kv-heads (units
    u = b * Hkv + h), in the canonical layout:

    k_codes  uint32  [U, cap/GK, d, GK*kb/32]  per (group, channel): the GK
                     tokens' codes packed along tokens          (kb in {2,4})
    k_sz     float16 [U, cap/GK, d, 2]         (scale, zero) per (group, channel)
    k_raw    uint16  [U, cap, d]               bf16 K            (kb == 16)
    k_tail   uint16  [U, GK, d]                bf16 K of the tokens of the
                     incomplete group, slot = position mod GK
    tail_mask uint32 [U, ceil(GK/32)]          protect bits of those slots
    v_codes  uint32  [U, cap, d*vb/32]         per token, packed along channels
    v_sz     float16 [U, cap, d/GV, 2]         (scale, zero) per (token, channel group)
    v_raw    uint16  [U, cap, d]               bf16 V            (vb == 16)
    prot_count  int32 [U]                      side-table entries in use
    prot_pos    int32 [U, P]                   their positions (ascending)
    prot_k      uint16 [U, P, d]               their K vectors, bf16 bits
    prot_gstart int32 [U, cap/GK + 1]          entries before group j
    """

    def __init__(self, B, Hq, Hkv, d, blk, k_bits, v_bits, k_group, v_group,
                 max_protected, capacity, sink_tokens=0, v_rotation=None):
        assert Hq % Hkv == 0
        assert k_bits in (2, 3, 4, 16) and v_bits in (2, 3, 4, 16)
        assert capacity % k_group == 0 and capacity % blk == 0
        assert d % v_group == 0
        self.B, self.Hq, self.Hkv, self.d, self.blk = B, Hq, Hkv, d, blk
        self.kb, self.vb, self.GK, self.GV = k_bits, v_bits, k_group, v_group
        self.P, self.cap = max_protected, capacity
        U = B * Hkv
        self.U = U
        self.len = 0
        self.flags = 0
        nG = capacity // k_group
        if k_bits < 16:
            self.k_codes = np.zeros((U, nG, d, k_group * k_bits // 32), np.uint32)
            self.k_sz = np.zeros((U, nG, d, 2), np.float16)
        else:
            self.k_raw = np.zeros((U, capacity, d), np.uint16)
        self.k_tail = np.zeros((U, k_group, d), np.uint16)
        self.tail_prot = np.zeros((U, k_group), bool)
        if v_bits < 16:
            self.v_codes = np.zeros((U, capacity, d * v_bits // 32), np.uint32)
            self.v_sz = np.zeros((U, capacity, d // v_group, 2), np.float16)
        else:
            self.v_raw = np.zeros((U, capacity, d), np.uint16)
        self.prot_count = np.zeros(U, np.int32)
        self.prot_pos = np.full((U, max(max_protected, 0)), -1, np.int32)
        self.prot_k = np.zeros((U, max(max_protected, 0), d), np.uint16)
        self.prot_gstart = np.zeros((U, nG + 1), np.int32)
        # Attention sink: the first sink_tokens positions of every sequence stay
        # in full precision (SoloQ, KV-only paragraph: at 2-bit KV, a
        # full-precision sink makes a large difference).  Reading: their K
        # is protected like any protected entry (side table), their V is kept
        # as bf16 next to the codes (which are still computed and stored).
        assert 0 <= sink_tokens <= capacity
        self.sink = int(sink_tokens)
        self.v_sink = np.zeros((U, self.sink, d), np.uint16)
        # Rotated V (K-RPBH, oracle/krpbh.py): (perm, mix, b) or None.  V rows
        # are quantized in the rotated basis; the active block's V enters the
        # attention rotated too (fp32 rotation rounded to bf16), and the
        # output is rotated back.  Needs quantized V and no sink.
        self.v_rot = None
        if v_rotation is not None:
            perm, mix, b = v_rotation
            assert v_bits < 16 and self.sink == 0
            krpbh.check_params(perm, mix, b, d)
            self.v_rot = (np.asarray(perm, np.int64), np.asarray(mix, np.float32), int(b))

    # -- derived sizes
    @property
    def n_quantized(self) -> int:
        """Tokens [0, Lq) whose K lives in quantized groups."""
        if self.kb == 16:
            return self.len
        return (self.len // self.GK) * self.GK

    @property
    def tail_mask(self) -> np.ndarray:
        return bool_to_mask_words(self.tail_prot)

    # -- commit (quantization happens here, when a block is committed)
    def commit(self, K_bits, V_bits, protect_words=None) -> int:
        """Append one block.  K_bits, V_bits: uint16 [B, Hkv, blk, d] bf16
        patterns; protect_words: uint32 [B, Hkv, ceil(blk/32)] (bit t = token
        t of the block is a protected K position) or None.  Returns the flags
        raised by this commit (also OR-ed into self.flags)."""
        B, Hkv, blk, d = self.B, self.Hkv, self.blk, self.d
        if self.len + blk > self.cap:
            raise CapacityError(f"len {self.len} + blk {blk} > capacity {self.cap}")
        K_bits = np.asarray(K_bits, np.uint16).reshape(self.U, blk, d)
        V_bits = np.asarray(V_bits, np.uint16).reshape(self.U, blk, d)
        if protect_words is None:
            prot = np.zeros((self.U, blk), bool)
        else:
            pw = np.asarray(protect_words, np.uint32).reshape(self.U, -1)
            prot = mask_words_to_bool(pw, blk)
        p0 = self.len
        # sink positions: K always protected, V kept in bf16
        ns = max(0, min(self.sink - p0, blk))
        if ns:
            prot = prot.copy()
            prot[:, :ns] = True
            self.v_sink[:, p0:p0 + ns] = V_bits[:, :ns]
        flags = 0
        for u in range(self.U):
            flags |= self._commit_v(u, p0, V_bits[u])
            flags |= self._commit_k(u, p0, K_bits[u], prot[u])
        self.len = p0 + blk
        self.flags |= flags
        return flags

    def _commit_v(self, u, p0, vbits) -> int:
        blk, d, GV, vb = self.blk, self.d, self.GV, self.vb
        x = bf16_to_f32(vbits)
        flag = FLAG_RANGE if (~np.isfinite(x) | (np.abs(x) > FP16_MAX)).any() else 0
        if vb == 16:
            self.v_raw[u, p0:p0 + blk] = vbits
            return flag
        x, _ = sanitize(x)
        if self.v_rot is not None:
            x = krpbh.rotate_f32(x, *self.v_rot)
            flag |= FLAG_RANGE if (~np.isfinite(x) | (np.abs(x) > FP16_MAX)).any() else 0
            x, _ = sanitize(x)
        # per token, one group per GV consecutive channels
        groups = x.reshape(blk * (d // GV), GV)
        q, s, z = quantize_groups(groups, np.ones_like(groups, bool), vb)
        self.v_codes[u, p0:p0 + blk] = pack_codes(q.reshape(blk, d), vb)
        self.v_sz[u, p0:p0 + blk] = np.stack([s, z], -1).reshape(blk, d // GV, 2)
        return flag

    def _commit_k(self, u, p0, kbits, prot) -> int:
        blk, d, GK, kb = self.blk, self.d, self.GK, self.kb
        x = bf16_to_f32(kbits)
        flag = FLAG_RANGE if (~np.isfinite(x) | (np.abs(x) > FP16_MAX)).any() else 0
        if kb == 16:
            self.k_raw[u, p0:p0 + blk] = kbits   # passthrough: protection has no meaning
            return flag
        # the pending stream = tokens of the incomplete group, then this block
        n_tail = p0 % GK
        pend_bits = np.concatenate([self.k_tail[u, :n_tail], kbits])
        pend_prot = np.concatenate([self.tail_prot[u, :n_tail], prot])
        start = p0 - n_tail                      # absolute position of pend[0]
        n_full = pend_bits.shape[0] // GK
        for gi in range(n_full):
            j = start // GK + gi
            gb = pend_bits[gi * GK:(gi + 1) * GK]
            gp = pend_prot[gi * GK:(gi + 1) * GK].copy()
            flag |= self._quantize_k_group(u, j, gb, gp)
        rest = pend_bits.shape[0] - n_full * GK
        self.k_tail[u, :rest] = pend_bits[n_full * GK:]
        self.tail_prot[u, :rest] = pend_prot[n_full * GK:]
        self.tail_prot[u, rest:] = False
        return flag

    def _quantize_k_group(self, u, j, gbits, gprot) -> int:
        """Quantize K group j (positions [j*GK, (j+1)*GK)) of unit u."""
        GK, kb = self.GK, self.kb
        flag = 0
        count = int(self.prot_count[u])
        want = np.nonzero(gprot)[0]
        room = self.P - count
        if want.size > room:
            # side table full: the first `room` (by position) stay protected
            flag |= FLAG_CAPACITY
            gprot[want[max(room, 0):]] = False
            want = want[:max(room, 0)]
        x, _ = sanitize(bf16_to_f32(gbits))      # [GK, d]
        keep = ~gprot                            # [GK]
        # per channel: one group over the GK tokens (KIVI per-channel)
        q, s, z = quantize_groups(x.T, keep[None, :], kb)   # q [d, GK]
        self.k_codes[u, j] = pack_codes(q, kb)
        self.k_sz[u, j] = np.stack([s, z], -1)
        for t in want:                           # ascending positions
            self.prot_pos[u, count] = j * GK + t
            self.prot_k[u, count] = gbits[t]
            count += 1
        self.prot_count[u] = count
        self.prot_gstart[u, j + 1] = count
        return flag

    # -- roll back to an earlier prefix
    def truncate(self, new_len: int) -> None:
        """Drop the committed tokens [new_len, len): new_len must be a
        multiple of the block and of the K group (so no incomplete group
        remains).  The side table keeps the entries of the surviving groups."""
        if new_len < 0 or new_len > self.len or new_len % self.blk:
            raise ValueError("new_len must be a multiple of the block within [0, len]")
        if self.kb < 16:
            if new_len % self.GK:
                raise ValueError("new_len must be a multiple of k_group")
            self.prot_count[:] = self.prot_gstart[:, new_len // self.GK]
            self.tail_prot[:] = False
        self.len = new_len

    # -- dequantization (fp64)
    def dequant_k(self, u) -> np.ndarray:
        """K_hat [len, d] fp64 of unit u: quantized groups (protected rows
        from the side table), then the bf16 tail."""
        L, d, GK = self.len, self.d, self.GK
        if self.kb == 16:
            return bf16_to_f64(self.k_raw[u, :L])
        Lq = self.n_quantized
        nG = Lq // GK
        out = np.zeros((L, d), np.float64)
        if nG:
            q = unpack_codes(self.k_codes[u, :nG], self.kb, GK).astype(np.float64)  # [nG, d, GK]
            s = self.k_sz[u, :nG, :, 0].astype(np.float64)[..., None]
            z = self.k_sz[u, :nG, :, 1].astype(np.float64)[..., None]
            out[:Lq] = (q * s + z).transpose(0, 2, 1).reshape(Lq, d)
            for i in range(int(self.prot_gstart[u, nG])):
                out[self.prot_pos[u, i]] = bf16_to_f64(self.prot_k[u, i])
        out[Lq:L] = bf16_to_f64(self.k_tail[u, :L - Lq])
        return out

    def dequant_v(self, u) -> np.ndarray:
        L, d, GV = self.len, self.d, self.GV
        if self.vb == 16:
            return bf16_to_f64(self.v_raw[u, :L])
        q = unpack_codes(self.v_codes[u, :L], self.vb, d).astype(np.float64)  # [L, d]
        q = q.reshape(L, d // GV, GV)
        s = self.v_sz[u, :L, :, 0].astype(np.float64)[..., None]
        z = self.v_sz[u, :L, :, 1].astype(np.float64)[..., None]
        v = (q * s + z).reshape(L, d)
        ns = min(self.sink, L)
        if ns:
            v[:ns] = bf16_to_f64(self.v_sink[u, :ns])
        return v

    # -- attention at one denoising step
    def block_attention(self, Q_bits, Kact_bits, Vact_bits, scale: float) -> np.ndarray:
        """O [B, Hq, blk, d] fp64 for the active block's queries over the
        committed cache plus the active block (bidirectional, no mask)."""
        B, Hq, Hkv, blk, d = self.B, self.Hq, self.Hkv, self.blk, self.d
        g = Hq // Hkv
        Q = bf16_to_f64(np.asarray(Q_bits).reshape(B, Hq, blk, d))
        Ka = bf16_to_f64(np.asarray(Kact_bits).reshape(B, Hkv, blk, d))
        Va_bits = np.asarray(Vact_bits, np.uint16).reshape(B, Hkv, blk, d)
        if self.v_rot is not None:
            Va_bits = krpbh.f32_to_bf16_bits(krpbh.rotate_f32(bf16_to_f32(Va_bits), *self.v_rot))
        Va = bf16_to_f64(Va_bits)
        O = np.zeros((B, Hq, blk, d), np.float64)
        for b in range(B):
            for h in range(Hkv):
                u = b * Hkv + h
                Kall = np.concatenate([self.dequant_k(u), Ka[b, h]])
                Vall = np.concatenate([self.dequant_v(u), Va[b, h]])
                for hq in range(h * g, (h + 1) * g):
                    O[b, hq] = dense_attention_f64(Q[b, hq], Kall, Vall, scale)
        if self.v_rot is not None:
            perm, mix, rb = self.v_rot
            O = krpbh.unrotate_f64(O, perm, mix.astype(np.float64), rb)
        return O

    def block_attention_dual(self, suffix: "OracleCache", Q_bits, Kact_bits, Vact_bits,
                             scale: float) -> np.ndarray:
        """Dual-cache attention (Fast-dLLM-style prefix and dual cache reuse,
        "KV Cache Quantization for Diffusion Language Models", abstract): the
        active block's queries attend to this (prefix) cache, the active block
        and a second cache holding the suffix region after the block, each
        cache dequantized with its own parameters; softmax over all of them
        (bidirectional, no mask).  Neither cache may rotate V; the suffix has
        no sink."""
        B, Hq, Hkv, blk, d = self.B, self.Hq, self.Hkv, self.blk, self.d
        assert (suffix.B, suffix.Hq, suffix.Hkv, suffix.blk, suffix.d) == (B, Hq, Hkv, blk, d)
        assert self.v_rot is None and suffix.v_rot is None and suffix.sink == 0
        g = Hq // Hkv
        Q = bf16_to_f64(np.asarray(Q_bits).reshape(B, Hq, blk, d))
        Ka = bf16_to_f64(np.asarray(Kact_bits).reshape(B, Hkv, blk, d))
        Va = bf16_to_f64(np.asarray(Vact_bits).reshape(B, Hkv, blk, d))
        O = np.zeros((B, Hq, blk, d), np.float64)
        for b in range(B):
            for h in range(Hkv):
                u = b * Hkv + h
                Kall = np.concatenate([self.dequant_k(u), Ka[b, h], suffix.dequant_k(u)])
                Vall = np.concatenate([self.dequant_v(u), Va[b, h], suffix.dequant_v(u)])
                for hq in range(h * g, (h + 1) * g):
                    O[b, hq] = dense_attention_f64(Q[b, hq], Kall, Vall, scale)
        return O

    def block_attention_selected(self, Q_bits, Kact_bits, Vact_bits, scale: float,
                                 budget: int, selection=None):
        """Attention over a selection of the committed entries (MaskAhead
        abstract: the mask queries of the block being denoised score every
        cached entry by how much it is expected to add to the attention
        output, and the block attends to the best-scored ones; the quantized
        variant scores and attends on the low-bit cache).  Readings (the abstract gives no
        formula): for each (sequence, kv-head) every committed entry j gets
        c_j = (sum over the group's query rows i of p_ij) * ||v_hat_j||_2,
        with p_ij the softmax weight of key j for row i over all committed
        and active keys, from the dequantized cache; the `budget` entries of
        largest c_j are kept (ties: the lower position), and every row
        attends to those entries plus the whole active block.
        `selection` (a list of position arrays, one per unit) replaces the
        ranking: the attention then runs over exactly those entries (to
        check another implementation's output on its own selection).
        Returns (O [B, Hq, blk, d] fp64, selected positions per unit, sorted,
        contributions per unit [L])."""
        B, Hq, Hkv, blk, d = self.B, self.Hq, self.Hkv, self.blk, self.d
        assert self.v_rot is None and budget >= 0
        g = Hq // Hkv
        Q = bf16_to_f64(np.asarray(Q_bits).reshape(B, Hq, blk, d))
        Ka = bf16_to_f64(np.asarray(Kact_bits).reshape(B, Hkv, blk, d))
        Va = bf16_to_f64(np.asarray(Vact_bits).reshape(B, Hkv, blk, d))
        O = np.zeros((B, Hq, blk, d), np.float64)
        selected, contribs = [], []
        L = self.len
        for b in range(B):
            for h in range(Hkv):
                u = b * Hkv + h
                Kc, Vc = self.dequant_k(u), self.dequant_v(u)
                Kall = np.concatenate([Kc, Ka[b, h]])
                Vall = np.concatenate([Vc, Va[b, h]])
                mass = np.zeros(L, np.float64)
                for hq in range(h * g, (h + 1) * g):
                    s = scale * (Q[b, hq] @ Kall.T)                  # [blk, L + blk]
                    p = np.exp(s - s.max(axis=1, keepdims=True))
                    p /= p.sum(axis=1, keepdims=True)
                    mass += p[:, :L].sum(axis=0)
                contrib = mass * np.linalg.norm(Vc, axis=1)
                contribs.append(contrib)
                if selection is not None:
                    sel = np.sort(np.asarray(selection[u], np.int64))
                else:
                    # largest first; equal contributions keep the lower position
                    order = np.lexsort((np.arange(L), -contrib))
                    sel = np.sort(order[:min(budget, L)])
                selected.append(sel)
                Ks = np.concatenate([Kc[sel], Ka[b, h]])
                Vs = np.concatenate([Vc[sel], Va[b, h]])
                for hq in range(h * g, (h + 1) * g):
                    O[b, hq] = dense_attention_f64(Q[b, hq], Ks, Vs, scale)
        return O, selected, contribs

    # -- canonical snapshot of the committed state (what an export returns)
    def snapshot(self) -> dict:
        L, GK = self.len, self.GK
        out = {"len": L, "flags": self.flags,
               "prot_count": self.prot_count.copy()}
        if self.kb < 16:
            nG = self.n_quantized // GK
            out["k_codes"] = self.k_codes[:, :nG].copy()
            out["k_sz"] = self.k_sz[:, :nG].copy()
            out["prot_gstart"] = self.prot_gstart[:, :nG + 1].copy()
            out["k_tail"] = self.k_tail[:, :L - self.n_quantized].copy()
            out["tail_mask"] = self.tail_mask.copy()
        else:
            out["k_raw"] = self.k_raw[:, :L].copy()
        if self.vb < 16:
            out["v_codes"] = self.v_codes[:, :L].copy()
            out["v_sz"] = self.v_sz[:, :L].copy()
        else:
            out["v_raw"] = self.v_raw[:, :L].copy()
        out["prot_pos"] = self.prot_pos.copy()
        out["prot_k"] = self.prot_k.copy()
        if self.sink and self.vb < 16:
            out["v_sink"] = self.v_sink[:, :min(self.sink, L)].copy()
        return out


class OracleRaggedCache:
    """Per-sequence committed lengths: each sequence of the batch commits its
    own blocks (block-diffusion sequences of one batch finish blocks at
    different steps), and each attends over its own committed tokens plus its
    active block.  Reading: the batch is B single-sequence caches with one
    shared configuration; a commit names the sequences it appends to."""

    def __init__(self, B, Hq, Hkv, d, blk, k_bits, v_bits, k_group, v_group,
                 max_protected, capacity, sink_tokens=0):
        self.B, self.Hq, self.Hkv, self.d, self.blk = B, Hq, Hkv, d, blk
        self.seqs = [OracleCache(1, Hq, Hkv, d, blk, k_bits, v_bits, k_group, v_group,
                                 max_protected, capacity, sink_tokens) for _ in range(B)]

    @property
    def lens(self) -> list:
        return [c.len for c in self.seqs]

    def commit(self, K_bits, V_bits, protect_words=None, seqs=None) -> int:
        """Append one block to the sequences listed in `seqs` (all if None);
        K_bits, V_bits [B, Hkv, blk, d], protect_words [B, Hkv, blk/32]: the
        rows of other sequences are ignored.  Returns the OR of the flags."""
        K = np.asarray(K_bits, np.uint16)
        V = np.asarray(V_bits, np.uint16)
        flags = 0
        for b in (range(self.B) if seqs is None else seqs):
            pw = None if protect_words is None else np.asarray(protect_words)[b:b + 1]
            flags |= self.seqs[b].commit(K[b:b + 1], V[b:b + 1], pw)
        return flags

    def truncate(self, b: int, new_len: int) -> None:
        self.seqs[b].truncate(new_len)

    def block_attention(self, Q_bits, Kact_bits, Vact_bits, scale: float) -> np.ndarray:
        Q = np.asarray(Q_bits, np.uint16)
        Ka = np.asarray(Kact_bits, np.uint16)
        Va = np.asarray(Vact_bits, np.uint16)
        return np.concatenate([c.block_attention(Q[b:b + 1], Ka[b:b + 1], Va[b:b + 1], scale)
                               for b, c in enumerate(self.seqs)])


def dense_attention_f64(q, K, V, scale) -> np.ndarray:
    """Textbook softmax attention in fp64: softmax_j(scale * <q_i, K_j>) V_j.
    q [n, d], K [m, d], V [m, d] -> [n, d].  Subtracting the row maximum
    leaves the softmax unchanged and keeps exp() finite."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    S = np.float64(scale) * (q @ K.T)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    return (P @ V) / P.sum(axis=1, keepdims=True)


def quantize_stream_oneshot(K_bits, V_bits, prot, k_bits, v_bits, k_group, v_group,
                            max_protected):
    """Quantize a whole token stream of ONE unit in one pass (no commits):
    K_bits, V_bits uint16 [n, d]; prot bool [n].  Returns the complete K
    groups' (codes, sz), the side table, and every token's V (codes, sz).
    Used to check that block-by-block commits give the same cache."""
    n, d = np.asarray(K_bits).shape
    GK, GV = k_group, v_group
    nG = n // GK
    kc = np.zeros((nG, d, GK * k_bits // 32), np.uint32)
    ksz = np.zeros((nG, d, 2), np.float16)
    ppos, pk = [], []
    for j in range(nG):
        gb = np.asarray(K_bits[j * GK:(j + 1) * GK])
        gp = np.asarray(prot[j * GK:(j + 1) * GK], bool).copy()
        want = np.nonzero(gp)[0]
        room = max_protected - len(ppos)
        if want.size > room:
            gp[want[max(room, 0):]] = False
            want = want[:max(room, 0)]
        x, _ = sanitize(bf16_to_f32(gb))
        q, s, z = quantize_groups(x.T, (~gp)[None, :], k_bits)
        kc[j] = pack_codes(q, k_bits)
        ksz[j] = np.stack([s, z], -1)
        for t in want:
            ppos.append(j * GK + t)
            pk.append(gb[t])
    xv, _ = sanitize(bf16_to_f32(np.asarray(V_bits)))
    groups = xv.reshape(n * (d // GV), GV)
    q, s, z = quantize_groups(groups, np.ones_like(groups, bool), v_bits)
    vc = pack_codes(q.reshape(n, d), v_bits)
    vsz = np.stack([s, z], -1).reshape(n, d // GV, 2)
    return {"k_codes": kc, "k_sz": ksz, "prot_pos": np.array(ppos, np.int32),
            "prot_k": np.array(pk, np.uint16).reshape(-1, d),
            "v_codes": vc, "v_sz": vsz}
