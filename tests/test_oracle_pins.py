"""Pins of the CPU oracle against things other than itself: hand-derived
cases, brute force, closed forms, invariants and an exact-arithmetic softmax.
CPU only."""
import decimal
import itertools
import os

import numpy as np
import pytest

from oracle import (FLAG_CAPACITY, FLAG_RANGE, CapacityError, OracleCache, bf16_to_f64,
                    bool_to_mask_words,
                    dense_attention_f64, mask_words_to_bool, pack_codes, quantize_groups,
                    quantize_stream_oneshot, to_fp16, unpack_codes)
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- fp16 rounding

def _all_finite_fp16():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = pats.view(np.float16).astype(np.float64)
    ok = np.isfinite(vals)
    return vals[ok], pats[ok]


def test_fp16_rounding_is_nearest_ties_even_bruteforce():
    vals, pats = _all_finite_fp16()
    order = np.argsort(vals, kind="stable")
    vals, pats = vals[order], pats[order]
    # drop -0 duplicate so neighbours are distinct
    keep = np.ones(len(vals), bool)
    keep[1:] = vals[1:] != vals[:-1]
    vals, pats = vals[keep], pats[keep]
    rng = np.random.default_rng(7)
    mags = np.exp(rng.uniform(np.log(2.0 ** -26), np.log(65000.0), 4000))
    x = (mags * rng.choice([-1, 1], 4000)).astype(np.float32)
    # exact midpoints between neighbours (ties) inside the normal range
    mid = ((vals[1000:1100] + vals[1001:1101]) / 2).astype(np.float32)
    x = np.concatenate([x, mid[mid.astype(np.float64) == (vals[1000:1100] + vals[1001:1101]) / 2]])
    got = to_fp16(x).astype(np.float64)
    for xi, gi in zip(x.astype(np.float64), got):
        dist = np.abs(vals - xi)
        best = np.nonzero(dist == dist.min())[0]
        if len(best) == 1:
            want = vals[best[0]]
        else:  # tie: the neighbour with an even last significand bit
            evens = [i for i in best if (int(pats[i]) & 1) == 0]
            assert len(evens) == 1
            want = vals[evens[0]]
        assert gi == want, (xi, gi, want)
    # overflow: at and beyond max + half an ulp (65520) rounds to infinity
    assert np.isinf(to_fp16(np.float32(65520.0)))
    assert to_fp16(np.float32(65519.0)) == np.float16(65504.0)


# ----------------------------------------------------------------- quantizer

def _golden_quantizer_cases():
    cases = []
    with open(os.path.join(GOLDEN, "quantizer_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            b, xs, ks, s, z, qs = [p.strip() for p in line.split("|")]
            cases.append((int(b), [float(v) for v in xs.split()],
                          [bool(int(v)) for v in ks.split()], float(s), float(z),
                          [int(v) for v in qs.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_quantizer_cases())
def test_quantizer_hand_derived_cases(case):
    bits, xs, keep, s, z, codes = case
    q, sh, zh = quantize_groups(np.array([xs], np.float32), np.array([keep]), bits)
    assert float(sh[0]) == s
    assert float(zh[0]) == z
    assert q[0].tolist() == codes


def _random_groups(rng, G, n, outliers=True):
    x = rng.standard_normal((G, n)).astype(np.float32)
    if outliers:
        x[: G // 4] *= 10
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantizer_extremes_and_error_bound(bits):
    rng = np.random.default_rng(bits)
    x = _random_groups(rng, 512, 32)
    q, s, z = quantize_groups(x, np.ones_like(x, bool), bits)
    levels = 2 ** bits - 1
    rows = np.arange(x.shape[0])
    # z is the group minimum (bf16 values in fp16's normal range convert exactly)
    assert np.all(z.astype(np.float32) == x.min(1))
    assert np.all(q[rows, x.argmin(1)] == 0)
    assert np.all(q[rows, x.argmax(1)] == levels)
    s64 = s.astype(np.float64)
    xhat = q * s64[:, None] + z.astype(np.float64)[:, None]
    s_f = (x.max(1).astype(np.float64) - x.min(1)) / levels
    ulp16 = 2.0 ** (np.floor(np.log2(s_f)) - 10)
    bound = s64 / 2 + levels * ulp16 / 2 + s64 * 2.0 ** -19
    assert np.all(np.abs(x - xhat) <= bound[:, None])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantizer_picks_nearest_code_bruteforce(bits):
    rng = np.random.default_rng(100 + bits)
    x = _random_groups(rng, 64, 32)
    keep = rng.random(x.shape) > 0.1
    keep[:, 0] = True
    q, s, z = quantize_groups(x, keep, bits)
    codes = np.arange(2 ** bits, dtype=np.float64)
    for gi in range(x.shape[0]):
        cand = codes * float(s[gi]) + float(z[gi])
        for j in range(x.shape[1]):
            if not keep[gi, j]:
                assert q[gi, j] == 0
                continue
            err = np.abs(cand - float(x[gi, j]))
            assert err[q[gi, j]] <= err.min() + float(s[gi]) * 2.0 ** -19


def test_quantizer_constant_group_is_exact():
    x = np.full((3, 32), 1.75, np.float32)
    x[1] = -0.125
    x[2] = 0.0
    q, s, z = quantize_groups(x, np.ones_like(x, bool), 4)
    assert np.all(q == 0) and np.all(s == 0)
    assert np.all(z.astype(np.float32)[:, None] == x)


def test_quantizer_exact_grid_recovered():
    """Values on a grid z0 + q*s0 (s0 a power of two) with codes 0 and
    2^b - 1 present are quantized without error."""
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        lv = 2 ** bits - 1
        q0 = rng.integers(0, lv + 1, (100, 32))
        q0[:, 0], q0[:, 1] = 0, lv
        e = rng.integers(-6, 2, 100).astype(np.float64)
        z0 = rng.integers(-40, 40, 100) * 2.0 ** e
        x = (z0[:, None] + q0 * (2.0 ** e)[:, None]).astype(np.float32)
        q, s, z = quantize_groups(x, np.ones_like(x, bool), bits)
        assert np.all(q == q0)
        assert np.all(s.astype(np.float64) == 2.0 ** e)
        assert np.all(z.astype(np.float64) == z0)


# ----------------------------------------------------------------- packing

def _golden_packing():
    out = []
    with open(os.path.join(GOLDEN, "packing_words.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            b, cs, ws = [p.strip() for p in line.split("|")]
            out.append((int(b), [int(v) for v in cs.split()], [int(v, 16) for v in ws.split()]))
    return out


@pytest.mark.parametrize("case", _golden_packing())
def test_packing_hand_derived_words(case):
    bits, codes, words = case
    got = pack_codes(np.array(codes, np.uint8), bits)
    assert got.tolist() == words
    assert unpack_codes(got, bits, len(codes)).tolist() == codes


@pytest.mark.parametrize("bits,n", [(2, 32), (2, 64), (4, 32), (4, 64), (4, 128), (3, 32),
                                    (3, 64), (3, 128)])
def test_pack_unpack_roundtrip(bits, n):
    rng = np.random.default_rng(bits * n)
    c = rng.integers(0, 2 ** bits, (7, 5, n)).astype(np.uint8)
    assert np.array_equal(unpack_codes(pack_codes(c, bits), bits, n), c)


def test_mask_words():
    w = np.array([0x80000001, 0x2], np.uint32)
    m = mask_words_to_bool(w, 64)
    assert np.nonzero(m)[0].tolist() == [0, 31, 33]


# ----------------------------------------------------------------- commit

def _cache(w, cap=None, P=None, **over):
    w = w.with_(**over) if over else w
    cap = cap if cap is not None else w.L + 4 * max(w.k_group, w.blk)
    P = P if P is not None else max(8, 2 * int(round(w.prot_frac * cap)) + 8)
    return w, OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits,
                          w.k_group, w.v_group, P, cap)


SMALL = synth.WORKLOADS["batch32"].with_(B=2, Hq=4, Hkv=2, L=256, prot_frac=0.05)


@pytest.mark.parametrize("kb,vb,gk,gv", [(4, 4, 32, 32), (2, 2, 64, 64), (2, 4, 128, 32),
                                         (4, 2, 64, 128), (3, 3, 64, 32), (3, 4, 32, 128)])
def test_incremental_commits_equal_one_shot(kb, vb, gk, gv):
    w, c = _cache(SMALL, k_bits=kb, v_bits=vb, k_group=gk, v_group=gv)
    n_blocks = w.L // w.blk + 1          # ends with an incomplete K group when gk > blk
    per_unit = {}
    for i in range(n_blocks):
        K, V, M = synth.block_inputs(w, i)
        c.commit(K, V, M)
        for b in range(w.B):
            for h in range(w.Hkv):
                per_unit.setdefault((b, h), []).append((K[b, h], V[b, h], M[b, h]))
    snap = c.snapshot()
    for (b, h), blocks in per_unit.items():
        u = b * w.Hkv + h
        Ks = np.concatenate([x[0] for x in blocks])
        Vs = np.concatenate([x[1] for x in blocks])
        prot = np.concatenate([mask_words_to_bool(x[2], w.blk) for x in blocks])
        ref = quantize_stream_oneshot(Ks, Vs, prot, kb, vb, gk, gv, c.P)
        nG = ref["k_codes"].shape[0]
        assert np.array_equal(snap["k_codes"][u], ref["k_codes"])
        assert np.array_equal(snap["k_sz"][u].view(np.uint16), ref["k_sz"].view(np.uint16))
        assert np.array_equal(snap["v_codes"][u], ref["v_codes"])
        assert np.array_equal(snap["v_sz"][u].view(np.uint16), ref["v_sz"].view(np.uint16))
        n = int(snap["prot_count"][u])
        assert np.array_equal(snap["prot_pos"][u, :n], ref["prot_pos"])
        assert np.array_equal(snap["prot_k"][u, :n], ref["prot_k"])
        # the tail holds the incomplete group's bf16 K verbatim
        assert np.array_equal(snap["k_tail"][u], Ks[nG * gk:])


def test_protected_entries_exact_and_excluded():
    w, c = _cache(SMALL, k_bits=4, v_bits=4, k_group=32, v_group=32)
    K, V, M = synth.block_inputs(w, 0)
    c.commit(K, V, M)
    prot = mask_words_to_bool(M.reshape(w.B * w.Hkv, -1), w.blk)
    snap = c.snapshot()
    for u in range(w.B * w.Hkv):
        want = np.nonzero(prot[u])[0]
        assert snap["prot_count"][u] == len(want)
        assert snap["prot_pos"][u, :len(want)].tolist() == want.tolist()
        Ku = K.reshape(w.B * w.Hkv, w.blk, w.d)[u]
        assert np.array_equal(snap["prot_k"][u, :len(want)], Ku[want])
        # protected slot codes are 0 in every channel
        codes = unpack_codes(snap["k_codes"][u, 0], 4, 32)     # [d, 32]
        assert np.all(codes[:, want] == 0)
        # dequantized K reproduces protected rows exactly
        kh = c.dequant_k(u)
        assert np.array_equal(kh[want], bf16_to_f64(Ku[want]))
    # changing the protected tokens' K values changes nothing else
    K2 = K.copy().reshape(w.B * w.Hkv, w.blk, w.d)
    for u in range(w.B * w.Hkv):
        K2[u, prot[u]] = synth.f32_to_bf16_bits(np.full((prot[u].sum(), w.d), 1000.0, np.float32))
    _, c2 = _cache(SMALL, k_bits=4, v_bits=4, k_group=32, v_group=32)
    c2.commit(K2.reshape(K.shape), V, M)
    s2 = c2.snapshot()
    assert np.array_equal(snap["k_codes"], s2["k_codes"])
    assert np.array_equal(snap["k_sz"].view(np.uint16), s2["k_sz"].view(np.uint16))


def test_all_protected_group_has_zero_scale_and_zero():
    w, c = _cache(SMALL.with_(B=1, Hkv=1, Hq=1), k_bits=2, v_bits=2, k_group=32, v_group=32, P=64)
    K, V, _ = synth.block_inputs(w, 0)
    M = np.full((1, 1, 1), 0xFFFFFFFF, np.uint32)
    c.commit(K, V, M)
    assert np.all(c.k_sz[0, 0] == 0) and np.all(c.k_codes[0, 0] == 0)
    assert np.array_equal(c.dequant_k(0), bf16_to_f64(K[0, 0]))


def test_side_table_overflow_keeps_first_and_flags():
    w = SMALL.with_(B=1, Hkv=1, Hq=1)
    K, V, _ = synth.block_inputs(w, 0)
    want = [1, 5, 9, 20, 30]
    M = synth.positions_to_mask(want, 32).reshape(1, 1, 1)
    _, c = _cache(w, k_bits=4, v_bits=4, k_group=32, v_group=32, P=3)
    f = c.commit(K, V, M)
    assert f & FLAG_CAPACITY
    assert c.prot_pos[0, :3].tolist() == [1, 5, 9]
    # the excess tokens are quantized as if never protected
    _, c_ref = _cache(w, k_bits=4, v_bits=4, k_group=32, v_group=32, P=3)
    c_ref.commit(K, V, synth.positions_to_mask([1, 5, 9], 32).reshape(1, 1, 1))
    assert np.array_equal(c.k_codes, c_ref.k_codes)
    assert np.array_equal(c.k_sz.view(np.uint16), c_ref.k_sz.view(np.uint16))
    assert c_ref.flags == 0


def test_capacity_error_leaves_state():
    w, c = _cache(SMALL, cap=64)
    for i in range(2):
        c.commit(*synth.block_inputs(w, i))
    before = c.snapshot()
    with pytest.raises(CapacityError):
        c.commit(*synth.block_inputs(w, 2))
    after = c.snapshot()
    assert before["len"] == after["len"] == 64
    assert np.array_equal(before["v_codes"], after["v_codes"])


def test_range_flag_and_clamp():
    w, c = _cache(SMALL.with_(B=1, Hkv=1, Hq=1), k_bits=4, v_bits=4, k_group=32, v_group=32)
    K, V, _ = synth.block_inputs(w, 0)
    V = V.copy()
    V[0, 0, 3, 7] = synth.f32_to_bf16_bits(np.array([1e6], np.float32))[0]
    f = c.commit(K, V, None)
    assert f & FLAG_RANGE
    vh = c.dequant_v(0)
    # the value was clamped to the fp16 maximum before quantization
    assert np.all(np.isfinite(vh))
    assert abs(vh[3, 7] - 65504.0) <= float(c.v_sz[0, 3, 0, 0]) / 2 + 16


# ----------------------------------------------------------------- attention

def _decimal_attention(q, K, V, scale):
    """Softmax attention in 40-digit decimal arithmetic, loops only."""
    ctx = decimal.Context(prec=40)
    D = lambda v: decimal.Decimal(float(v))  # noqa: E731
    out = []
    for qi in q:
        logits = [ctx.multiply(D(scale), sum((ctx.multiply(D(a), D(b)) for a, b in zip(qi, kj)),
                                             decimal.Decimal(0))) for kj in K]
        m = max(logits)
        e = [ctx.exp(ctx.subtract(x, m)) for x in logits]
        tot = sum(e, decimal.Decimal(0))
        row = []
        for c in range(len(V[0])):
            num = sum((ctx.multiply(ei, D(V[j][c])) for j, ei in enumerate(e)), decimal.Decimal(0))
            row.append(float(ctx.divide(num, tot)))
        out.append(row)
    return np.array(out)


def test_dense_attention_matches_exact_arithmetic():
    rng = np.random.default_rng(11)
    for (n, m, d) in [(1, 1, 1), (2, 5, 3), (3, 7, 4)]:
        q = rng.standard_normal((n, d)) * 3
        K = rng.standard_normal((m, d))
        V = rng.standard_normal((m, d))
        got = dense_attention_f64(q, K, V, 0.7)
        want = _decimal_attention(q, K, V, 0.7)
        assert np.allclose(got, want, rtol=0, atol=1e-13)


def _filled(w, n_blocks, **over):
    w, c = _cache(w, **over)
    for i in range(n_blocks):
        c.commit(*synth.block_inputs(w, i))
    return w, c


def test_passthrough_equals_dense_attention():
    w, c = _filled(SMALL, 5, k_bits=16, v_bits=16)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    O = c.block_attention(Q, Ka, Va, w.softmax_scale)
    g = w.Hq // w.Hkv
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // g
            Ks = np.concatenate([synth.unit_kv_bits(w, b, h, 5 * w.blk)[0], Ka[b, h]])
            Vs = np.concatenate([synth.unit_kv_bits(w, b, h, 5 * w.blk)[1], Va[b, h]])
            ref = _decimal_attention(bf16_to_f64(Q[b, hq, :2]), bf16_to_f64(Ks), bf16_to_f64(Vs),
                                     w.softmax_scale) if (b, hq) == (0, 0) else \
                dense_attention_f64(bf16_to_f64(Q[b, hq]), bf16_to_f64(Ks), bf16_to_f64(Vs),
                                    w.softmax_scale)
            rows = ref.shape[0]
            assert np.allclose(O[b, hq, :rows], ref, rtol=0, atol=1e-12)


def _grid_block(rng, blk, d, bits, GK, GV, prot_rows):
    """K with every (group, channel) on a grid z0 + q*2^e (codes 0 and 2^b-1
    present among non-protected tokens) and V with every (token, channel
    group) on such a grid: quantization is then lossless."""
    lv = 2 ** bits - 1
    K = np.zeros((blk, d))
    keep = np.ones(blk, bool)
    keep[prot_rows] = False
    kidx = np.nonzero(keep)[0]
    for g0 in range(0, blk, GK):
        for ch in range(d):
            e = rng.integers(-4, 1)
            q = rng.integers(0, lv + 1, GK)
            ks = [i - g0 for i in kidx if g0 <= i < g0 + GK]
            q[ks[0]], q[ks[1]] = 0, lv
            z0 = rng.integers(-30, 30)
            K[g0:g0 + GK, ch] = (z0 + q) * 2.0 ** e
    for r in prot_rows:
        K[r] = rng.standard_normal(d) * 5
    V = np.zeros((blk, d))
    for t in range(blk):
        for c0 in range(0, d, GV):
            e = rng.integers(-4, 1)
            q = rng.integers(0, lv + 1, GV)
            q[0], q[-1] = 0, lv
            V[t, c0:c0 + GV] = (rng.integers(-30, 30) + q) * 2.0 ** e
    return synth.f32_to_bf16_bits(K.astype(np.float32)), synth.f32_to_bf16_bits(V.astype(np.float32))


@pytest.mark.parametrize("bits,GK,GV", [(4, 32, 32), (2, 32, 64), (2, 32, 32), (4, 32, 128),
                                        (3, 32, 32), (3, 32, 128)])
def test_grid_exact_cache_attention_equals_dense(bits, GK, GV):
    """Commit + dequant + attention in quantized mode equal dense attention
    over the original K/V when the inputs sit on each group's grid."""
    rng = np.random.default_rng(bits * GK + GV)
    B, Hq, Hkv, d, blk = 1, 4, 2, 128, 32
    nb = 4
    c = OracleCache(B, Hq, Hkv, d, blk, bits, bits, GK, GV, 16, 256)
    allK = [[[] for _ in range(Hkv)] for _ in range(B)]
    allV = [[[] for _ in range(Hkv)] for _ in range(B)]
    for i in range(nb):
        K = np.zeros((B, Hkv, blk, d), np.uint16)
        V = np.zeros_like(K)
        M = np.zeros((B, Hkv, 1), np.uint32)
        for h in range(Hkv):
            prot = [3 + h, 17] if i % 2 == 0 else []
            K[0, h], V[0, h] = _grid_block(rng, blk, d, bits, GK, GV, prot)
            M[0, h] = synth.positions_to_mask(prot, blk)
            allK[0][h].append(K[0, h])
            allV[0][h].append(V[0, h])
        c.commit(K, V, M)
    Q = synth.f32_to_bf16_bits(rng.standard_normal((B, Hq, blk, d)).astype(np.float32))
    Ka = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, blk, d)).astype(np.float32))
    Va = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, blk, d)).astype(np.float32))
    O = c.block_attention(Q, Ka, Va, 0.09)
    for hq in range(Hq):
        h = hq // 2
        Ks = np.concatenate(allK[0][h] + [Ka[0, h]])
        Vs = np.concatenate(allV[0][h] + [Va[0, h]])
        ref = dense_attention_f64(bf16_to_f64(Q[0, hq]), bf16_to_f64(Ks), bf16_to_f64(Vs), 0.09)
        assert np.allclose(O[0, hq], ref, rtol=0, atol=1e-12)


def test_grid_exact_with_64_token_groups_and_tail():
    """Same as above with K groups of 64 spanning two commits, ending with
    a 32-token bf16 tail."""
    rng = np.random.default_rng(64)
    B, Hq, Hkv, d, blk, GK, GV, bits = 1, 2, 1, 128, 32, 64, 32, 2
    c = OracleCache(B, Hq, Hkv, d, blk, bits, bits, GK, GV, 16, 256)
    Kg, Vg = _grid_block(rng, 192, d, bits, GK, GV, [5, 70, 130])
    prot = np.zeros(192, bool)
    prot[[5, 70, 130]] = True
    for i in range(6):
        sl = slice(32 * i, 32 * (i + 1))
        M = synth.positions_to_mask(np.nonzero(prot[sl])[0], 32).reshape(1, 1, 1)
        c.commit(Kg[sl].reshape(1, 1, 32, d), Vg[sl].reshape(1, 1, 32, d), M)
    Kt, Vt = _grid_block(rng, 32, d, bits, 32, GV, [])
    c.commit(Kt.reshape(1, 1, 32, d), Vt.reshape(1, 1, 32, d), None)   # stays in the tail
    assert c.n_quantized == 192 and c.len == 224
    Q = synth.f32_to_bf16_bits(rng.standard_normal((B, Hq, blk, d)).astype(np.float32))
    Ka = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, blk, d)).astype(np.float32))
    Va = synth.f32_to_bf16_bits(rng.standard_normal((B, Hkv, blk, d)).astype(np.float32))
    O = c.block_attention(Q, Ka, Va, 0.09)
    Ks = np.concatenate([Kg, Kt, Ka[0, 0]])
    Vs = np.concatenate([Vg, Vt, Va[0, 0]])
    for hq in range(Hq):
        ref = dense_attention_f64(bf16_to_f64(Q[0, hq]), bf16_to_f64(Ks), bf16_to_f64(Vs), 0.09)
        assert np.allclose(O[0, hq], ref, rtol=0, atol=1e-12)


def test_empty_cache_attends_active_block_only():
    w, c = _filled(SMALL, 0)
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    O = c.block_attention(Q, Ka, Va, w.softmax_scale)
    g = w.Hq // w.Hkv
    for b, hq in itertools.product(range(w.B), range(w.Hq)):
        ref = dense_attention_f64(bf16_to_f64(Q[b, hq]), bf16_to_f64(Ka[b, hq // g]),
                                  bf16_to_f64(Va[b, hq // g]), w.softmax_scale)
        assert np.allclose(O[b, hq], ref, rtol=0, atol=1e-13)


def test_zero_queries_give_mean_of_values():
    w, c = _filled(SMALL, 6)
    Q = np.zeros((w.B, w.Hq, w.blk, w.d), np.uint16)
    Ka, Va = synth.active_block_bits(w, 2)
    O = c.block_attention(Q, Ka, Va, w.softmax_scale)
    g = w.Hq // w.Hkv
    for b, hq in itertools.product(range(w.B), range(w.Hq)):
        u = b * w.Hkv + hq // g
        allv = np.concatenate([c.dequant_v(u), bf16_to_f64(Va[b, hq // g])])
        assert np.allclose(O[b, hq], allv.mean(0)[None, :], rtol=0, atol=1e-12)


def test_constant_values_give_constant_output():
    w, c = _cache(SMALL)
    cval = synth.f32_to_bf16_bits(np.float32(-0.6875))
    for i in range(5):
        K, V, M = synth.block_inputs(w, i)
        c.commit(K, np.full_like(V, cval), M)
    Q = synth.queries_bits(w, 3)
    Ka, _ = synth.active_block_bits(w, 3)
    O = c.block_attention(Q, Ka, np.full_like(Ka, cval), w.softmax_scale)
    assert np.allclose(O, -0.6875, rtol=0, atol=1e-13)


def test_permuting_whole_groups_leaves_output():
    w, c = _filled(SMALL.with_(k_group=32), 6)
    Q = synth.queries_bits(w, 4)
    Ka, Va = synth.active_block_bits(w, 4)
    O = c.block_attention(Q, Ka, Va, w.softmax_scale)
    # rebuild the committed stream with K-groups (and their V rows) permuted
    perm = [3, 0, 5, 1, 4, 2]
    _, c2 = _cache(SMALL.with_(k_group=32))
    for i in perm:
        c2.commit(*synth.block_inputs(w, i))
    O2 = c2.block_attention(Q, Ka, Va, w.softmax_scale)
    assert np.allclose(O, O2, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_replicated_kv():
    w = SMALL.with_(B=1, Hq=4, Hkv=2)
    _, c = _cache(w)
    w4 = w.with_(Hkv=4)
    _, c4 = _cache(w4)
    for i in range(5):
        K, V, M = synth.block_inputs(w, i)
        c.commit(K, V, M)
        rep = [0, 0, 1, 1]
        c4.commit(K[:, rep], V[:, rep], M[:, rep])
    Q = synth.queries_bits(w, 5)
    Ka, Va = synth.active_block_bits(w, 5)
    O = c.block_attention(Q, Ka, Va, 0.1)
    O4 = c4.block_attention(Q, Ka[:, [0, 0, 1, 1]], Va[:, [0, 0, 1, 1]], 0.1)
    assert np.array_equal(O, O4)


def test_quantized_attention_uses_dequantized_cache():
    """Quantized attention equals dense attention over K_hat, V_hat built
    here from the stored codes with x_hat = q*s + z (per-channel K groups,
    per-token V groups) and the side table's rows."""
    w, c = _filled(SMALL.with_(k_group=64, v_group=32, k_bits=2, v_bits=4), 5)
    Q = synth.queries_bits(w, 6)
    Ka, Va = synth.active_block_bits(w, 6)
    O = c.block_attention(Q, Ka, Va, w.softmax_scale)
    u, b, h = 1, 0, 1
    n_q = c.n_quantized
    khat = np.zeros((c.len, w.d))
    for j in range(n_q // 64):
        for ch in range(w.d):
            codes = unpack_codes(c.k_codes[u, j, ch], 2, 64)
            s, z = c.k_sz[u, j, ch]
            khat[64 * j:64 * j + 64, ch] = codes * float(s) + float(z)
    for i in range(c.prot_count[u]):
        khat[c.prot_pos[u, i]] = bf16_to_f64(c.prot_k[u, i])
    khat[n_q:] = bf16_to_f64(c.k_tail[u, :c.len - n_q])
    vhat = np.zeros((c.len, w.d))
    for t in range(c.len):
        codes = unpack_codes(c.v_codes[u, t], 4, w.d)
        for g0 in range(w.d // 32):
            s, z = c.v_sz[u, t, g0]
            vhat[t, 32 * g0:32 * g0 + 32] = codes[32 * g0:32 * g0 + 32] * float(s) + float(z)
    g = w.Hq // w.Hkv
    for hq in range(h * g, h * g + g):
        ref = dense_attention_f64(bf16_to_f64(Q[b, hq]),
                                  np.concatenate([khat, bf16_to_f64(Ka[b, h])]),
                                  np.concatenate([vhat, bf16_to_f64(Va[b, h])]),
                                  w.softmax_scale)
        assert np.allclose(O[b, hq], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("gk", [32, 64])
def test_truncate_then_recommit_equals_fresh_cache(gk):
    """Rolling back to a prefix and committing new blocks gives the same
    state as committing prefix + new blocks into an empty cache."""
    w = SMALL.with_(k_group=gk, prot_frac=0.1)
    _, c = _cache(w)
    for i in range(7):
        c.commit(*synth.block_inputs(w, i))
    c.truncate(128)
    for i in (9, 10, 11):
        c.commit(*synth.block_inputs(w, i))
    _, f = _cache(w)
    for i in (0, 1, 2, 3, 9, 10, 11):
        f.commit(*synth.block_inputs(w, i))
    a, b = c.snapshot(), f.snapshot()
    for key in ("k_codes", "v_codes", "k_tail", "tail_mask", "prot_count", "prot_gstart"):
        assert np.array_equal(a[key], b[key]), key
    for u in range(c.U):
        n = int(b["prot_count"][u])
        assert np.array_equal(a["prot_pos"][u, :n], b["prot_pos"][u, :n])
        assert np.array_equal(a["prot_k"][u, :n], b["prot_k"][u, :n])
    with pytest.raises(ValueError):
        c.truncate(32 if gk == 64 else 33)


# -- attention sink (positions [0, sink) kept in full precision)

@pytest.mark.parametrize("sink,kb,gk", [(1, 4, 32), (5, 2, 64), (40, 4, 32), (96, 2, 32)])
def test_sink_rows_exact_in_k_and_v(sink, kb, gk):
    """Sink positions come back bit-exact in both K and V; V rows past the
    sink are the quantized ones; K statistics leave the sink out exactly as
    an explicit protection mask does."""
    w = SMALL.with_(B=1, Hkv=2, Hq=2, prot_frac=0.0)
    cap = 256
    c = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, kb, kb, gk, 32, 128, cap, sink_tokens=sink)
    ref = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, kb, kb, gk, 32, 128, cap)
    nblk = 4
    Ks, Vs = [], []
    for i in range(nblk):
        K, V, _ = synth.block_inputs(w, i)
        Ks.append(K.reshape(2, w.blk, w.d))
        Vs.append(V.reshape(2, w.blk, w.d))
        c.commit(K, V, None)
        # the same tokens protected explicitly in the reference cache
        pos = np.arange(i * w.blk, (i + 1) * w.blk)
        prot = np.broadcast_to(pos < sink, (2, w.blk))
        ref.commit(K, V, bool_to_mask_words(prot).reshape(1, 2, -1))
    Kall, Vall = np.concatenate(Ks, 1), np.concatenate(Vs, 1)   # [U, L, d]
    ns = min(sink, nblk * w.blk)
    sa, sr = c.snapshot(), ref.snapshot()
    for key in ("k_codes", "prot_count", "prot_gstart", "prot_pos", "prot_k", "v_codes"):
        assert np.array_equal(sa[key], sr[key]), key
    for u in range(2):
        assert sa["prot_pos"][u, :ns].tolist() == list(range(ns))
        assert np.array_equal(c.dequant_k(u)[:ns], bf16_to_f64(Kall[u, :ns]))
        vh = c.dequant_v(u)
        assert np.array_equal(vh[:ns], bf16_to_f64(Vall[u, :ns]))
        # past the sink V is the quantized value, as without a sink
        assert np.array_equal(vh[ns:], ref.dequant_v(u)[ns:])
        assert np.array_equal(sa["v_sink"][u], Vall[u, :ns])


def test_sink_survives_truncation_and_recommit():
    w = SMALL.with_(B=1, Hkv=1, Hq=1, prot_frac=0.0)
    c = OracleCache(1, 1, 1, w.d, w.blk, 2, 2, 32, 32, 64, 256, sink_tokens=48)
    blocks = [synth.block_inputs(w, i) for i in range(6)]
    for K, V, _ in blocks[:3]:
        c.commit(K, V, None)
    c.truncate(32)
    K5, V5, _ = blocks[5]
    c.commit(K5, V5, None)     # positions 32..63: 32..47 are sink positions again
    vh = c.dequant_v(0)
    assert np.array_equal(vh[:32], bf16_to_f64(blocks[0][1].reshape(w.blk, w.d)))
    assert np.array_equal(vh[32:48], bf16_to_f64(V5.reshape(w.blk, w.d)[:16]))
    assert c.snapshot()["prot_pos"][0, :48].tolist() == list(range(48))


# ------------------------------------------------------------ K-RPBH rotated V

from oracle import krpbh  # noqa: E402


def _perm_and_mix(seed, b, dyadic=False):
    """A permutation and an orthogonal mix for the pins: Haar (fp64, from
    this test's own QR) or, dyadic=True, a non-symmetric permutation matrix
    (every fp32 step stays exact)."""
    r = np.random.default_rng(seed)
    k = 128 // b
    perm = r.permutation(128)
    if dyadic:
        mix = np.roll(np.eye(k), 1, axis=1) if k > 1 else np.eye(1)
    else:
        q, rr = np.linalg.qr(r.standard_normal((k, k)))
        mix = q * np.sign(np.diag(rr))[None, :]
    return perm, mix


@pytest.mark.parametrize("b", [1, 2, 4, 16, 32, 64, 128])
def test_hadamard_matches_scipy(b):
    import scipy.linalg
    assert np.array_equal(krpbh.hadamard_f64(b), scipy.linalg.hadamard(b).astype(np.float64))


def test_krpbh_with_one_block_is_scaled_hadamard_of_permuted_vector():
    """k = 1 (b = d): the map is plain RPBH, x[perm] @ H_d / sqrt(d)."""
    import scipy.linalg
    perm, _ = _perm_and_mix(3, 128)
    x = np.random.default_rng(4).standard_normal((5, 128))
    want = x[:, perm] @ scipy.linalg.hadamard(128) / np.sqrt(128)
    np.testing.assert_allclose(krpbh.rotate_f64(x, perm, np.eye(1), 128), want, atol=1e-12)
    np.testing.assert_allclose(krpbh.rotate_f64(x, perm, -np.eye(1), 128), -want, atol=1e-12)


def test_krpbh_block_structure_against_scipy():
    """Identity permutation and a block-swapping mix: output block r is the
    scaled Hadamard of input block sigma(r), with w_r = sum_c mix[r, c] y_c."""
    import scipy.linalg
    b, k = 32, 4
    mix = np.zeros((k, k))
    sigma = [2, 0, 3, 1]
    for r, c in enumerate(sigma):
        mix[r, c] = 1.0
    x = np.random.default_rng(5).standard_normal(128)
    H = scipy.linalg.hadamard(b) / np.sqrt(b)
    want = np.concatenate([x[c * b:(c + 1) * b] @ H for c in sigma])
    np.testing.assert_allclose(krpbh.rotate_f64(x, np.arange(128), mix, b), want, atol=1e-12)


@pytest.mark.parametrize("b", [16, 32, 64, 128])
def test_krpbh_is_orthogonal_and_inverted(b):
    perm, mix = _perm_and_mix(b, b)
    R = krpbh.rotation_matrix_f64(perm, mix, b)
    np.testing.assert_allclose(R @ R.T, np.eye(128), atol=1e-12)
    x = np.random.default_rng(6).standard_normal((7, 128))
    np.testing.assert_allclose(krpbh.rotate_f64(x, perm, mix, b), x @ R, atol=1e-12)
    np.testing.assert_allclose(krpbh.unrotate_f64(krpbh.rotate_f64(x, perm, mix, b), perm, mix, b),
                               x, atol=1e-12)
    # norms are kept, and energy in one coordinate spreads over all blocks
    e = np.zeros(128)
    e[int(perm[0])] = 1.0
    w = krpbh.rotate_f64(e, perm, mix, b)
    assert abs(np.linalg.norm(w) - 1.0) < 1e-12
    assert np.count_nonzero(np.abs(w) > 1e-12) == b * np.count_nonzero(np.abs(mix[:, 0]) > 1e-12)


@pytest.mark.parametrize("b", [4, 16, 64])
def test_krpbh_f32_order_exact_on_dyadic_inputs(b):
    """Small-integer inputs, 1/sqrt(b) a power of two and a permutation mix:
    no fp32 step rounds, so the fp32 evaluation equals the fp64 map exactly
    (a wrong butterfly index, sign or mix orientation would show)."""
    perm, mix = _perm_and_mix(b + 1, b, dyadic=True)
    x = np.random.default_rng(b).integers(-8, 9, (9, 128)).astype(np.float32)
    got = krpbh.rotate_f32(x, perm, mix, b)
    assert np.array_equal(got.astype(np.float64), krpbh.rotate_f64(x, perm, mix, b))


@pytest.mark.parametrize("b", [16, 32, 64, 128])
def test_krpbh_f32_close_to_f64(b):
    perm, mix = synth.krpbh_params(11, b)
    x = np.random.default_rng(12).standard_normal((16, 128)).astype(np.float32) * 3
    got = krpbh.rotate_f32(x, perm, mix, b).astype(np.float64)
    want = krpbh.rotate_f64(x.astype(np.float64), perm, mix.astype(np.float64), b)
    assert np.abs(got - want).max() < 2e-5


def test_f32_to_bf16_is_nearest_ties_even_bruteforce():
    r = np.random.default_rng(13)
    x = np.concatenate([r.standard_normal(4000).astype(np.float32) * 10,
                        # exact ties between two bf16 neighbours
                        (bf16_to_f64(np.arange(0x3F00, 0x3F40, dtype=np.uint16)) * (1 + 2.0 ** -8))
                        .astype(np.float32)])
    got = bf16_to_f64(krpbh.f32_to_bf16_bits(x))
    cand = bf16_to_f64(np.arange(0, 0x7F80, dtype=np.uint16))
    cand = np.concatenate([cand, -cand])
    for xi, gi in zip(x.astype(np.float64), got):
        dist = np.abs(cand - xi)
        best = dist.min()
        near = cand[dist == best]
        assert abs(gi - xi) == best
        if near.size > 1:  # tie: the even mantissa wins
            gb = krpbh.f32_to_bf16_bits(np.array([gi], np.float32))
            assert int(gb[0]) % 2 == 0


@pytest.mark.parametrize("vb,GV", [(4, 32), (2, 32), (4, 64), (2, 128)])
def test_rotated_v_cache_exact_on_grid_equals_dense(vb, GV):
    """Rotated rows built on the quantization grid (one nonzero per 16-channel
    block, the group's largest at levels * s with s a power of two, zero
    point 0), V = R^-1(w) exact in bf16, a permutation mix and b = 16: every
    step is exact, so the rotated cache's attention equals textbook dense
    attention over the unrotated V (K passthrough)."""
    b, d, blk = 16, 128, 32
    perm, mix = _perm_and_mix(21, b, dyadic=True)
    levels = 2 ** vb - 1
    r = np.random.default_rng(22)

    def rows(n):
        w = np.zeros((n, d))
        per = GV // b                          # nonzeros per V group
        for t in range(n):
            s = 2.0 ** int(r.integers(-3, 2))
            for g in range(d // GV):
                vals = r.integers(0, levels + 1, per).astype(np.float64)
                vals[0] = levels
                w[t, g * GV:(g + 1) * GV:b] = vals * s
        v = krpbh.unrotate_f64(w, perm, mix, b)
        bits = krpbh.f32_to_bf16_bits(v.astype(np.float32))
        assert np.array_equal(bf16_to_f64(bits), v)   # exact in bf16
        return bits

    n_blocks = 4
    oc = OracleCache(1, 2, 1, d, blk, 16, vb, 32, GV, 0, n_blocks * blk + blk,
                     v_rotation=(perm, mix, b))
    Ks, Vs = [], []
    for i in range(n_blocks):
        K = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
        V = rows(blk).reshape(1, 1, blk, d)
        oc.commit(K, V)
        Ks.append(K)
        Vs.append(V)
    Ka = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
    Va = rows(blk).reshape(1, 1, blk, d)
    Q = synth.f32_to_bf16_bits(r.standard_normal((1, 2, blk, d)).astype(np.float32))
    got = oc.block_attention(Q, Ka, Va, 0.1)
    Kall = bf16_to_f64(np.concatenate(Ks + [Ka], 2)[0, 0])
    Vall = bf16_to_f64(np.concatenate(Vs + [Va], 2)[0, 0])
    for h in range(2):
        want = dense_attention_f64(bf16_to_f64(Q[0, h]), Kall, Vall, 0.1)
        np.testing.assert_allclose(got[0, h], want, atol=1e-12)


def test_rotated_v_cache_stores_codes_of_rotated_rows():
    """The committed codes are the quantizer applied to the fp32-rotated rows."""
    w = synth.WORKLOADS["tiny"]
    perm, mix = synth.krpbh_params(0, 32)
    oc = OracleCache(1, 4, 1, 128, 32, 4, 2, 32, 64, 0, 64, v_rotation=(perm, mix, 32))
    K, V, _ = synth.block_inputs(w, 0)
    oc.commit(K, V)
    x = krpbh.rotate_f32(bf16_to_f64(V[0, 0]).astype(np.float32), perm, mix, 32)
    q, s, z = quantize_groups(x.reshape(-1, 64), np.ones((64, 64), bool), 2)
    assert np.array_equal(oc.v_codes[0, :32], pack_codes(q.reshape(32, 128), 2))
    assert np.array_equal(oc.v_sz[0, :32, :, 0].view(np.uint16), s.reshape(32, 2).view(np.uint16))
    assert np.array_equal(oc.v_sz[0, :32, :, 1].view(np.uint16), z.reshape(32, 2).view(np.uint16))


@pytest.mark.parametrize("seed", [31, 7])
def test_rotation_spreads_v_outliers(seed):
    """What the rotation is for: V rows with a few large channels (4 of 128,
    x50) lose less to per-token 4-bit quantization over whole-row groups in
    the rotated basis, where the outliers no longer set every group's range
    (K passthrough, so only V quantization separates the two caches from the
    exact output).  Measured ratio about 0.4; narrow groups gain less."""
    r = np.random.default_rng(seed)
    d, blk, nb = 128, 32, 6
    perm, mix = synth.krpbh_params(5, 32)
    out_ch = r.choice(d, 4, replace=False)
    caches = [OracleCache(1, 4, 1, d, blk, 16, 4, 32, 128, 0, nb * blk + blk,
                          v_rotation=rot) for rot in (None, (perm, mix, 32))]
    Ks, Vs = [], []
    for i in range(nb):
        K = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
        v = r.standard_normal((1, 1, blk, d))
        v[..., out_ch] *= 50.0
        V = synth.f32_to_bf16_bits(v.astype(np.float32))
        for c in caches:
            c.commit(K, V)
        Ks.append(K)
        Vs.append(V)
    Q = synth.f32_to_bf16_bits(r.standard_normal((1, 4, blk, d)).astype(np.float32))
    Ka, Va = Ks[0], Vs[0]
    Kall = bf16_to_f64(np.concatenate(Ks + [Ka], 2)[0, 0])
    Vall = bf16_to_f64(np.concatenate(Vs + [Va], 2)[0, 0])
    want = np.stack([dense_attention_f64(bf16_to_f64(Q[0, h]), Kall, Vall, 1 / np.sqrt(d))
                     for h in range(4)])
    err = [np.abs(c.block_attention(Q, Ka, Va, 1 / np.sqrt(d))[0] - want).mean() for c in caches]
    assert err[1] < 0.6 * err[0], err


# ------------------------------------------------------------ dual cache

def _dual_setup(kb=4, vb=4, gk=32, gv=32, nA=4, nB=3, prot=0.03):
    w = synth.WORKLOADS["tiny"].with_(Hq=4, Hkv=2, k_bits=kb, v_bits=vb, k_group=gk,
                                      v_group=gv, prot_frac=prot, seed=9)
    mk = lambda cap: OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, kb, vb, gk, gv, 64, cap)
    blocks = [synth.block_inputs(w, i) for i in range(nA + nB)]
    return w, mk, blocks[:nA], blocks[nA:]


def test_dual_with_empty_suffix_is_single_cache_attention():
    w, mk, A, _ = _dual_setup()
    pre, suf = mk(256), mk(128)
    for K, V, M in A:
        pre.commit(K, V, M)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    assert np.array_equal(pre.block_attention_dual(suf, Q, Ka, Va, 0.1),
                          pre.block_attention(Q, Ka, Va, 0.1))


def test_dual_equals_one_cache_holding_both_regions():
    """K groups of one block (GK = blk): each block quantizes on its own, so a
    suffix cache holding blocks X gives the same dequantized keys and values as
    appending X to the prefix; softmax attention does not depend on key order."""
    w, mk, A, X = _dual_setup(kb=2, vb=4, gk=32, gv=64)
    pre, suf, one = mk(256), mk(128), mk(384)
    for K, V, M in A:
        pre.commit(K, V, M)
        one.commit(K, V, M)
    for K, V, M in X:
        suf.commit(K, V, M)
        one.commit(K, V, M)
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    np.testing.assert_allclose(pre.block_attention_dual(suf, Q, Ka, Va, 0.1),
                               one.block_attention(Q, Ka, Va, 0.1), atol=1e-13)


def test_dual_prefix_and_suffix_roles_swap():
    """Attention is symmetric in which cache holds which region."""
    w, mk, A, X = _dual_setup(kb=4, vb=2, gk=64, gv=32)
    a1, b1, a2, b2 = mk(256), mk(256), mk(256), mk(256)
    for K, V, M in A:
        a1.commit(K, V, M)
        a2.commit(K, V, M)
    for K, V, M in X:
        b1.commit(K, V, M)
        b2.commit(K, V, M)
    Q = synth.queries_bits(w, 2)
    Ka, Va = synth.active_block_bits(w, 2)
    np.testing.assert_allclose(a1.block_attention_dual(b1, Q, Ka, Va, 0.1),
                               b2.block_attention_dual(a2, Q, Ka, Va, 0.1), atol=1e-13)


def test_dual_passthrough_is_dense_attention():
    w, mk, A, X = _dual_setup(kb=16, vb=16)
    pre, suf = mk(256), mk(128)
    for K, V, M in A:
        pre.commit(K, V, M)
    for K, V, M in X:
        suf.commit(K, V, M)
    Q = synth.queries_bits(w, 3)
    Ka, Va = synth.active_block_bits(w, 3)
    got = pre.block_attention_dual(suf, Q, Ka, Va, 0.1)
    for h in range(w.Hkv):
        Kall = bf16_to_f64(np.concatenate([b[0][0, h] for b in A] + [Ka[0, h]] +
                                          [b[0][0, h] for b in X]))
        Vall = bf16_to_f64(np.concatenate([b[1][0, h] for b in A] + [Va[0, h]] +
                                          [b[1][0, h] for b in X]))
        for hq in range(h * 2, h * 2 + 2):
            want = dense_attention_f64(bf16_to_f64(Q[0, hq]), Kall, Vall, 0.1)
            np.testing.assert_allclose(got[0, hq], want, atol=1e-13)


# ------------------------------------------------------------ MaskAhead selection

def _sel_cache(kb=4, vb=4, n_blocks=6, seed=0):
    w = synth.WORKLOADS["tiny"].with_(Hq=4, Hkv=2, k_bits=kb, v_bits=vb, prot_frac=0.02,
                                      seed=seed)
    oc = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, kb, vb, 32, 32, 64, (n_blocks + 1) * 32)
    for i in range(n_blocks):
        oc.commit(*synth.block_inputs(w, i))
    return w, oc


def test_selection_with_full_budget_is_plain_attention():
    w, oc = _sel_cache()
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    O, sel, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, oc.len + 5)
    assert all(np.array_equal(s, np.arange(oc.len)) for s in sel)
    assert np.array_equal(O, oc.block_attention(Q, Ka, Va, w.softmax_scale))


def test_selection_with_zero_budget_attends_the_active_block_only():
    w, oc = _sel_cache()
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    O, sel, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 0)
    assert all(s.size == 0 for s in sel)
    empty = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, 4, 4, 32, 32, 0, 64)
    np.testing.assert_allclose(O, empty.block_attention(Q, Ka, Va, w.softmax_scale), atol=1e-13)


def test_selection_finds_planted_heavy_hitters():
    """Keys pointing along a direction every query shares, with ordinary
    values, take almost all attention mass: exactly they are selected."""
    r = np.random.default_rng(3)
    d, blk, nb = 128, 32, 4
    L = nb * blk
    oc = OracleCache(1, 2, 1, d, blk, 16, 16, 32, 32, 0, L + blk)
    e0 = np.zeros(d)
    e0[0] = 1.0
    T = np.sort(r.choice(L, 9, replace=False))
    K = r.standard_normal((L, d)) * 0.1
    K[:, 0] = 0.0
    K[T] += 6.0 * e0
    V = r.standard_normal((L, d))
    for i in range(nb):
        sl = slice(i * blk, (i + 1) * blk)
        oc.commit(synth.f32_to_bf16_bits(K[sl].astype(np.float32))[None, None],
                  synth.f32_to_bf16_bits(V[sl].astype(np.float32))[None, None])
    q = r.standard_normal((1, 2, blk, d)) * 0.3
    q[..., 0] = 1.0
    Q = synth.f32_to_bf16_bits(q.astype(np.float32))
    Ka = synth.f32_to_bf16_bits((r.standard_normal((1, 1, blk, d)) * 0.1).astype(np.float32))
    Va = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
    _, sel, _ = oc.block_attention_selected(Q, Ka, Va, 1.0, len(T))
    assert np.array_equal(sel[0], T)


def test_selection_ties_keep_the_lowest_positions():
    """Zero queries give every key the same weight; V rows that differ only
    in signs have the same norm: all contributions tie exactly."""
    d, blk, nb = 128, 32, 3
    L = nb * blk
    r = np.random.default_rng(4)
    base = r.standard_normal(d)
    oc = OracleCache(1, 1, 1, d, blk, 16, 16, 32, 32, 0, L + blk)
    for i in range(nb):
        V = base[None] * r.choice([-1.0, 1.0], (blk, d))
        K = r.standard_normal((blk, d))
        oc.commit(synth.f32_to_bf16_bits(K.astype(np.float32))[None, None],
                  synth.f32_to_bf16_bits(V.astype(np.float32))[None, None])
    Q = np.zeros((1, 1, blk, d), np.uint16)
    Ka = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
    _, sel, _ = oc.block_attention_selected(Q, Ka, Ka, 1.0, 40)
    assert np.array_equal(sel[0], np.arange(40))


def test_selection_follows_entries_when_blocks_are_permuted():
    w, oc = _sel_cache(kb=2, vb=4, n_blocks=5, seed=2)
    order = [3, 0, 4, 1, 2]
    oc2 = OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, 2, 4, 32, 32, 64, 6 * 32)
    for i in order:
        oc2.commit(*synth.block_inputs(w, i))
    Q = synth.queries_bits(w, 2)
    Ka, Va = synth.active_block_bits(w, 2)
    O1, s1, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 37)
    O2, s2, _ = oc2.block_attention_selected(Q, Ka, Va, w.softmax_scale, 37)
    np.testing.assert_allclose(O1, O2, atol=1e-12)
    # position p of block order[p // 32] in the permuted cache is position
    # order[p // 32] * 32 + p % 32 of the original
    for a, b in zip(s1, s2):
        mapped = np.sort(np.array([order[p // 32] * 32 + p % 32 for p in b]))
        assert np.array_equal(a, mapped)


def test_selection_by_contribution_beats_random_selection():
    """What the ranking is for: with peaked attention, keeping the entries of
    highest contribution score approximates full attention better than
    keeping as many random entries."""
    r = np.random.default_rng(5)
    d, blk, nb = 128, 32, 8
    L = nb * blk
    oc = OracleCache(1, 4, 1, d, blk, 4, 4, 32, 32, 0, L + blk)
    K = r.standard_normal((L, d))
    K[r.choice(L, 24, replace=False)] *= 3.0
    V = r.standard_normal((L, d))
    for i in range(nb):
        sl = slice(i * blk, (i + 1) * blk)
        oc.commit(synth.f32_to_bf16_bits(K[sl].astype(np.float32))[None, None],
                  synth.f32_to_bf16_bits(V[sl].astype(np.float32))[None, None])
    Q = synth.f32_to_bf16_bits(r.standard_normal((1, 4, blk, d)).astype(np.float32))
    Ka = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
    Va = synth.f32_to_bf16_bits(r.standard_normal((1, 1, blk, d)).astype(np.float32))
    scale = 1.0 / np.sqrt(d)
    full = oc.block_attention(Q, Ka, Va, scale)
    O, _, _ = oc.block_attention_selected(Q, Ka, Va, scale, 64)
    err_sel = np.abs(O - full).mean()
    # random subsets of the same size, attended the same way
    Kc, Vc = oc.dequant_k(0), oc.dequant_v(0)
    Qf, Kaf, Vaf = bf16_to_f64(Q[0]), bf16_to_f64(Ka[0, 0]), bf16_to_f64(Va[0, 0])
    errs = []
    for t in range(5):
        sub = np.sort(r.choice(L, 64, replace=False))
        Ks, Vs = np.concatenate([Kc[sub], Kaf]), np.concatenate([Vc[sub], Vaf])
        Or = np.stack([dense_attention_f64(Qf[h], Ks, Vs, scale) for h in range(4)])
        errs.append(np.abs(Or - full[0]).mean())
    assert err_sel < 0.5 * min(errs), (err_sel, errs)


def test_selection_weighs_attention_mass_by_value_norm():
    """Entries A take more attention mass but carry values near zero; entries
    B take less mass with large values.  Their contribution to the output is
    B's, so B is selected."""
    r = np.random.default_rng(6)
    d, blk, nb = 128, 32, 4
    L = nb * blk
    oc = OracleCache(1, 1, 1, d, blk, 16, 16, 32, 32, 0, L + blk)
    idx = r.permutation(L)
    A, B = np.sort(idx[:6]), np.sort(idx[6:12])
    K = r.standard_normal((L, d)) * 0.05
    K[:, 0] = 0.0
    K[A, 0] = 4.0
    K[B, 0] = 3.0
    V = r.standard_normal((L, d)) * 0.05
    V[A] *= 0.01
    V[B] *= 100.0
    for i in range(nb):
        sl = slice(i * blk, (i + 1) * blk)
        oc.commit(synth.f32_to_bf16_bits(K[sl].astype(np.float32))[None, None],
                  synth.f32_to_bf16_bits(V[sl].astype(np.float32))[None, None])
    q = np.zeros((1, 1, blk, d))
    q[..., 0] = 1.0
    Q = synth.f32_to_bf16_bits(q.astype(np.float32))
    Ka = np.zeros((1, 1, blk, d), np.uint16)
    _, sel, _ = oc.block_attention_selected(Q, Ka, Ka, 2.0, 6)
    assert np.array_equal(sel[0], B)


# ------------------------------------------------------------ per-sequence lengths

from oracle import OracleRaggedCache  # noqa: E402


def _ragged_setup():
    w = synth.WORKLOADS["tiny"].with_(B=3, Hq=4, Hkv=2, prot_frac=0.03, seed=5)
    args = (w.B, w.Hq, w.Hkv, w.d, w.blk, w.k_bits, w.v_bits, 64, w.v_group, 32, 256)
    return w, args


def test_ragged_with_every_sequence_committing_is_the_batched_cache():
    w, args = _ragged_setup()
    rc, bc = OracleRaggedCache(*args), OracleCache(*args)
    for i in range(5):
        K, V, M = synth.block_inputs(w, i)
        assert rc.commit(K, V, M) == bc.commit(K, V, M)
    Q = synth.queries_bits(w, 0)
    Ka, Va = synth.active_block_bits(w, 0)
    np.testing.assert_allclose(rc.block_attention(Q, Ka, Va, 0.1),
                               bc.block_attention(Q, Ka, Va, 0.1), atol=1e-13)
    snap = bc.snapshot()
    for b in range(w.B):
        one = rc.seqs[b].snapshot()
        units = slice(b * w.Hkv, (b + 1) * w.Hkv)
        for key in ("k_codes", "k_sz", "v_codes", "v_sz", "k_tail", "prot_count"):
            assert np.array_equal(one[key], snap[key][units]), key


def test_each_sequence_sees_only_its_own_commits():
    """Sequence b's output equals that of a one-sequence cache given only the
    blocks b committed (its rows of those blocks), whatever the others did."""
    w, args = _ragged_setup()
    rc = OracleRaggedCache(*args)
    plan = [[0, 1, 2], [0, 2], [1], [0, 1, 2], [2], [0]]     # sequences per commit
    for i, seqs in enumerate(plan):
        rc.commit(*synth.block_inputs(w, i), seqs=seqs)
    assert rc.lens == [4 * 32, 3 * 32, 4 * 32]
    Q = synth.queries_bits(w, 1)
    Ka, Va = synth.active_block_bits(w, 1)
    O = rc.block_attention(Q, Ka, Va, 0.1)
    for b in range(w.B):
        one = OracleCache(1, *args[1:])
        for i, seqs in enumerate(plan):
            if b in seqs:
                K, V, M = synth.block_inputs(w, i)
                one.commit(K[b:b + 1], V[b:b + 1], M[b:b + 1])
        np.testing.assert_allclose(O[b:b + 1], one.block_attention(Q[b:b + 1], Ka[b:b + 1],
                                                                   Va[b:b + 1], 0.1),
                                   atol=1e-13)


def test_selection_given_explicitly_reproduces_the_ranking():
    """Passing the ranking's own selection back gives the same output; a
    different selection of the same size gives another output."""
    w, oc = _sel_cache(seed=7)
    Q = synth.queries_bits(w, 3)
    Ka, Va = synth.active_block_bits(w, 3)
    O, sel, contrib = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 48)
    O2, sel2, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 48, selection=sel)
    assert np.array_equal(O, O2) and all(np.array_equal(a, b) for a, b in zip(sel, sel2))
    # the selected entries hold the 48 largest contributions
    for s, c in zip(sel, contrib):
        assert c[s].min() >= np.sort(c)[-48]
    other = [np.sort(np.setdiff1d(np.arange(oc.len), s))[:48] for s in sel]
    O3, _, _ = oc.block_attention_selected(Q, Ka, Va, w.softmax_scale, 48, selection=other)
    assert not np.allclose(O, O3)


def test_dual_with_a_sink_in_the_prefix_equals_one_cache():
    """The prefix's sink positions keep full precision; the suffix has none.
    With one-block K groups the combined cache (sink at its start, the
    suffix appended) dequantizes to the same entries."""
    w = synth.WORKLOADS["tiny"].with_(Hq=4, Hkv=2, k_bits=2, v_bits=2, prot_frac=0.02, seed=11)
    mk = lambda cap, sink: OracleCache(w.B, w.Hq, w.Hkv, w.d, w.blk, 2, 2, 32, 32, 96, cap, sink)
    pre, suf, one = mk(256, 40), mk(128, 0), mk(384, 40)
    for i in range(4):
        K, V, M = synth.block_inputs(w, i)
        pre.commit(K, V, M)
        one.commit(K, V, M)
    for i in range(4, 7):
        K, V, M = synth.block_inputs(w, i)
        suf.commit(K, V, M)
        one.commit(K, V, M)
    Q = synth.queries_bits(w, 4)
    Ka, Va = synth.active_block_bits(w, 4)
    np.testing.assert_allclose(pre.block_attention_dual(suf, Q, Ka, Va, 0.1),
                               one.block_attention(Q, Ka, Va, 0.1), atol=1e-13)
