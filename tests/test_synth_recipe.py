"""The seeded input generators follow the stated workload recipe: shapes,
protected counts, outlier channels, distributions, determinism.  CPU only."""
import math

import numpy as np
import pytest

import synth

TABLE = {
    # name: (B, Hq, Hkv, L, k_bits, v_bits, k_group, v_group, protected per unit, outliers)
    "tiny": (1, 4, 1, 256, 4, 4, 32, 32, 0, 4),
    "mha8b": (1, 32, 32, 4096, 4, 4, 32, 32, 41, 6),
    "gqa7b": (8, 28, 4, 8192, 2, 2, 32, 32, 82, 6),
    "batch32": (32, 32, 8, 16384, 2, 2, 64, 64, 328, 6),
    "longprompt": (1, 32, 8, 131072, 4, 4, 32, 32, 655, 0),
}


@pytest.mark.parametrize("name", list(TABLE))
def test_workload_table(name):
    w = synth.WORKLOADS[name]
    B, Hq, Hkv, L, kb, vb, gk, gv, npro, nout = TABLE[name]
    assert (w.B, w.Hq, w.Hkv, w.L, w.k_bits, w.v_bits, w.k_group, w.v_group) == \
        (B, Hq, Hkv, L, kb, vb, gk, gv)
    assert w.d == 128 and w.blk == 32
    assert w.n_prot_prefill == npro
    assert w.n_outlier == nout
    # the 8B MHA layer's queries carry 1/sqrt(d) themselves (scale 1)
    if name == "mha8b":
        assert w.softmax_scale == 1.0 and abs(w.q_std - 1 / math.sqrt(128)) < 1e-15
    else:
        assert abs(w.softmax_scale - 1 / math.sqrt(128)) < 1e-15 and w.q_std == 1.0


@pytest.mark.parametrize("name", ["mha8b", "batch32"])
def test_prefill_protected_positions_are_exact(name):
    """round(p L) distinct positions per unit, and the per-block masks add up
    to exactly that set."""
    w = synth.WORKLOADS[name].with_(L=2048)
    for (b, h) in [(0, 0), (0, w.Hkv - 1)]:
        pos = synth.prefill_protected_positions(w, b, h)
        assert pos.size == w.n_prot_prefill == int(round(w.prot_frac * w.L))
        assert np.unique(pos).size == pos.size and pos.min() >= 0 and pos.max() < w.L
        got = []
        for blk in range(w.L // w.blk):
            words = synth.block_protect_words(w, b, h, blk)
            bits = [t for t in range(w.blk) if (int(words[t // 32]) >> (t % 32)) & 1]
            got += [blk * w.blk + t for t in bits]
        assert np.array_equal(np.array(got), pos)


def test_late_positions_are_protected_at_the_rate():
    w = synth.WORKLOADS["batch32"].with_(L=64)
    n, hits = 0, 0
    for blk in range(2, 402):
        words = synth.block_protect_words(w, 0, 0, blk)
        hits += sum(bin(int(x)).count("1") for x in words)
        n += w.blk
    rate = hits / n
    assert abs(rate - w.prot_frac) < 0.3 * w.prot_frac, rate


@pytest.mark.parametrize("name", ["tiny", "gqa7b"])
def test_outlier_channels_are_ten_times_wider(name):
    w = synth.WORKLOADS[name]
    h = w.Hkv - 1
    oc = synth.outlier_channels(w, h)
    assert oc.size == w.n_outlier and np.unique(oc).size == oc.size
    assert np.array_equal(oc, np.sort(oc))
    ks = np.concatenate([synth.kv_block_f32(w, 0, h, blk)[0] for blk in range(64)])
    std = ks.std(axis=0)
    mask = np.zeros(w.d, bool)
    mask[oc] = True
    ratio = std[mask].mean() / std[~mask].mean()
    assert 8.5 < ratio < 11.5, ratio
    # the same channels in every sequence and in the active block
    ka = synth.active_block_bits(w, 0)[0][0, h]
    stda = synth.bf16_bits_to_f32(ka).std(axis=0)
    assert stda[mask].mean() / stda[~mask].mean() > 5


def test_long_prompt_keys_are_heavy_tailed():
    """Student-t with 3 degrees of freedom: far more mass beyond 5 standard
    normal deviations than a normal draw has."""
    w = synth.WORKLOADS["longprompt"]
    k = np.concatenate([synth.kv_block_f32(w, 0, 0, blk)[0] for blk in range(64)]).ravel()
    v = np.concatenate([synth.kv_block_f32(w, 0, 0, blk)[1] for blk in range(64)]).ravel()
    assert (np.abs(k) > 5).mean() > 1e-3      # t3: P(|x| > 5) ~ 1.5e-2
    assert (np.abs(v) > 5).mean() < 1e-5      # normal: 5.7e-7
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1) < 0.02


def test_draws_are_deterministic_and_keyed():
    w = synth.WORKLOADS["gqa7b"].with_(B=2)
    a = synth.block_inputs(w, 3)
    b = synth.block_inputs(w, 3)
    c = synth.block_inputs(w, 4)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert not np.array_equal(a[0], c[0])
    # one unit regenerated alone equals its slice of the full draw
    K1, V1, M1 = synth.block_inputs(w, 3, units=[(1, 2)])
    assert np.array_equal(K1[1, 2], a[0][1, 2]) and np.array_equal(V1[1, 2], a[1][1, 2])
    assert np.array_equal(M1[1, 2], a[2][1, 2])
    assert np.array_equal(synth.queries_bits(w, 5), synth.queries_bits(w, 5))
    assert not np.array_equal(synth.queries_bits(w, 5), synth.queries_bits(w, 6))


def test_bf16_rounding_of_inputs_is_nearest_even():
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5], np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    # bf16 steps near 1 are 2^-7.  1 + 2^-8 lies halfway between 1 (even
    # mantissa) and 1 + 2^-7; 1 + 3*2^-8 halfway between 1 + 2^-7 and
    # 1 + 2^-6 (even): both go to the even neighbour.
    assert got[0] == 1.0 and got[1] == 1.0 + 2.0 ** -6 and got[2] == -2.5
