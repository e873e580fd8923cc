"""Property-based pins of the oracle's quantizer and code packing (random
widths, group sizes, value scales and protection patterns, drawn by
hypothesis): each property follows from the definitions, not from the
oracle's code."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import synth
from oracle import pack_codes, quantize_groups, unpack_codes


@settings(max_examples=60, deadline=None)
@given(bits=st.sampled_from([2, 3, 4]), words=st.integers(1, 6),
       lead=st.integers(1, 3), seed=st.integers(0, 2 ** 32 - 1))
def test_packing_is_a_bijection_with_the_bit_stream(bits, words, lead, seed):
    """pack then unpack is the identity, and stream bit i of the words is bit
    (i - bits*e) of element e = i // bits (checked bit by bit)."""
    n = words * 32
    r = np.random.default_rng(seed)
    c = r.integers(0, 2 ** bits, (lead, n)).astype(np.uint8)
    w = pack_codes(c, bits)
    assert w.shape == (lead, n * bits // 32)
    assert np.array_equal(unpack_codes(w, bits, n), c)
    for row in range(lead):
        for i in range(0, n * bits, 7):
            stream_bit = (int(w[row, i // 32]) >> (i % 32)) & 1
            assert stream_bit == (int(c[row, i // bits]) >> (i % bits)) & 1


@settings(max_examples=60, deadline=None)
@given(bits=st.sampled_from([2, 3, 4]), n=st.sampled_from([8, 32, 64, 128]),
       scale_exp=st.integers(-8, 8), frac_prot=st.floats(0.0, 0.9),
       seed=st.integers(0, 2 ** 32 - 1))
def test_quantizer_properties(bits, n, scale_exp, frac_prot, seed):
    """Codes in range; protected slots 0; kept members dequantize within
    about half a step of themselves; the kept minimum gets code 0 and the
    kept maximum the top code (when the range is not degenerate)."""
    r = np.random.default_rng(seed)
    G = 16
    x = (r.standard_normal((G, n)) * 2.0 ** scale_exp).astype(np.float32)
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    keep = r.random((G, n)) >= frac_prot
    keep[:, 0] = True
    q, s, z = quantize_groups(x, keep, bits)
    levels = 2 ** bits - 1
    assert q.max() <= levels
    assert np.all(q[~keep] == 0)
    s64, z64 = s.astype(np.float64), z.astype(np.float64)
    for g in range(G):
        xs = x[g][keep[g]].astype(np.float64)
        mn, mx = xs.min(), xs.max()
        if s64[g] == 0.0:
            assert np.all(q[g] == 0)
            continue
        if not (np.isfinite(s64[g]) and abs(mn) >= 2.0 ** -14):
            continue   # fp16 subnormal or overflowed parameters: only range checked
        xhat = q[g][keep[g]] * s64[g] + z64[g]
        # half a step, plus the fp16 rounding of s (carried over up to `levels`
        # steps) and of z
        tol = s64[g] / 2 + levels * s64[g] * 2.0 ** -11 + abs(z64[g]) * 2.0 ** -11 + 1e-30
        assert np.all(np.abs(xhat - xs) <= tol)
        assert q[g][keep[g]][np.argmin(xs)] == 0 or abs(z64[g] - mn) > 0
        if mx - mn > 4 * s64[g]:
            assert q[g][keep[g]][np.argmax(xs)] >= levels - 1
