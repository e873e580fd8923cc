"""The commit kernel computes each code as rint of (x - z) * fl(1/s), taking
the exact division only when that estimate lies within 2^-12 of a tie
k + 1/2.  This checks, in numpy fp32 on many seeded (x, z, s) triples in the
cache's number formats (x bf16, z and s fp16), that the shortcut gives the
same clamped code as rint of the correctly rounded quotient.  The kernel's
unrolled pass clamps the estimate to [0, levels] before rounding it (by adding
1.5 * 2^23) and tests |t - rint(t)| > 1/2 - 2^-12 on the clamped value; that
form is checked against the same division-based codes."""
import numpy as np
import pytest

import synth


def _codes(x, z, s, levels):
    num = (x - z).astype(np.float32)
    exact = np.rint((num / s).astype(np.float32))
    rs = (np.float32(1) / s).astype(np.float32)
    t = (num * rs).astype(np.float32)
    near = np.abs(np.abs(t - np.rint(t)) - np.float32(0.5)) < np.float32(2.0 ** -12)
    fast = np.where(near, exact, np.rint(t))
    return (np.clip(exact, 0, levels), np.clip(fast, 0, levels), near)


def _codes_clamped_first(x, z, s, levels):
    """The kernel's form: clamp, round by the 1.5 * 2^23 addition, tie test on
    the clamped estimate, exact division where it fires."""
    num = (x - z).astype(np.float32)
    exact = np.clip(np.rint((num / s).astype(np.float32)), 0, levels)
    rs = (np.float32(1) / s).astype(np.float32)
    t = np.clip((num * rs).astype(np.float32), np.float32(0), np.float32(levels))
    big = np.float32(12582912.0)
    y = (t + big).astype(np.float32)
    code = (y.view(np.uint32) & np.uint32(levels)).astype(np.float32)
    near = np.abs((t - (y - big).astype(np.float32)).astype(np.float32)) > np.float32(0.499755859375)
    return exact, np.where(near, exact, code), near


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_reciprocal_shortcut_matches_division(bits):
    levels = (1 << bits) - 1
    r = np.random.default_rng(1234 + bits)
    n = 2_000_000
    mn = r.standard_normal(n).astype(np.float32) * np.float32(4)
    span = np.exp2(r.uniform(-12, 6, n)).astype(np.float32)
    s = (span / np.float32(levels)).astype(np.float16).astype(np.float32)
    z = mn.astype(np.float16).astype(np.float32)
    ok = s > 0
    x = mn + span * r.uniform(-0.05, 1.05, n).astype(np.float32)
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    exact, fast, near = _codes(x[ok], z[ok], s[ok], levels)
    assert np.array_equal(exact, fast)
    exact_c, fast_c, near_c = _codes_clamped_first(x[ok], z[ok], s[ok], levels)
    assert np.array_equal(exact_c, exact) and np.array_equal(fast_c, exact)
    assert near_c.sum() <= near.sum()    # the clamp only removes out-of-range ties
    # exact ties (grid inputs) take the division path
    xs = (np.arange(2 * levels + 1, dtype=np.float32) / np.float32(2))
    e2, f2, n2 = _codes(xs, np.float32(0), np.float32(1), levels)
    assert np.array_equal(e2, f2) and n2[1::2].all()
    e3, f3, n3 = _codes_clamped_first(xs, np.float32(0), np.float32(1), levels)
    assert np.array_equal(e3, e2) and np.array_equal(f3, e2) and n3[1:-1:2].all()
