"""Pins of the float64 RoPE oracle (oracle/rope.py): a hand-worked rotation,
closed forms of the NTK and YaRN frequency scalings, and the invariants that
make RoPE a relative position encoding."""

import math

import numpy as np
import pytest

from oracle.rope import apply_rope, rope_frequencies, yarn_attention_factor


def test_hand_worked_rotation():
    # D = 4, base 100: theta = (1, 0.1).  x = e0 at position 2 rotates pair 0
    # (channels 0 and 2 in the half layout) by 2 radians.
    theta = rope_frequencies(4, base=100.0)
    np.testing.assert_allclose(theta, [1.0, 0.1], rtol=0, atol=1e-15)
    out = apply_rope(np.array([[1.0, 0.0, 0.0, 0.0]]), [2], theta)
    np.testing.assert_allclose(out, [[math.cos(2), 0.0, math.sin(2), 0.0]], atol=1e-15)
    out = apply_rope(np.array([[0.0, 0.0, 0.0, 3.0]]), [10], theta)   # pair 1, angle 1 rad
    np.testing.assert_allclose(out, [[0.0, -3 * math.sin(1), 0.0, 3 * math.cos(1)]], atol=1e-15)


@pytest.mark.parametrize("layout", ["half", "interleaved"])
def test_position_zero_is_identity_and_pairs_keep_their_norm(layout):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 7, 64))
    theta = rope_frequencies(64)
    assert np.array_equal(apply_rope(x, np.zeros(7), theta, layout=layout), x)
    y = apply_rope(x, rng.integers(0, 40000, 7), theta, layout=layout)
    if layout == "half":
        nx = x[..., :32] ** 2 + x[..., 32:] ** 2
        ny = y[..., :32] ** 2 + y[..., 32:] ** 2
    else:
        nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
        ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


@pytest.mark.parametrize("layout", ["half", "interleaved"])
@pytest.mark.parametrize("scaling", [None, "ntk", "yarn"])
def test_scores_depend_only_on_the_position_difference(layout, scaling):
    rng = np.random.default_rng(2)
    D = 128
    theta = rope_frequencies(D, scaling=scaling, factor=4.0, original_len=4096)
    q = rng.standard_normal((1, D))
    k = rng.standard_normal((1, D))
    for p, pk in ((5, 3), (1000, 17), (32767, 30000)):
        qr = apply_rope(q, [p], theta, layout=layout)[0]
        kr = apply_rope(k, [pk], theta, layout=layout)[0]
        lhs = float(qr @ kr)
        rhs = float(apply_rope(q, [p - pk], theta, layout=layout)[0] @ k[0])
        assert abs(lhs - rhs) <= 1e-10 * (1 + abs(rhs))


def test_layouts_are_the_same_rotation_under_a_channel_permutation():
    rng = np.random.default_rng(3)
    D = 16
    x = rng.standard_normal((5, D))
    theta = rope_frequencies(D)
    pos = rng.integers(0, 1000, 5)
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])   # interleaved -> half
    y_int = apply_rope(x, pos, theta, layout="interleaved")
    y_half = apply_rope(x[:, perm], pos, theta, layout="half")
    np.testing.assert_allclose(y_half, y_int[:, perm], atol=1e-14)


def test_ntk_scaling_keeps_the_highest_and_divides_the_lowest_frequency():
    for D, alpha in ((64, 2.0), (128, 8.0)):
        plain = rope_frequencies(D)
        ntk = rope_frequencies(D, scaling="ntk", factor=alpha)
        assert ntk[0] == plain[0] == 1.0
        np.testing.assert_allclose(ntk[-1], plain[-1] / alpha, rtol=1e-13)
        assert np.all(np.diff(ntk / plain) < 0)          # interpolation grows with wavelength
    np.testing.assert_array_equal(rope_frequencies(64, scaling="ntk", factor=1.0),
                                  rope_frequencies(64))


def test_yarn_ramp_limits():
    D, s, L = 128, 8.0, 4096
    plain = rope_frequencies(D)
    yarn = rope_frequencies(D, scaling="yarn", factor=s, original_len=L)
    r = L * plain / (2 * math.pi)                        # full turns within the original length
    fast, slow = r >= 32.0, r <= 1.0
    assert fast.any() and slow.any()
    np.testing.assert_array_equal(yarn[fast], plain[fast])                  # unchanged
    np.testing.assert_allclose(yarn[slow], plain[slow] / s, rtol=1e-15)     # interpolated
    mid = ~fast & ~slow
    assert np.all((yarn[mid] < plain[mid]) & (yarn[mid] > plain[mid] / s))
    np.testing.assert_allclose(rope_frequencies(D, scaling="yarn", factor=1.0, original_len=L),
                               plain, rtol=1e-15)
    assert yarn_attention_factor(1.0) == 1.0
    assert abs(yarn_attention_factor(math.e) - 1.1) < 1e-15


# --- the float32 table and rotation (the form the quantised mode reproduces bit for bit)
from fractions import Fraction  # noqa: E402

from oracle.rope import apply_rope_f32, rope_table  # noqa: E402


def _rn32(q):
    """Exact rational rounded to the nearest float32 (ties to even), as a float."""
    return float(np.float32(float(q))) if q == 0 else _rn32_exact(q)


def _rn32_exact(q):
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (e - 23)
    r = round(a / quantum) * quantum
    return float(r if q > 0 else -r)


def test_f32_rotation_hand_worked():
    # exact values: a' = 1*0.5 - 2*0.25 = 0, b' = 1*0.25 + 2*0.5 = 1.25
    table = np.zeros((4, 2, 1), dtype=np.float32)
    table[3] = [[0.5], [0.25]]
    out = apply_rope_f32(np.array([[1.0, 2.0]], np.float32), [3], table)
    assert out.tolist() == [[0.0, 1.25]]
    # position 0 with cos 1, sin 0 is the identity, channels past R pass through
    table = rope_table(2, np.array([1.0, 0.5]))
    x = np.arange(1, 7, dtype=np.float32)[None]
    assert np.array_equal(apply_rope_f32(x, [0], table), x)


def test_f32_rotation_rounds_each_product_and_the_sum():
    # a, b, c, s chosen so that rounding each product before the subtraction gives
    # another float32 than a fused a*c - RN(b*s); the expected value is worked with
    # exact rationals.
    rng = np.random.default_rng(4)
    found = 0
    for _ in range(20000):
        a, b, c, s = (np.float32(v) for v in rng.standard_normal(4))
        A, B, Cc, S = (Fraction(float(v)) for v in (a, b, c, s))
        want = _rn32(Fraction(_rn32(A * Cc)) - Fraction(_rn32(B * S)))
        fused = _rn32(A * Cc - Fraction(_rn32(B * S)))
        if want == fused:
            continue
        table = np.array([[[c], [s]]], dtype=np.float32)
        got = apply_rope_f32(np.array([[a, b]], np.float32), [0], table)[0, 0]
        assert float(got) == want
        found += 1
        if found == 5:
            break
    assert found == 5


@pytest.mark.parametrize("layout", ["half", "interleaved"])
@pytest.mark.parametrize("R", [128, 64, 32])
def test_f32_rotation_within_rounding_of_float64(layout, R):
    rng = np.random.default_rng(R)
    D, S = 128, 50
    theta = rope_frequencies(R, scaling="yarn", factor=4.0, original_len=4096)
    m = yarn_attention_factor(4.0) if R == D else 1.0
    x = (rng.standard_normal((2, S, D)) * 3).astype(np.float32)
    pos = rng.integers(0, 40000, S)
    table = rope_table(40000, theta, mscale=m)
    got = apply_rope_f32(x, pos, table, layout=layout).astype(np.float64)
    ref = apply_rope(x.astype(np.float64), pos, theta, layout=layout, mscale=m)
    if R < D:   # channels past R are unchanged
        assert np.array_equal(got[..., R:], x[..., R:])
    if layout == "half":
        mag = np.concatenate([np.abs(x[..., :R // 2]) + np.abs(x[..., R // 2:R])] * 2, axis=-1)
    else:
        pair = np.abs(x[..., 0:R:2]) + np.abs(x[..., 1:R:2])
        mag = np.repeat(pair, 2, axis=-1)
    # table entries, two products and one sum each rounded once: < 4 ulps of |a| + |b|
    assert np.all(np.abs(got[..., :R] - ref[..., :R]) <= 4 * 2.0 ** -24 * m * mag + 1e-30)


def test_rope_table_obeys_the_angle_addition_formulas():
    theta = rope_frequencies(64, base=10000.0)
    t = rope_table(3000, theta).astype(np.float64)
    rng = np.random.default_rng(5)
    for p, q in rng.integers(0, 1500, (50, 2)):
        c = t[p, 0] * t[q, 0] - t[p, 1] * t[q, 1]
        s = t[p, 1] * t[q, 0] + t[p, 0] * t[q, 1]
        np.testing.assert_allclose(c, t[p + q, 0], atol=2e-6)
        np.testing.assert_allclose(s, t[p + q, 1], atol=2e-6)
    np.testing.assert_allclose(t[:, 0] ** 2 + t[:, 1] ** 2, 1.0, atol=1e-6)
    assert np.all(t[0, 0] == 1.0) and np.all(t[0, 1] == 0.0)
    m = rope_table(10, theta, mscale=1.5).astype(np.float64)
    np.testing.assert_allclose(m[:, 0] ** 2 + m[:, 1] ** 2, 2.25, rtol=1e-6)
