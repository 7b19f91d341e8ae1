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
