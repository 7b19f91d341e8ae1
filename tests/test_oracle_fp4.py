"""Pins of the MXFP4 reference quantiser (oracle/fp4.py): the E2M1 values the OCP
MX definition lists, hand-worked ties and saturation, an independently written
arithmetic round-half-even, and closed forms of the E8M0 block scale."""

import numpy as np
import pytest

from oracle.fp4 import (E2M1_MAX, MX_BLOCK, e2m1_decode, e2m1_encode, mxfp4_dequantize,
                        mxfp4_quantize)


def test_decode_table_is_the_listed_e2m1_values():
    assert list(e2m1_decode(np.arange(8))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(e2m1_decode(np.arange(8, 16))) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0,
                                                   -6.0]


@pytest.mark.parametrize("x,code", [
    (0.25, 0x0),   # tie 0 / 0.5 -> even code 0
    (0.75, 0x2),   # tie 0.5 / 1 -> code 2 (1.0)
    (1.25, 0x2),   # tie 1 / 1.5 -> 1.0
    (1.75, 0x4),   # tie 1.5 / 2 -> code 4 (2.0)
    (2.5, 0x4),    # tie 2 / 3 -> 2.0
    (3.5, 0x6),    # tie 3 / 4 -> code 6 (4.0)
    (5.0, 0x6),    # tie 4 / 6 -> 4.0
    (5.01, 0x7),
    (7.0, 0x7),    # saturates to 6
    (1e30, 0x7),
    (-0.3, 0x9),   # -0.5
    (-0.0, 0x8),   # negative zero keeps its sign
    (-6.5, 0xF),
])
def test_hand_worked_codes(x, code):
    assert int(e2m1_encode(np.array([x]))[0]) == code


def _rne_arith(x):
    """Round half to even by binade arithmetic: the spacing of E2M1 values is 0.5
    below 2, 1 in [2, 4) and 2 from 4 on; np.rint rounds half to even."""
    a = np.abs(x)
    ulp = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.minimum(ulp * np.rint(a / ulp), E2M1_MAX)
    return np.copysign(q, x)


def test_encoder_matches_an_arithmetic_round_half_even():
    rng = np.random.default_rng(5)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    x = np.concatenate([rng.uniform(-8, 8, 200_000), np.linspace(-7, 7, 100_001),
                        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 9)])
    np.testing.assert_array_equal(e2m1_decode(e2m1_encode(x)), _rne_arith(x))


def test_block_scale_closed_forms():
    def one_block(amax_value, fill=0.0):
        v = np.full(MX_BLOCK, fill)
        v[3] = amax_value
        return v
    # amax 6 -> floor(log2 6) - 2 = 0 -> X = 1 (biased 127); 6 itself is exact
    c, s = mxfp4_quantize(one_block(6.0))
    assert s[0] == 127 and e2m1_decode(c[3]) == 6.0
    # amax 1 -> X = 2^-2, 1 / X = 4 -> code of 4.0
    c, s = mxfp4_quantize(one_block(1.0))
    assert s[0] == 125 and int(c[3]) == 0x6
    # amax 7.9 -> X = 1: 7.9 saturates to 6 (the MX conversion's known clipping)
    c, s = mxfp4_quantize(one_block(7.9))
    assert s[0] == 127 and mxfp4_dequantize(c, s)[3] == 6.0
    # all-zero block: smallest scale, zero codes
    c, s = mxfp4_quantize(np.zeros(MX_BLOCK))
    assert s[0] == 0 and not c.any()


def test_representable_blocks_round_trip_and_errors_are_bounded():
    rng = np.random.default_rng(6)
    mags = e2m1_decode(np.arange(16))
    for e in (-10, 0, 7):
        v = rng.choice(mags, size=(4, 2 * MX_BLOCK)) * 2.0 ** e
        v[:, 0] = 6.0 * 2.0 ** e                          # fix each block's amax at 6 X
        v[:, MX_BLOCK] = -6.0 * 2.0 ** e
        c, s = mxfp4_quantize(v)
        np.testing.assert_array_equal(mxfp4_dequantize(c, s), v)
    x = rng.standard_normal((8, 4 * MX_BLOCK))
    c, s = mxfp4_quantize(x)
    d = mxfp4_dequantize(c, s)
    X = 2.0 ** (s.astype(np.float64) - 127)
    err = np.abs(d - x).reshape(8, 4, MX_BLOCK)
    # within a block: at most half a spacing below 6 X (spacing <= 2 X), more only where
    # |x| > 6 X saturates
    sat = np.abs(x).reshape(8, 4, MX_BLOCK) > 6 * X[..., None]
    assert np.all(err[~sat] <= (X[..., None] * np.ones_like(err))[~sat] + 1e-12)
