"""Pins of the diagonal-tiled mixed-precision oracle (``attention_f64_mixed``,
``diagonal_band_start``): the two special cases that reduce to plain attention,
hand-worked band boundaries, and the band's position in a tiny brute force."""

import math

import numpy as np
import pytest

from oracle import attention_f64, attention_f64_mixed, diagonal_band_start


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_without_causal_mask_it_is_attention_on_the_low_precision_operands():
    q, k, v = _rand((1, 4, 40, 16), 1), _rand((1, 2, 70, 16), 2), _rand((1, 2, 70, 16), 3)
    ql, kl = q + 0.1 * _rand(q.shape, 4), k + 0.1 * _rand(k.shape, 5)
    o, lse = attention_f64_mixed(q, k, ql, kl, v, causal=False)
    ro, rl = attention_f64(ql, kl, v)
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(lse, rl, atol=1e-12)


def test_when_every_key_is_in_the_band_it_is_attention_on_the_exact_operands():
    # one query tile of 100 rows at positions 0..99: the band starts at key 0
    q, k, v = _rand((2, 2, 100, 8), 6), _rand((2, 2, 100, 8), 7), _rand((2, 2, 100, 8), 8)
    ql, kl = np.zeros_like(q), np.zeros_like(k)
    o, lse = attention_f64_mixed(q, k, ql, kl, v, causal=True)
    ro, rl = attention_f64(q, k, v, causal=True)
    np.testing.assert_allclose(o, ro, atol=1e-12)
    np.testing.assert_allclose(lse, rl, atol=1e-12)


@pytest.mark.parametrize("i,hq,start_pos,want", [
    # 4 query heads over 2 kv heads, Sq = 600: a unit stacks head 0 (rows 0..599) then
    # head 1 (rows 600..1199); 256-row tiles.
    (300, 0, 0, 256),     # tile 256..511 of head 0: positions 256..511 -> key tile 2
    (10, 1, 0, 0),        # stacked row 610, tile 512..767 holds head 1 positions 0..167
    (599, 2, 0, 0),       # head 2 is head 0 of the second unit; tile 512..767 straddles
                          # heads: head 1's positions 0..167 put the band at key 0
    (400, 2, 0, 256),     # second unit, tile 256..511: positions 256..511
    (255, 0, 0, 0),       # tile 0..255: positions 0..255 -> key tile 0
    (256, 0, 1000, 1152), # chunked prefill: positions 1256..1511 -> 128 * floor(1257/128)
    (0, 0, 127, 128),     # positions 127..382: tile 0 needs no mask (127 <= 127)
    (0, 0, 126, 0),       # positions 126..381: key 127 is masked for row 0
])
def test_hand_worked_band_starts(i, hq, start_pos, want):
    assert diagonal_band_start(i, hq, Sq=600, n_q_heads=4, n_kv_heads=2,
                               start_pos=start_pos) == want


def test_no_band_without_causal():
    assert diagonal_band_start(5, 0, Sq=600, n_q_heads=4, n_kv_heads=2,
                               causal=False) > 10 ** 15


def test_brute_force_uses_exact_scores_exactly_on_the_band():
    # 1 head, 300 rows: tile 0 = rows 0..255 (band from key 0), tile 1 = rows 256..299
    # (band from key 256).  Row 290 uses exact scores for keys 256..290 and low ones
    # for keys 0..255.
    q, k, v = _rand((1, 1, 300, 4), 9), _rand((1, 1, 300, 4), 10), _rand((1, 1, 300, 4), 11)
    ql, kl = q * 0.5, k * 2.0 + 0.3
    o, lse = attention_f64_mixed(q, k, ql, kl, v, causal=True, rows=[290])
    s = [(sum(q[0, 0, 290, d] * k[0, 0, j, d] for d in range(4)) if j >= 256 else
          sum(ql[0, 0, 290, d] * kl[0, 0, j, d] for d in range(4))) / 2.0 for j in range(291)]
    w = [math.exp(x) for x in s]
    ref = [sum(w[j] * v[0, 0, j, d] for j in range(291)) / sum(w) for d in range(4)]
    np.testing.assert_allclose(o[0, 0, 0], ref, rtol=1e-12)
    assert abs(lse[0, 0, 0] - math.log(sum(w))) < 1e-12
