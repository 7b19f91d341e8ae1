"""Pins of the float64 attention oracle against things other than itself.

Each check is chosen so that a plausible slip in the oracle (a dropped scale, a
swapped K/V, a wrong GQA index, a causal or window off-by-one, an ignored start
position) fails at least one of them:

* the hand-worked 2x3x2 example in ``golden/hand_2x3x2.json``;
* a separately written pure-Python brute force (textbook softmax, no max
  subtraction, explicit index loops) on tiny random problems;
* torch's CPU float64 ``scaled_dot_product_attention`` with an explicit
  boolean mask (an independent library routine);
* invariants: softmax rows sum to one, one-hot V returns a column of P, zero
  scores give the mean of visible V rows, masked keys have no influence,
  single visible key returns that V row, GQA equals MHA with repeated K/V.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention_f64, attention_flops, gather_paged, visible_pairs, visible_range

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _frac(s):
    if s == "-inf":
        return -math.inf
    if s.startswith("ln"):
        return math.log(float(s[2:]))
    if "/" in s:
        a, b = s.split("/")
        return float(a) / float(b)
    return float(s)


def test_hand_worked_example():
    d = json.load(open(os.path.join(GOLDEN, "hand_2x3x2.json")))
    q = np.array(d["q"], dtype=np.float64)[None, None]
    k = np.array(d["k"], dtype=np.float64)[None, None]
    v = np.array(d["v"], dtype=np.float64)[None, None]
    scale = math.log(2.0)
    for case in d["cases"]:
        o, lse = attention_f64(q, k, v, scale=scale, causal=case["causal"],
                               start_pos=case["start_pos"], window_lo=case["window_lo"],
                               window_size=case.get("window_size", 0))
        want_o = np.array([[_frac(x) for x in row] for row in case["o"]])
        want_lse = np.array([_frac(x) for x in case["lse"]])
        np.testing.assert_allclose(o[0, 0], want_o, rtol=0, atol=1e-15, err_msg=case["name"])
        np.testing.assert_allclose(lse[0, 0], want_lse, rtol=1e-15, atol=1e-15, err_msg=case["name"])


def _brute(q, k, v, scale, causal, start_pos, window_lo, window_size=0):
    """Independent restatement: explicit loops, softmax as exp(s)/sum(exp(s))."""
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Sq, D))
    lse = np.full((B, Hq, Sq), -math.inf)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            for i in range(Sq):
                pos = start_pos + i
                keys = [j for j in range(Skv)
                        if j >= window_lo and (not causal or j <= pos)
                        and (window_size == 0 or pos - j < window_size)]
                if not keys:
                    continue
                e = {}
                for j in keys:
                    s = 0.0
                    for c in range(D):
                        s += q[b, h, i, c] * k[b, kvh, j, c]
                    e[j] = math.exp(scale * s)
                tot = sum(e.values())
                lse[b, h, i] = math.log(tot)
                for c in range(D):
                    o[b, h, i, c] = sum(e[j] * v[b, kvh, j, c] for j in keys) / tot
    return o, lse


@pytest.mark.parametrize("seed", range(10))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 3))
    Hkv = int(rng.integers(1, 3))
    G = int(rng.integers(1, 3))
    Hq = Hkv * G
    Sq = int(rng.integers(1, 6))
    Skv = int(rng.integers(1, 9))
    D = int(rng.integers(1, 5))
    causal = bool(seed % 2)
    start_pos = int(rng.integers(0, 5))
    window_lo = int(rng.integers(0, 3))
    window_size = int(rng.integers(0, 4)) if seed >= 2 else 0
    scale = float(rng.uniform(0.2, 1.5))
    q = rng.standard_normal((B, Hq, Sq, D))
    k = rng.standard_normal((B, Hkv, Skv, D))
    v = rng.standard_normal((B, Hkv, Skv, D))
    o, lse = attention_f64(q, k, v, scale=scale, causal=causal, start_pos=start_pos,
                           window_lo=window_lo, window_size=window_size)
    bo, blse = _brute(q, k, v, scale, causal, start_pos, window_lo, window_size)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, blse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal,start_pos,window_lo", [
    (False, 0, 0), (True, 0, 0), (True, 7, 0), (False, 0, 5), (True, 20, 9), (True, 3, 2)])
def test_against_torch_sdpa(causal, start_pos, window_lo):
    g = torch.Generator().manual_seed(17)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 13, 29, 16
    q = torch.randn(B, Hq, Sq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Skv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Skv, D, generator=g, dtype=torch.float64)
    mask = torch.zeros(Sq, Skv, dtype=torch.bool)
    for i in range(Sq):
        for j in range(Skv):
            mask[i, j] = j >= window_lo and (not causal or j <= start_pos + i)
    ok_rows = mask.any(dim=1)
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1), attn_mask=mask)
    o, _ = attention_f64(q, k, v, causal=causal, start_pos=start_pos, window_lo=window_lo)
    np.testing.assert_allclose(o[:, :, ok_rows.numpy()], ref[:, :, ok_rows].numpy(),
                               rtol=1e-12, atol=1e-12)
    assert np.all(o[:, :, ~ok_rows.numpy()] == 0.0)


def test_probability_rows_sum_to_one_and_lse():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, 9, 8))
    k = rng.standard_normal((1, 2, 40, 8))
    v = rng.standard_normal((1, 2, 40, 8))
    o, lse, p = attention_f64(q, k, v, causal=True, start_pos=10, window_lo=4, return_probs=True)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p >= 0)
    # masked keys carry exactly zero probability
    for i in range(9):
        lo, hi = visible_range(i, kv_len=40, start_pos=10, causal=True, window_lo=4)
        assert np.all(p[..., i, :lo] == 0) and np.all(p[..., i, hi + 1:] == 0)
    # lse is log sum exp of the visible scaled scores
    from scipy.special import logsumexp
    s = (q[0, 1] @ k[0, 1].T) / math.sqrt(8)
    for i in range(9):
        lo, hi = visible_range(i, kv_len=40, start_pos=10, causal=True, window_lo=4)
        assert abs(lse[0, 1, i] - logsumexp(s[i, lo:hi + 1])) < 1e-12


def test_one_hot_v_returns_probability_column():
    rng = np.random.default_rng(4)
    Skv, D = 12, 12
    q = rng.standard_normal((1, 1, 5, D))
    k = rng.standard_normal((1, 1, Skv, D))
    v = np.eye(Skv)[None, None]  # V[j, c] = [j == c]
    o, _, p = attention_f64(q, k, v, causal=True, start_pos=6, return_probs=True)
    np.testing.assert_allclose(o[0, 0], p[0, 0], rtol=0, atol=1e-15)


def test_zero_scores_give_mean_of_visible_v():
    rng = np.random.default_rng(5)
    q = np.zeros((1, 1, 6, 8))
    k = rng.standard_normal((1, 1, 30, 8))
    v = rng.standard_normal((1, 1, 30, 8))
    o, lse = attention_f64(q, k, v, causal=True, start_pos=10, window_lo=3)
    for i in range(6):
        lo, hi = visible_range(i, kv_len=30, start_pos=10, causal=True, window_lo=3)
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, lo:hi + 1].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(hi - lo + 1)) < 1e-14


def test_masked_keys_have_no_influence():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 2, 7, 8))
    k = rng.standard_normal((1, 1, 40, 8))
    v = rng.standard_normal((1, 1, 40, 8))
    kw = dict(causal=True, start_pos=20, window_lo=5)
    o1, l1 = attention_f64(q, k, v, **kw)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, :5] = np.nan          # below the window
    k2[:, :, 27:] = 1e30           # beyond every row's causal limit (20 + 6)
    v2[:, :, :5] = 1e30
    v2[:, :, 27:] = -1e30
    o2, l2 = attention_f64(q, k2, v2, **kw)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_single_visible_key_and_causal_first_row():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 4, 8))
    k = rng.standard_normal((1, 1, 1, 8))
    v = rng.standard_normal((1, 1, 1, 8))
    o, _ = attention_f64(q, k, v)
    np.testing.assert_allclose(o[0, 0], np.repeat(v[0, 0], 4, axis=0), atol=1e-15)
    k = rng.standard_normal((1, 1, 9, 8))
    v = rng.standard_normal((1, 1, 9, 8))
    q = rng.standard_normal((1, 1, 9, 8))
    o, _ = attention_f64(q, k, v, causal=True)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-15)
    # a window that leaves exactly one key
    o, _ = attention_f64(q, k, v, causal=True, start_pos=0, window_lo=4)
    np.testing.assert_allclose(o[0, 0, 4], v[0, 0, 4], atol=1e-15)


def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((2, 6, 5, 8))
    k = rng.standard_normal((2, 2, 11, 8))
    v = rng.standard_normal((2, 2, 11, 8))
    o1, l1 = attention_f64(q, k, v, causal=True, start_pos=6)
    o2, l2 = attention_f64(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), causal=True,
                           start_pos=6)
    np.testing.assert_allclose(o1, o2, atol=1e-15)
    # head 2 of group 0 must not read kv head 1 (hq // G, not hq % Hkv)
    o3, _ = attention_f64(q[:, 2:3], k[:, 0:1], v[:, 0:1], causal=True, start_pos=6)
    np.testing.assert_allclose(o1[:, 2:3], o3, atol=1e-15)


def test_row_subset_matches_full():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 2, 20, 8))
    k = rng.standard_normal((1, 2, 20, 8))
    v = rng.standard_normal((1, 2, 20, 8))
    o, l = attention_f64(q, k, v, causal=True)
    rows = np.array([0, 3, 19, 7])
    os_, ls = attention_f64(q, k, v, causal=True, rows=rows)
    np.testing.assert_allclose(os_, o[:, :, rows], atol=1e-15)
    np.testing.assert_allclose(ls, l[:, :, rows], atol=1e-15)


def test_flop_count_reproduces_page_tops():
    # 42 ms for the FP4 kernel at 1 x 40 x 32760 x 128 is quoted as about 520 TOPS.
    f = attention_flops(1, 40, 32760, 32760, 128)
    assert abs(f / 0.042 / 1e12 - 520) < 10
    assert attention_flops(4, 32, 8192, 8192, 128, causal=True) == f * 0 + 4 * 4 * 32 * 8192 * 8192 * 128 / 2
    assert visible_pairs(4, 4096, start_pos=4092, causal=True) == 4093 + 4094 + 4095 + 4096
    assert visible_pairs(3, 3, causal=True) == 6


def test_no_keys_at_all():
    # kv_len = 0: every row sees no key -> O = 0, lse = -inf (the empty-row reading)
    q = np.ones((1, 2, 3, 4))
    k = np.zeros((1, 1, 0, 4))
    o, lse = attention_f64(q, k, k, causal=True)
    assert o.shape == (1, 2, 3, 4) and np.all(o == 0) and np.all(lse == -math.inf)


# Per-row sliding window (window_size W): row i at position p sees keys
# max(window_lo, p - W + 1) .. p (causal).
@pytest.mark.parametrize("W,start_pos,window_lo", [(1, 0, 0), (3, 5, 0), (16, 40, 0), (7, 30, 33),
                                                   (64, 0, 0)])
def test_sliding_window_against_torch_sdpa(W, start_pos, window_lo):
    g = torch.Generator().manual_seed(23)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 11, 57, 8
    q = torch.randn(B, Hq, Sq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Skv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Skv, D, generator=g, dtype=torch.float64)
    mask = torch.zeros(Sq, Skv, dtype=torch.bool)
    for i in range(Sq):
        p = start_pos + i
        for j in range(Skv):
            mask[i, j] = j >= window_lo and j <= p and p - j < W
    ok_rows = mask.any(dim=1)
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1), attn_mask=mask)
    o, lse = attention_f64(q, k, v, causal=True, start_pos=start_pos, window_lo=window_lo,
                           window_size=W)
    np.testing.assert_allclose(o[:, :, ok_rows.numpy()], ref[:, :, ok_rows].numpy(),
                               rtol=1e-12, atol=1e-12)
    assert np.all(o[:, :, ~ok_rows.numpy()] == 0.0)
    assert np.all(lse[:, :, ~ok_rows.numpy()] == -math.inf)


def test_window_of_one_returns_own_value_row():
    """W = 1, causal: row i sees only key start_pos + i, so O is that row of V and
    lse is its scaled score."""
    rng = np.random.default_rng(31)
    q = rng.standard_normal((1, 2, 6, 8))
    k = rng.standard_normal((1, 2, 20, 8))
    v = rng.standard_normal((1, 2, 20, 8))
    o, lse = attention_f64(q, k, v, causal=True, start_pos=9, window_size=1)
    np.testing.assert_allclose(o[0], v[0, :, 9:15], atol=1e-15)
    s = np.einsum("hid,hid->hi", q[0], k[0, :, 9:15]) / math.sqrt(8)
    np.testing.assert_allclose(lse[0], s, atol=1e-13)


def test_keys_outside_the_sliding_window_have_no_influence():
    rng = np.random.default_rng(32)
    q = rng.standard_normal((1, 1, 5, 8))
    k = rng.standard_normal((1, 1, 64, 8))
    v = rng.standard_normal((1, 1, 64, 8))
    kw = dict(causal=True, start_pos=50, window_size=10)   # rows see 41..50 .. 45..54
    o1, l1 = attention_f64(q, k, v, **kw)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, :41] = np.nan
    v2[:, :, :41] = 1e30
    k2[:, :, 55:] = 1e30
    v2[:, :, 55:] = np.nan
    o2, l2 = attention_f64(q, k2, v2, **kw)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # a window at least as long as every row's causal range changes nothing
    o3, l3 = attention_f64(q, k, v, causal=True, start_pos=50, window_size=55)
    o4, l4 = attention_f64(q, k, v, causal=True, start_pos=50)
    assert np.array_equal(o3, o4) and np.array_equal(l3, l4)


# Paged cache: the block-table gather.
def test_gather_paged_identity_table_is_a_reshape():
    rng = np.random.default_rng(41)
    B, Hkv, n, D = 2, 3, 5, 4
    dense = rng.standard_normal((B, Hkv, 128 * n, D))
    # block b * n + t holds positions 128 t .. of batch entry b
    pool = dense.reshape(B, Hkv, n, 128, D).transpose(0, 2, 1, 3, 4).reshape(B * n, Hkv, 128, D)
    table = np.arange(B * n).reshape(B, n)
    assert np.array_equal(gather_paged(pool, table, 128 * n), dense)


def test_gather_paged_inverts_a_scatter_through_a_random_table():
    rng = np.random.default_rng(42)
    B, Hkv, D, kv_len = 3, 2, 8, 300                 # 3 blocks per entry, the last one partial
    nbt = -(-kv_len // 128)
    dense = rng.standard_normal((B, Hkv, kv_len, D))
    nblocks = B * nbt + 4                             # spare blocks nobody references
    table = rng.permutation(nblocks)[:B * nbt].reshape(B, nbt)
    pool = np.full((nblocks, Hkv, 128, D), np.nan)
    for b in range(B):
        for t in range(nbt):
            m = min(128, kv_len - 128 * t)
            pool[table[b, t], :, :m] = dense[b, :, 128 * t:128 * t + m]
    got = gather_paged(pool, table, kv_len)
    assert np.array_equal(got, dense)                 # no NaN from spare blocks or the tail
    q = rng.standard_normal((B, 4, 5, D))
    o1, l1 = attention_f64(q, got, got, causal=True, start_pos=295)
    o2, l2 = attention_f64(q, dense, dense, causal=True, start_pos=295)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
