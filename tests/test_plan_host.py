"""The kernel choice (``attn_plan_for``: the same host arithmetic as ``attn_create``, no
device) on hand-worked cases for a 148-SM B200 and other SM counts: which kernel runs,
how many key splits, and the short-last-wave split."""

import pytest

from attention_forward_flash_b200 import _abi


def _p(**kw):
    base = dict(batch=1, n_q_heads=2, n_kv_heads=2, q_len=256, kv_len=256, head_dim=128,
                start_pos=0, causal=0, window_lo=0, scale=0.0, dtype=0, precision=0,
                num_splits=0)
    base.update(kw)
    return _abi.AttnParams(**base)


SINGLE, SPLIT, DECODE, TAIL = (_abi.ATTN_PATH_SINGLE_PASS, _abi.ATTN_PATH_SPLIT_MERGE,
                               _abi.ATTN_PATH_DECODE, _abi.ATTN_PATH_SINGLE_PASS_TAIL)


def test_video_fills_whole_waves_but_the_last_one_stays():
    # 40 units x 128 row tiles = 5120 CTAs = 34 waves of 148 + 88: the last wave is more
    # than half full, so no CTA is moved
    pl = _abi.attn_plan_for(_p(n_q_heads=40, n_kv_heads=40, q_len=32760, kv_len=32760), 148)
    assert (pl["path"], pl["ctas"], pl["tail_items"]) == (SINGLE, 5120, 0)


def test_image_short_last_wave_goes_to_the_split_kernel():
    # 20 units x 16 tiles = 320 = 2 x 148 + 24; k = floor(148 / 24) = 6 (32 key tiles)
    img = dict(batch=2, n_q_heads=10, n_kv_heads=10, q_len=4096, kv_len=4096, head_dim=64)
    pl = _abi.attn_plan_for(_p(**img), 148)
    assert (pl["path"], pl["ctas"], pl["tail_items"], pl["tail_splits"]) == (TAIL, 296, 24, 6)
    # the INT8 mode too; not the FP4 or band modes, not causal, not when forced to one pass
    assert _abi.attn_plan_for(_p(**img, precision=1), 148)["path"] == TAIL
    assert _abi.attn_plan_for(_p(**img, precision=3), 148)["path"] == SINGLE
    assert _abi.attn_plan_for(_p(**img, causal=1), 148)["path"] == SINGLE
    assert _abi.attn_plan_for(_p(**img, num_splits=1), 148)["path"] == SINGLE
    # 132 SMs: 320 = 2 x 132 + 56, 56 <= 66 -> k = floor(132 / 56) = 2
    pl = _abi.attn_plan_for(_p(**img), 132)
    assert (pl["tail_items"], pl["tail_splits"], pl["ctas"]) == (56, 2, 264)
    # 160 SMs: 320 = 2 x 160, no short wave
    assert _abi.attn_plan_for(_p(**img), 160)["path"] == SINGLE


def test_rows_not_in_whole_256_row_tiles_keep_the_single_pass_grid():
    # 40 units x 300 rows: not whole 256-row tiles
    pl = _abi.attn_plan_for(_p(n_q_heads=40, n_kv_heads=40, q_len=300, kv_len=4096), 148)
    assert pl["path"] == SINGLE


def test_decode_shapes_take_the_cluster_kernel():
    dec = dict(n_q_heads=16, n_kv_heads=8, q_len=4, kv_len=4096, causal=1, start_pos=4092,
               dtype=1)
    pl = _abi.attn_plan_for(_p(**dec), 148)
    # 8 rows per unit; 148 / 8 = 18 -> 16 CTAs per cluster; 4096 keys / 32 = 128 chunks
    assert (pl["path"], pl["splits"], pl["ctas"], pl["decode_chunk"], pl["decode_chunks"]) == \
        (DECODE, 16, 128, 32, 128)
    # a window bound at key 40 and 4133 keys: keys 40..4132 -> chunks 1..129
    pl = _abi.attn_plan_for(_p(**dict(dec, kv_len=4133, start_pos=4129, window_lo=40)), 148)
    assert pl["decode_chunks"] == 129
    # head_dim 64: chunks of 64 keys
    assert _abi.attn_plan_for(_p(**dict(dec, head_dim=64)), 148)["decode_chunk"] == 64
    # forced splits up to the cluster limit stay on it; above it, the split kernel
    assert _abi.attn_plan_for(_p(**dec, num_splits=7), 148)["splits"] == 7
    pl = _abi.attn_plan_for(_p(**dec, num_splits=32), 148)
    assert (pl["path"], pl["splits"], pl["tiles_per_split"]) == (SPLIT, 32, 1)
    assert _abi.attn_plan_for(_p(**dec, num_splits=1), 148)["path"] == SINGLE
    # the quantised modes take the split kernel for few rows
    assert _abi.attn_plan_for(_p(**dec, precision=1), 148)["path"] == SPLIT
    # 16 rows still decode, 17 do not
    assert _abi.attn_plan_for(_p(n_q_heads=16, n_kv_heads=1, q_len=1, kv_len=999), 148)["path"] \
        == DECODE
    assert _abi.attn_plan_for(_p(n_q_heads=17, n_kv_heads=1, q_len=1, kv_len=999), 148)["path"] \
        == SPLIT


def test_cluster_size_follows_units_and_keys():
    # 100 units: 148 / 100 = 1 CTA per cluster
    pl = _abi.attn_plan_for(_p(batch=50, n_q_heads=4, n_kv_heads=2, q_len=1, kv_len=4096), 148)
    assert (pl["path"], pl["splits"], pl["ctas"]) == (DECODE, 1, 100)
    # few keys: 100 keys at head_dim 128 -> 4 chunks -> at most 4 CTAs per cluster
    pl = _abi.attn_plan_for(_p(n_q_heads=2, n_kv_heads=2, q_len=3, kv_len=100, causal=1,
                               start_pos=97), 148)
    assert (pl["splits"], pl["decode_chunks"]) == (4, 4)
    # no row sees a key: no chunk, one CTA per unit
    pl = _abi.attn_plan_for(_p(n_q_heads=4, n_kv_heads=2, q_len=4, kv_len=300, causal=1,
                               start_pos=50, window_lo=200), 148)
    assert (pl["path"], pl["splits"], pl["decode_chunks"]) == (DECODE, 1, 0)


def test_few_ctas_take_the_split_kernel():
    # 40 rows per unit, 2 units, 2000 keys: 128-row tiles, 2 x 148 / 2 -> capped by 16 key tiles
    pl = _abi.attn_plan_for(_p(n_q_heads=2, n_kv_heads=2, q_len=40, kv_len=2000), 148)
    assert (pl["path"], pl["splits"], pl["tiles_per_split"], pl["ctas"]) == (SPLIT, 16, 1, 32)


@pytest.mark.parametrize("bad,status", [(dict(head_dim=96), _abi.ATTN_ERR_UNSUPPORTED),
                                        (dict(n_q_heads=3, n_kv_heads=2),
                                         _abi.ATTN_ERR_INVALID_ARG)])
def test_invalid_problems_are_rejected(bad, status):
    with pytest.raises(_abi.AttnError) as e:
        _abi.attn_plan_for(_p(**bad), 148)
    assert e.value.status == status


def test_num_sms_must_be_positive():
    assert _abi.lib().attn_plan_for(_p(), 0, None) == _abi.ATTN_ERR_INVALID_ARG
