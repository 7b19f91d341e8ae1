"""Host-side RoPE pieces of the C ABI (no GPU): the library's cos/sin table against
the oracle's, argument checks of the table builder, and validation of the RoPE
fields of ``attn_params``."""

import ctypes

import numpy as np
import pytest

import attention_forward_flash_b200 as afb
from attention_forward_flash_b200 import _abi
from oracle import rope_frequencies, rope_table, yarn_attention_factor


@pytest.mark.parametrize("R,n_pos,scaling,factor", [
    (128, 40000, None, 1.0), (64, 9000, "ntk", 8.0), (128, 33000, "yarn", 4.0),
    (32, 5000, "yarn", 16.0), (16, 100, None, 1.0)])
def test_library_table_matches_the_oracle_table(R, n_pos, scaling, factor):
    got = afb.rope_table(R, n_pos, base=10000.0, scaling=scaling, factor=factor,
                         original_len=4096, beta_fast=32.0, beta_slow=1.0).numpy()
    theta = rope_frequencies(R, base=10000.0, scaling=scaling, factor=factor,
                             original_len=4096 if scaling == "yarn" else None)
    m = yarn_attention_factor(factor) if scaling == "yarn" else 1.0
    ref = rope_table(n_pos, theta, mscale=m)
    assert got.shape == ref.shape == (n_pos, 2, R // 2) and got.dtype == np.float32
    # both round a float64 cosine or sine once.  Different libm implementations may
    # differ in the last float64 bits, which near a zero of cos or sin of a large
    # angle p * theta (up to ~4e4 rad) is an absolute ~1e-12: allow one float32
    # step plus that
    step = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(got.astype(np.float64) - ref) <= step + 2e-11)
    assert np.mean(got == ref) > 0.999


def test_table_builder_rejects_bad_arguments():
    L = afb.lib()
    buf = (ctypes.c_float * 64)()
    ok = _abi.AttnRopeFreq(10000.0, 0, 1.0, 0, 32.0, 1.0)
    assert L.attn_rope_table(16, 2, ctypes.byref(ok), buf) == _abi.ATTN_OK
    bad = [
        (15, 2, ok), (0, 2, ok), (16, 0, ok), (16, 2, None),
        (16, 2, _abi.AttnRopeFreq(0.0, 0, 1.0, 0, 32.0, 1.0)),
        (16, 2, _abi.AttnRopeFreq(10000.0, 0, 0.5, 0, 32.0, 1.0)),
        (16, 2, _abi.AttnRopeFreq(10000.0, 7, 1.0, 0, 32.0, 1.0)),
        (16, 2, _abi.AttnRopeFreq(10000.0, 2, 4.0, 0, 32.0, 1.0)),      # YaRN without length
        (16, 2, _abi.AttnRopeFreq(10000.0, 2, 4.0, 4096, 1.0, 32.0)),   # ramp bounds swapped
    ]
    for R, n, f in bad:
        fp = ctypes.byref(f) if f is not None else None
        assert L.attn_rope_table(R, n, fp, buf) == _abi.ATTN_ERR_INVALID_ARG, (R, n)
    assert L.attn_rope_table(16, 2, ctypes.byref(ok), None) == _abi.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(rope_dim=8), dict(rope_dim=-16), dict(rope_dim=100),
                                dict(rope_dim=144, head_dim=128), dict(rope_dim=64,
                                                                       rope_interleaved=2),
                                dict(rope_dim=64, rope_keys_rotated=3)])
def test_create_rejects_bad_rope_fields(kw):
    base = dict(batch=1, n_q_heads=2, n_kv_heads=2, q_len=256, kv_len=256, head_dim=128,
                start_pos=0, causal=0, window_lo=0, scale=0.0, dtype=0, precision=0,
                num_splits=0)
    base.update(kw)
    p = _abi.AttnParams(**base)
    ctx = ctypes.c_void_p(1234)
    assert afb.lib().attn_create(ctypes.byref(p), ctypes.byref(ctx)) == _abi.ATTN_ERR_INVALID_ARG
    assert ctx.value is None


def test_rope_entry_points_reject_a_null_context():
    L = afb.lib()
    assert L.attn_set_rope_table(None, None, 0) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_rope_apply(None, None, None, 1, 0, 0, None) == _abi.ATTN_ERR_INVALID_ARG
    p = _abi.AttnParams(1, 2, 2, 4, 4096, 128, 4092, 1, 0, 0.0, 1, 0, 0, 0, 64, 0, 0)
    p.rope_dim = 0
    fake = ctypes.c_void_p(1 << 20)
    # the split-free entry point has no RoPE
    p.rope_dim = 64
    assert L.attn_forward_splitkv_noalloc(ctypes.byref(p), fake, fake, fake, fake, None, None,
                                          None) == _abi.ATTN_ERR_UNSUPPORTED
