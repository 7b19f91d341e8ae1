"""The FP4 microscaled mode (precision "fp4", ``ATTN_MXFP4QK_FP8PV``) against the oracle.

* The MXFP4 quantiser (E2M1 codes, one E8M0 scale per 32 channels of a row) is
  bit-exact against the oracle's OCP MX conversion (``oracle.fp4``): codes unpacked
  from their nibbles, scales read from the tensor core's 512-byte chunks.
* Attention: against float64 attention on the values the codes represent (MXFP4 Q
  and K dequantised, FP8 V dequantised) within the quantised mode's kernel bound,
  which isolates the kernel's own error (FP8 P, the 16-bit output); and against the
  exact result within the reading this mode is held to (no tolerance is given for
  FP4: E2M1 keeps one mantissa bit, so a value moves by up to a quarter of itself;
  the pages' SageAttention 3 figure is 19% on its workload).
"""

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv, sample_rows
from oracle import attention_f64, dequantize_v, quantize_v_fp8
from oracle.fp4 import mxfp4_dequantize, mxfp4_quantize
from parity_util import check_lse, rel_rmse

pytestmark = pytest.mark.gpu

KERNEL_RMSE = 3.6e-2   # vs float64 on the represented operands (as the quantised mode)
FP4_RMSE = 0.30        # vs the exact result: the reading for FP4 Q K^T


def _att(w, num_splits=0):
    return Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                     dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                     window_lo=w.window_lo, window_size=w.window_size, precision="fp4",
                     num_splits=num_splits)


def _unpack(codes):
    """[..., D/2] bytes -> [..., D] 4-bit codes (channel 2i in the low nibble)."""
    c = codes.cpu().numpy().astype(np.uint8)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def _scales(sf, n_seq, tiles, L):
    """E8M0 bytes [n_seq, L, 2] from the 512-byte chunks."""
    ch = sf.cpu().numpy()[: n_seq * tiles * 512].reshape(n_seq, tiles, 512)
    r = np.arange(tiles * 128)
    t, rr = r // 128, r % 128
    off = (rr % 32) * 16 + (rr // 32) * 4
    out = np.stack([ch[:, t, off], ch[:, t, off + 1]], axis=-1)     # [n_seq, rows, 2]
    return out[:, :L], ch, off


@pytest.mark.parametrize("w", [
    Workload("q4a", 1, 4, 2, 300, 777, 64, "bf16", seed=9101),
    Workload("q4b", 2, 2, 2, 256, 1024, 64, "fp16", seed=9102, k_outlier_frac=0.01,
             k_outlier_mult=20.0),
], ids=["gqa_ragged_bf16", "outliers_fp16"])
def test_mxfp4_quantiser_bit_exact(w):
    q, k, v = make_qkv(w)
    att = _att(w)
    qb = att.quantize(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    G = w.n_q_heads // w.n_kv_heads
    units = w.batch * w.n_kv_heads
    R = G * w.q_len
    q_tiles = 2 * ((R + 255) // 256)
    k_tiles = (w.kv_len + 127) // 128
    # Q: the stacked rows of each unit; K: the keys of each (batch, kv head)
    for x, codes, sf, L, tiles in ((q, qb.q, qb.q_sf, R, q_tiles), (k, qb.k, qb.k_sf, w.kv_len,
                                                                     k_tiles)):
        xs = x.float().numpy().reshape(units, L, w.head_dim)
        ref_codes, ref_exp = mxfp4_quantize(xs)                       # [units, L, 64], [units, L, 2]
        got_codes = _unpack(codes).reshape(units, L, w.head_dim)
        assert np.array_equal(got_codes, ref_codes)
        got_exp, chunks, off = _scales(sf, units, tiles, L)
        assert np.array_equal(got_exp, ref_exp)
        # padding rows and the unused bytes hold 127 (scale 1)
        assert np.all(chunks[:, :, off + 2] == 127) and np.all(chunks[:, :, off + 3] == 127)
        pad = np.arange(tiles * 128) >= L
        if pad.any():
            r = np.arange(tiles * 128)[pad]
            assert np.all(chunks[:, r // 128, (r % 128 % 32) * 16 + (r % 128 // 32) * 4] == 127)
    # V as in the quantised mode
    vt, vs = quantize_v_fp8(v.float().numpy())
    assert np.array_equal(qb.v_t.cpu().numpy(), vt) and np.array_equal(qb.v_scale.cpu().numpy(), vs)


def _represented(w, q, k, v):
    """float64 values of MXFP4 Q and K and FP8 V (the oracle's quantisers)."""
    G = w.n_q_heads // w.n_kv_heads
    units = w.batch * w.n_kv_heads
    out = []
    for x, L in ((q, G * w.q_len), (k, w.kv_len)):
        xs = x.float().numpy().reshape(units, L, w.head_dim)
        out.append(mxfp4_dequantize(*mxfp4_quantize(xs)).reshape(x.shape))
    out.append(dequantize_v(*quantize_v_fp8(v.float().numpy()), w.kv_len))
    return out


CASES = [
    Workload("f4_prefill", 1, 4, 4, 700, 700, 64, "bf16", seed=9201, oracle_rows=128),
    Workload("f4_causal_gqa", 2, 8, 2, 513, 1111, 64, "fp16", causal=True, start_pos=598,
             seed=9202, oracle_rows=128),
    Workload("f4_window", 1, 4, 2, 600, 1300, 64, "bf16", causal=True, start_pos=700,
             window_size=300, seed=9203, oracle_rows=128),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fp4_attention(w):
    q, k, v = make_qkv(w)
    att = _att(w)
    o, lse = att.forward(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    att.check_error()
    assert att.num_splits == 1
    o = o.double().cpu().numpy()
    lse = lse.cpu().numpy()
    rows = sample_rows(w).numpy()
    qd, kd, vd = _represented(w, q, k, v)
    rm, rml = attention_f64(qd, kd, vd, causal=w.causal, start_pos=w.start_pos,
                            window_lo=w.window_lo, window_size=w.window_size, rows=rows)
    e = rel_rmse(o[:, :, rows], rm)
    assert e <= KERNEL_RMSE, f"{w.name}: vs represented operands {e:.3e}"
    check_lse(lse[:, :, rows], rml, w.name, tol=1e-3)
    ro, _ = attention_f64(q, k, v, causal=w.causal, start_pos=w.start_pos,
                          window_lo=w.window_lo, window_size=w.window_size, rows=rows)
    ex = rel_rmse(o[:, :, rows], ro)
    print(f"{w.name}: rel RMSE vs exact {ex:.4e}, vs represented {e:.4e}")
    assert ex <= FP4_RMSE, f"{w.name}: vs exact {ex:.3e}"


def test_fp4_image_workload():
    """The image workload (head_dim 64, K with per-channel offsets), all rows."""
    w = WORKLOADS["image"]
    q, k, v = make_qkv(w)
    att = _att(w)
    o = att.forward(q.cuda(), k.cuda(), v.cuda()).double().cpu().numpy()
    att.check_error()
    rows = sample_rows(w, n=256).numpy()
    qd, kd, vd = _represented(w, q, k, v)
    rm, _ = attention_f64(qd, kd, vd, rows=rows)
    assert rel_rmse(o[:, :, rows], rm) <= KERNEL_RMSE
    ro, _ = attention_f64(q, k, v, rows=rows)
    ex = rel_rmse(o[:, :, rows], ro)
    print(f"image fp4: rel RMSE vs exact {ex:.4e}")
    assert ex <= FP4_RMSE


def test_fp4_rejects_head_dim_128():
    from attention_forward_flash_b200 import _abi
    with pytest.raises(_abi.AttnError) as e:
        Attention(1, 2, 2, 128, 128, 128, precision="fp4")
    assert e.value.status == _abi.ATTN_ERR_UNSUPPORTED
