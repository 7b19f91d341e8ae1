"""Diagonal-tiled mixed precision (precision "mixed", ``ATTN_MIXED_DIAG``) against the
oracle.

The mode is the quantised one (INT8 Q K^T, FP8 E4M3 P and V) except on the key
tiles of each query tile's causal diagonal band, whose Q K^T uses the 16-bit
inputs.  Two references, as for the quantised mode: the float64 exact result
(reported against the quantised mode's error on the same inputs), and float64
attention on the operands the mode multiplies -- exact Q and K on each row's band
(``oracle.diagonal_band_start``), the oracle quantiser's values elsewhere,
dequantised FP8 V -- which isolates the kernel's own error (FP8 P, 16-bit output).
"""

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv, sample_rows
from oracle import (attention_f64_mixed, dequantize_qk, dequantize_v, quantize_qk_int8,
                    quantize_v_fp8)
from parity_util import QUANT_RMSE, check_lse, oracle_for, rel_rmse

pytestmark = pytest.mark.gpu

QUANT_VS_DEQUANT_RMSE = 3.6e-2   # as for the quantised mode: FP8 P and the 16-bit output


def _run(w, precision, q, k, v, num_splits=0):
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                    precision=precision, num_splits=num_splits)
    o, lse = att.forward(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    att.check_error()
    if precision == "mixed":
        assert att.num_splits == 1   # the band mode always runs the single-pass kernel
    return o.double().cpu().numpy(), lse.cpu().numpy()


def _mixed_oracle(w, q, k, v, rows):
    qd = dequantize_qk(*quantize_qk_int8(q.float().numpy()))
    kd = dequantize_qk(*quantize_qk_int8(k.float().numpy()))
    vd = dequantize_v(*quantize_v_fp8(v.float().numpy()), w.kv_len)
    return attention_f64_mixed(q, k, qd, kd, vd, causal=w.causal, start_pos=w.start_pos,
                               rows=rows)


CASES = [
    # causal GQA prefill with 1% of K entries x20 (the llm workload's recipe), smaller
    Workload("llm_s", 1, 8, 2, 2048, 2048, 128, "bf16", causal=True, seed=9001,
             k_outlier_frac=0.01, k_outlier_mult=20.0, oracle_rows=96),
    # ragged rows: 256-row tiles straddle heads, chunked prefill at a start position
    Workload("ragged", 2, 4, 2, 700, 1500, 128, "bf16", causal=True, start_pos=800, seed=9002,
             oracle_rows=96),
    Workload("d64", 1, 4, 4, 1000, 1000, 64, "fp16", causal=True, seed=9003, oracle_rows=96),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_mixed_against_its_operands_and_the_exact_result(w):
    q, k, v = make_qkv(w)
    rows = sample_rows(w).numpy()
    o, lse = _run(w, "mixed", q, k, v)
    rm, rml = _mixed_oracle(w, q, k, v, rows)
    e = rel_rmse(o[:, :, rows], rm)
    assert e <= QUANT_VS_DEQUANT_RMSE, f"{w.name}: vs the mode's operands {e:.3e}"
    check_lse(lse[:, :, rows], rml, w.name, tol=1e-3)
    # against the exact result, beside the quantised mode on the same inputs.  With
    # K outliers (llm_s) the INT8 scores dominate the error and the exact band lowers
    # it; on N(0,1) inputs FP8 P and V dominate, and the two modes' errors differ
    # only by how those roundings fall (a few per cent either way).
    ro, _ = oracle_for(w, q, k, v, rows=rows)
    e_mixed = rel_rmse(o[:, :, rows], ro)
    oq, _ = _run(w, "quant", q, k, v)
    e_quant = rel_rmse(oq[:, :, rows], ro)
    print(f"{w.name}: rel RMSE mixed {e_mixed:.4e}, quantised {e_quant:.4e}")
    if w.name == "llm_s":
        assert e_mixed < e_quant, (e_mixed, e_quant)
    else:
        assert e_mixed <= QUANT_RMSE and abs(e_mixed - e_quant) <= 0.1 * e_quant, (e_mixed,
                                                                                   e_quant)


def test_mixed_without_causal_mask_is_the_quantised_mode():
    w = Workload("nc", 1, 4, 2, 600, 900, 128, "bf16", seed=9004)
    q, k, v = make_qkv(w)
    o_m, l_m = _run(w, "mixed", q, k, v)
    o_q, l_q = _run(w, "quant", q, k, v, num_splits=1)   # the same single-pass order
    assert np.array_equal(o_m, o_q) and np.array_equal(l_m, l_q)


def test_llm_workload_accuracy():
    """The causal GQA prefill workload at full size, 256 sampled rows per head.  The
    per-128-token-block INT8 K cannot meet the 6e-2 target on its 20x element
    outliers (the quantised mode's strict xfail in test_gpu_parity.py); the band
    mode's exact diagonal band lowers the error, not below the target."""
    w = WORKLOADS["llm"]
    q, k, v = make_qkv(w)
    rows = sample_rows(w).numpy()
    ro, _ = oracle_for(w, q, k, v, rows=rows)
    e = {}
    for mode in ("quant", "mixed"):
        o, _ = _run(w, mode, q, k, v)
        e[mode] = rel_rmse(o[:, :, rows], ro)
    print(f"llm: rel RMSE mixed {e['mixed']:.4e}, quantised {e['quant']:.4e}")
    assert e["mixed"] < e["quant"] <= 7.5e-2, e
