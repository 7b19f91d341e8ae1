"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the float64 oracle.

Tolerances (stated for the whole problem, relative RMSE = ||o - r||_2 / ||r||_2
over every compared element, max abs = max |o - r|):
  * exact bf16/fp16 mode: rel RMSE <= 5e-3 and max abs <= 2e-2;
  * INT8-QK / FP8-PV mode: rel RMSE <= 6e-2 against the float64 exact result.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from attention_forward_flash_b200 import Attention
from attention_forward_flash_b200.inputs import make_qkv, sample_rows
from oracle import attention_f64

EXACT_RMSE = 5e-3
EXACT_MAXABS = 2e-2
QUANT_RMSE = 6e-2


def rel_rmse(o, r):
    o = np.asarray(o, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    den = np.sqrt(np.sum(r * r))
    return float(np.sqrt(np.sum((o - r) ** 2)) / den) if den > 0 else float(np.sqrt(np.sum(o * o)))


def max_abs(o, r):
    return float(np.max(np.abs(np.asarray(o, np.float64) - np.asarray(r, np.float64)))) if np.size(r) else 0.0


def attention_for(w, precision="exact", num_splits=0):
    return Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                     dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                     window_lo=w.window_lo, precision=precision, num_splits=num_splits,
                     window_size=w.window_size)


def run_gpu(w, q, k, v, precision="exact", num_splits=0):
    """Returns (out [B,Hq,Sq,D] on CPU as float64 numpy, lse numpy, attention object)."""
    att = attention_for(w, precision, num_splits)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = att.forward(qd, kd, vd, return_lse=True)
    att.check_error()
    return out.double().cpu().numpy(), lse.cpu().numpy(), att


def oracle_for(w, q, k, v, rows=None):
    return attention_f64(q, k, v, causal=w.causal, start_pos=w.start_pos, window_lo=w.window_lo,
                         window_size=w.window_size,
                         rows=rows)


def check_exact(o, r, what=""):
    e, m = rel_rmse(o, r), max_abs(o, r)
    assert e <= EXACT_RMSE and m <= EXACT_MAXABS, f"{what}: rel_rmse={e:.3e} max_abs={m:.3e}"
    return e, m


def check_lse(lse, ref, what="", tol=1e-3):
    lse = np.asarray(lse, np.float64)
    ref = np.asarray(ref, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: -inf pattern differs"
    assert np.all(lse[~fin] == -math.inf)
    if fin.any():
        err = np.max(np.abs(lse[fin] - ref[fin]))
        assert err <= tol, f"{what}: lse max err {err:.3e}"
