"""CUDA path (through the C ABI) against the float64 oracle on the same seeded inputs.

Covers every workload at its full size (all rows where the oracle is quick,
a seeded subset of 256 query rows per head on the largest), in both precision
modes where the workload uses them, plus the boundary matrix of key lengths,
start positions, windows and query-row counts, empty rows, the single-pass and
split-KV variants (quantised too), determinism, masked-key independence, the
bounded-wait error path in both modes, long contexts (131072 keys in one CTA,
32768-key decodes), per-row sliding windows, and the qsa2 audit's decode matrix
on a 32768-cell cache.
"""

import math

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv, sample_rows
from oracle import attention_f64
from parity_util import (EXACT_MAXABS, EXACT_RMSE, QUANT_RMSE, check_exact, check_lse, max_abs,
                         oracle_for, rel_rmse, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode", "decode_window", "image"])
def test_exact_full(name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v)
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, name)
    check_lse(lse, rl, name)
    if name.startswith("decode"):
        assert att.num_splits > 1  # few-row problems take the split-KV path


@pytest.mark.parametrize("name", ["video", "llm", "llm_window"])
def test_exact_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v)
    rows = sample_rows(w).numpy()
    ro, rl = oracle_for(w, q, k, v, rows=rows)
    check_exact(o[:, :, rows], ro, name)
    check_lse(lse[:, :, rows], rl, name)


# INT8-QK / FP8-PV mode.  Two references: the float64 exact result (the 6e-2
# target), and float64 attention on the inputs as the oracle's own quantiser
# represents them (Q, K, V dequantised), which isolates the kernel's error (FP8 P,
# the 16-bit output) from the quantiser's.  On the causal GQA prefill workload,
# whose K has 1% of entries scaled by 20, the quantiser alone already gives
# 6.83e-2 (INT8 K 5.96e-2, FP8 V 2.64e-2, INT8 Q 2.06e-2 measured separately), so
# the 6e-2 target cannot be met with one scale per 128-token block there.
QUANT_VS_DEQUANT_RMSE = 3.6e-2   # RMS of a uniform +-2^-4 relative error on every P weight

QUANT_TARGET = [pytest.param("image"), pytest.param("video"),
                pytest.param("llm", marks=pytest.mark.xfail(
                    strict=True, reason="per-128-token-block INT8 K with 20x element outliers: "
                                        "the quantiser alone is 6.83e-2 from exact"))]


def _quant_case(name):
    from oracle import dequantize_qk, dequantize_v, quantize_qk_int8, quantize_v_fp8
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v, precision="quant")
    rows = sample_rows(w).numpy()
    ro, rl = oracle_for(w, q, k, v, rows=rows)
    qd = dequantize_qk(*quantize_qk_int8(q.float().numpy()))
    kd = dequantize_qk(*quantize_qk_int8(k.float().numpy()))
    vd = dequantize_v(*quantize_v_fp8(v.float().numpy()), w.kv_len)
    rq, rql = attention_f64(qd, kd, vd, causal=w.causal, start_pos=w.start_pos,
                            window_lo=w.window_lo, rows=rows)
    return o[:, :, rows], lse[:, :, rows], ro, rl, rq, rql


@pytest.mark.parametrize("name", QUANT_TARGET)
def test_quant_mode_target(name):
    o, lse, ro, rl, rq, rql = _quant_case(name)
    e = rel_rmse(o, ro)
    assert e <= QUANT_RMSE, f"{name} quant rel_rmse={e:.4f}"


@pytest.mark.parametrize("name", ["image", "video", "llm"])
def test_quant_mode_against_dequantised_oracle(name):
    o, lse, ro, rl, rq, rql = _quant_case(name)
    e = rel_rmse(o, rq)
    assert e <= QUANT_VS_DEQUANT_RMSE, f"{name}: rel_rmse vs dequantised oracle {e:.4f}"
    # lse comes from the float32 weights of the dequantised scores
    check_lse(lse, rql, name, tol=1e-3)


def _small(**kw):
    base = dict(name="small", batch=1, n_q_heads=4, n_kv_heads=2, q_len=4, kv_len=4096,
                head_dim=128, dtype="fp16", causal=True, start_pos=4092, seed=41)
    base.update(kw)
    return Workload(**base)


# query-row counts x start positions x key lengths x window bounds, in the spirit of
# the qsa2 audit's 40 position/window cases (partial chunks included)
BOUNDARY = []
for ntok in (1, 2, 4, 8):
    for pos0 in (0, 1, 63, 64, 127, 128, 129, 512, 2047, 2048, 2050, 4095):
        for kv_extra, win in ((1, 0), (0, 40), (37, 127)):
            kv_len = pos0 + ntok + kv_extra - 1
            win = min(win, max(pos0, 0))
            BOUNDARY.append((ntok, pos0, kv_len, win))


@pytest.mark.parametrize("ntok,pos0,kv_len,win", BOUNDARY)
def test_decode_boundary_matrix(ntok, pos0, kv_len, win):
    w = _small(q_len=ntok, start_pos=pos0, kv_len=kv_len, window_lo=win, seed=41 + pos0)
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v)
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, str((ntok, pos0, kv_len, win)))
    check_lse(lse, rl)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal,start_pos,window_lo,Sq,Skv", [
    (False, 0, 0, 1000, 1000),
    (True, 0, 0, 1000, 1000),
    (True, 0, 0, 777, 1291),
    (True, 300, 0, 700, 1000),
    (False, 0, 200, 513, 1111),
    (True, 0, 130, 1000, 1000),
    (True, 0, 0, 129, 129),
])
def test_single_pass_ragged(D, causal, start_pos, window_lo, Sq, Skv):
    w = Workload("ragged", 2, 4, 2, Sq, Skv, D, "bf16", causal=causal, start_pos=start_pos,
                 window_lo=window_lo, seed=7 + Sq)
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v, num_splits=1)
    assert att.num_splits == 1
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro)
    check_lse(lse, rl)


@pytest.mark.parametrize("splits", [2, 3, 7])
def test_forced_splits(splits):
    w = Workload("split", 1, 4, 1, 300, 2000, 128, "bf16", causal=True, start_pos=1700, seed=9)
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v, num_splits=splits)
    assert att.num_splits > 1
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro)
    check_lse(lse, rl)


@pytest.mark.parametrize("num_splits", [0, 1])
def test_rows_that_see_no_key(num_splits):
    # causal from position 0 with a window starting at key 5: rows 0..4 see nothing
    w = Workload("empty", 1, 2, 2, 300, 300, 64, "bf16", causal=True, window_lo=5, seed=3)
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v, num_splits=num_splits)
    assert np.all(o[:, :, :5] == 0) and np.all(lse[:, :, :5] == -math.inf)
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro)
    check_lse(lse, rl)


def test_zero_kv_len_and_window_past_end():
    w = Workload("nokv", 1, 2, 1, 5, 0, 128, "fp16")
    att = Attention(1, 2, 1, 5, 0, 128, dtype=torch.float16)
    q = torch.randn(1, 2, 5, 128, device="cuda").half()
    kv = torch.empty(1, 1, 0, 128, device="cuda").half()
    out = torch.full((1, 2, 5, 128), 7.0, device="cuda").half()
    out, lse = att.forward(q, kv, kv, out=out, return_lse=True)
    att.check_error()
    assert torch.all(out == 0) and torch.all(lse == -math.inf)
    w = Workload("pastend", 1, 2, 1, 5, 100, 128, "fp16", window_lo=100, seed=2)
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v)
    assert np.all(o == 0) and np.all(lse == -math.inf)


def test_deterministic():
    w = WORKLOADS["image"].scaled(batch=1)
    q, k, v = (t.cuda() for t in make_qkv(w))
    for precision in ("exact", "quant"):
        att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                        precision=precision)
        a = att.forward(q, k, v)
        b = att.forward(q, k, v)
        att.check_error()
        assert torch.equal(a, b)


def test_masked_keys_do_not_matter():
    w = Workload("mask", 1, 4, 2, 200, 700, 128, "bf16", causal=True, start_pos=300,
                 window_lo=77, seed=4)
    q, k, v = make_qkv(w)
    o1, l1, _ = run_gpu(w, q, k, v)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, :77] = 1e4
    v2[:, :, :77] = -3e4
    k2[:, :, 500:] = float("nan")   # beyond every row's causal limit (300 + 199)
    v2[:, :, 500:] = 3e4
    o2, l2, _ = run_gpu(w, q, k2, v2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_wait_timeout_is_reported_and_context_survives():
    from attention_forward_flash_b200 import _abi
    w = Workload("timeout", 1, 2, 2, 256, 1024, 64, "bf16", seed=8)
    q, k, v = (t.cuda() for t in make_qkv(w))
    att = Attention(1, 2, 2, 256, 1024, 64, num_splits=1)
    _abi.attn_debug_set(att.ctx, 1)
    att.forward(q, k, v)
    with pytest.raises(_abi.AttnError) as e:
        att.check_error()
    assert e.value.status == _abi.ATTN_ERR_TIMEOUT
    _abi.attn_debug_set(att.ctx, 0)
    o = att.forward(q, k, v)
    att.check_error()
    ro, _ = oracle_for(w, *(t.cpu() for t in (q, k, v)))
    check_exact(o.double().cpu().numpy(), ro)


@pytest.mark.parametrize("D", [64, 128])
def test_quantised_wait_timeout_is_reported_and_context_survives(D):
    """The same test hook in the quantised mode, whose kernel hands P to the MMA
    warp through shared memory and has waits of its own: the loader never loads
    the second key tile, every wait ends, the timeout is reported, and the next
    call is correct."""
    from attention_forward_flash_b200 import _abi
    w = Workload("timeout_q", 1, 2, 2, 512, 1024, D, "bf16", seed=9)
    q, k, v = (t.cuda() for t in make_qkv(w))
    att = Attention(1, 2, 2, 512, 1024, D, num_splits=1, precision="quant")
    qb = att.quantize(q, k, v)
    att.check_error()
    _abi.attn_debug_set(att.ctx, 1)
    att.forward(qbufs=qb)
    with pytest.raises(_abi.AttnError) as e:
        att.check_error()
    assert e.value.status == _abi.ATTN_ERR_TIMEOUT
    _abi.attn_debug_set(att.ctx, 0)
    o = att.forward(qbufs=qb)
    att.check_error()
    ro, _ = oracle_for(w, *(t.cpu() for t in (q, k, v)))
    assert rel_rmse(o.double().cpu().numpy(), ro) <= QUANT_RMSE


def test_polynomial_exp2_against_cuda_exp2():
    """The FMA-pipe exponential used for part of the softmax against torch's
    float32 exp2 on the GPU: relative error below 1e-4 on [-125, 126]."""
    from attention_forward_flash_b200 import _abi
    x = torch.cat([torch.linspace(-125, 126, 2_000_001, device="cuda"),
                   torch.rand(1_000_000, device="cuda") * -20,
                   torch.tensor([0.0, -0.5, 0.5, -1e-7, 1e-7, 8.0, -125.0], device="cuda")])
    y = torch.empty_like(x)
    _abi.attn_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    assert abs(y[-1].item() / 2.0 ** -125 - 1) < 1e-4
    z = torch.tensor([-200.0, float("-inf")], device="cuda")
    w = torch.empty_like(z)
    _abi.attn_debug_exp2(z.data_ptr(), w.data_ptr(), 2, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.all(w == y[-1])  # clamped to the value at -125


# Long contexts: one CTA runs 1024 key tiles (131072 keys) in the single-pass
# kernel (forced: the library would split a single unit of 1024 rows), and decode
# problems with 32768 keys reach the library's split count for a few rows (merge
# over ~37 partials, most of them empty under the window).
LONG = [
    ("long_prefill", Workload("long_prefill", 1, 2, 1, 512, 131072, 128, "bf16",
                              modes=("exact", "quant"), seed=5101, oracle_rows=64)),
    ("long_decode", Workload("long_decode", 1, 16, 8, 4, 32768, 128, "fp16", causal=True,
                             start_pos=32764, seed=5102)),
    ("long_decode_window", Workload("long_decode_window", 1, 16, 8, 1, 32768, 128, "fp16",
                                    causal=True, start_pos=32767, window_lo=28672, seed=5103)),
]


@pytest.mark.parametrize("name,w", LONG, ids=[n for n, _ in LONG])
def test_long_context_exact(name, w):
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v, num_splits=1 if name == "long_prefill" else 0)
    rows = sample_rows(w).numpy()
    ro, rl = oracle_for(w, q, k, v, rows=rows)
    check_exact(o[:, :, rows], ro, name)
    check_lse(lse[:, :, rows], rl, name)
    if name.startswith("long_decode"):
        assert att.num_splits > 8
    else:
        assert att.num_splits == 1


# The quantised mode on both kernels: the single-pass one (forced) and the
# split-KV one with its merge (the library's choice for these shapes).
@pytest.mark.parametrize("name,num_splits", [("long_prefill", 1), ("long_prefill", 0),
                                             ("long_decode", 0)])
def test_long_context_quant(name, num_splits):
    w = dict(LONG)[name]
    q, k, v = make_qkv(w)
    o, _, att = run_gpu(w, q, k, v, precision="quant", num_splits=num_splits)
    assert (att.num_splits == 1) == (num_splits == 1)
    rows = sample_rows(w).numpy()
    ro, _ = oracle_for(w, q, k, v, rows=rows)
    e = rel_rmse(o[:, :, rows], ro)
    assert e <= QUANT_RMSE, f"{name}: quantised rel_rmse {e:.3e}"


# Per-row sliding window (window_size W): row i at position p sees keys
# max(window_lo, p - W + 1) .. p.  Windows narrower than, equal to and wider
# than a key tile, crossing tile edges at ragged offsets, with and without
# window_lo, in the single-pass and split-KV kernels.
SLIDING = [
    # D, Sq, Skv, start_pos, W, window_lo, causal, num_splits
    (128, 700, 1291, 591, 1, 0, True, 1),
    (128, 700, 1291, 591, 64, 0, True, 1),
    (128, 700, 1291, 591, 127, 0, True, 1),
    (128, 700, 1291, 591, 128, 0, True, 0),
    (64, 700, 1291, 591, 129, 0, True, 1),
    (64, 700, 1291, 591, 300, 650, True, 1),
    (128, 1000, 1000, 0, 1000, 0, True, 1),
    (128, 1000, 1000, 0, 5000, 0, True, 0),
    (64, 513, 1111, 500, 300, 0, False, 1),
    (128, 4, 32768, 32764, 1, 0, True, 0),
    (128, 4, 32768, 32764, 100, 0, True, 0),
    (128, 1, 32768, 32767, 4096, 0, True, 0),
]


@pytest.mark.parametrize("D,Sq,Skv,start_pos,W,window_lo,causal,num_splits", SLIDING)
def test_sliding_window(D, Sq, Skv, start_pos, W, window_lo, causal, num_splits):
    w = Workload("sliding", 1, 8, 2, Sq, Skv, D, "bf16" if D == 64 else "fp16", causal=causal,
                 start_pos=start_pos, window_lo=window_lo, window_size=W, seed=6000 + W + Sq)
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v, num_splits=num_splits)
    if num_splits == 1:
        assert att.num_splits == 1
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, f"W={W}")
    check_lse(lse, rl, f"W={W}")


def test_sliding_window_quantised():
    w = Workload("sliding_q", 2, 8, 2, 700, 1291, 128, "bf16", causal=True, start_pos=591,
                 window_size=256, seed=6101)
    q, k, v = make_qkv(w)
    o, _, _ = run_gpu(w, q, k, v, precision="quant")
    ro, _ = oracle_for(w, q, k, v)
    assert rel_rmse(o, ro) <= QUANT_RMSE


# The qsa2 audit's decode matrix ("build and reproduction"): a 32768-cell KV cache,
# 1/2/4/8 query rows, first positions 0, 1, 63, 64, 512, 2047, 2048, 2050, 8192 and
# 30000 (causal: the cells past each row's position are masked), each with and
# without a 1024-position sliding window.
QSA2_CELLS = 32768
QSA2 = [(ntok, pos0, W) for ntok in (1, 2, 4, 8)
        for pos0 in (0, 1, 63, 64, 512, 2047, 2048, 2050, 8192, 30000) for W in (0, 1024)]


@pytest.mark.parametrize("ntok,pos0,W", QSA2)
def test_decode_qsa2_positions(ntok, pos0, W):
    w = _small(q_len=ntok, start_pos=pos0, kv_len=QSA2_CELLS, window_size=W,
               seed=41 + 7 * pos0 + ntok + W)
    q, k, v = make_qkv(w)
    o, lse, _ = run_gpu(w, q, k, v)
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, str((ntok, pos0, W)))
    check_lse(lse, rl)


# The lazy O correction of the exact mode: O and the row sums are rescaled only
# when a row maximum grows by more than 8 (base-2 units) over the maximum in use.
# Keys are built so that every 128-key tile raises each row's maximum by a set
# amount G: K[j, 0] = g * (j // 128) + N(0, 1) with Q[i, 0] = 4, the other channels
# small, so scale * log2(e) * 4 * g = G.  G = 7.5 stays under the threshold (the
# stale maximum is kept and P reaches 2^7.5), G = 8.5 and G = 20 cross it on every
# tile.  Single-pass kernel (head_dim 64 and 128) and split-KV kernel.
def _ramp_inputs(D, Sq, Skv, G, seed):
    g_ = torch.Generator().manual_seed(seed)
    q = torch.randn(1, 2, Sq, D, generator=g_) * 0.25
    k = torch.randn(1, 2, Skv, D, generator=g_) * 0.25
    v = torch.randn(1, 2, Skv, D, generator=g_)
    q[..., 0] = 4.0
    step = G / (4.0 * (1.0 / math.sqrt(D)) * math.log2(math.e))
    tile = torch.div(torch.arange(Skv), 128, rounding_mode="floor").float()
    k[..., 0] = step * tile + torch.randn(1, 2, Skv, generator=g_)
    return tuple(t.to(torch.bfloat16) for t in (q, k, v))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [7.5, 8.5, 20.0])
@pytest.mark.parametrize("path", ["single_pass", "split_merge", "decode"])
def test_exact_rescale_forced(D, G, path):
    # 300 rows: the single-pass kernel; 40 rows with 3 forced splits: the split-KV
    # kernel and its merge; 8 rows: the decode kernel (its own online softmax
    # rescales on every chunk whose maximum grows)
    Sq, splits = {"single_pass": (300, 1), "split_merge": (40, 3), "decode": (8, 3)}[path]
    Skv = 10 * 128 + 37
    q, k, v = _ramp_inputs(D, Sq, Skv, G, seed=int(7000 + 10 * G + D))
    w = Workload("ramp", 1, 2, 2, Sq, Skv, D, "bf16", seed=0)
    o, lse, att = run_gpu(w, q, k, v, num_splits=splits)
    assert att.kernel_path == path and att.num_splits == splits
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, f"G={G}")
    check_lse(lse, rl, f"G={G}")


# Short last wave of the single-pass grid: 40 units x 4 row tiles of 256 = 160 CTAs on
# 148 SMs would leave a last wave of 12 CTAs; their rows run instead on the split kernel
# (keys split across CTAs) and a merge.  Every row is checked against the oracle, lse
# included, in both modes; and with unit ranges (the host-buffer pipeline) the rows come
# out bit-identical to the whole-problem call.
TAIL = [Workload("tail_d64", 1, 40, 40, 1024, 1000, 64, "bf16", seed=9401),
        Workload("tail_gqa_d128", 2, 40, 10, 512, 777, 128, "fp16", window_lo=100, seed=9402)]


@pytest.mark.parametrize("w", TAIL, ids=[t.name for t in TAIL])
def test_short_last_wave_runs_on_the_split_kernel(w):
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v)
    assert att.kernel_path == "single_pass_tail"
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, w.name)
    check_lse(lse, rl, w.name)
    oq, _, attq = run_gpu(w, q, k, v, precision="quant")
    assert attq.kernel_path == "single_pass_tail"
    assert rel_rmse(oq, ro) <= QUANT_RMSE
    # the forced single-pass kernel agrees to rounding
    o1, _, att1 = run_gpu(w, q, k, v, num_splits=1)
    assert att1.kernel_path == "single_pass"
    check_exact(o1, ro, w.name + " single pass")


def test_tail_rows_bit_identical_across_unit_ranges():
    w = TAIL[0]
    q, k, v = make_qkv(w)
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype)
    assert att.kernel_path == "single_pass_tail"
    ref, rl = att.forward(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    att.check_error()
    for chunks in (3, 7):
        o, lse = att.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                  return_lse=True, chunks=chunks)
        torch.cuda.synchronize()
        att.check_error()
        assert torch.equal(o.view(torch.int16), ref.cpu().view(torch.int16)), chunks
        assert torch.equal(lse, rl.cpu()), chunks
