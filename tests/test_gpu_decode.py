"""The decode kernel (``ATTN_PATH_DECODE``: exact mode, at most 16 stacked query rows
per kv head) against the float64 oracle.

It runs for decode-shaped problems (a few query rows at a start position against a
long key/value cache: the page "perf(metal): widen four-row flash KV tiles - #89",
"Performance evidence"), splitting the rows' visible keys across the CTAs of one
thread-block cluster per (batch, kv head) and merging them in the same launch.  The
cases cover 1 to 16 stacked rows, both head sizes and 16-bit types, causal and
non-causal masks, start positions, window bounds and sliding windows, ragged key
lengths (a partial last chunk), the library's split choice and forced splits up to
the cluster limit, rows that see no key, RoPE, a paged cache whose unused positions
hold NaN, and the bounded-wait error path.  Tolerances are the exact mode's.
"""

import math

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention, _abi
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv
from oracle import gather_paged
from parity_util import check_exact, check_lse, oracle_for, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # name, workload, num_splits
    ("decode", WORKLOADS["decode"], 0),
    ("decode_window", WORKLOADS["decode_window"], 0),
    ("r1_d64", Workload("r1", 1, 4, 4, 1, 777, 64, "bf16", causal=True, start_pos=776, seed=9301), 0),
    ("r16_d64_noncausal", Workload("r16", 3, 32, 2, 1, 2000, 64, "fp16", seed=9302), 0),
    ("r16_forced16", Workload("f16", 1, 8, 1, 2, 5000, 128, "bf16", causal=True, start_pos=4998,
                              seed=9303), 16),
    ("r10_forced7", Workload("f7", 2, 6, 3, 5, 1000, 128, "fp16", causal=True, start_pos=995,
                             seed=9304), 7),
    ("forced2", Workload("f2", 1, 4, 2, 4, 3000, 64, "bf16", causal=True, start_pos=2996,
                         seed=9305), 2),
    ("few_keys", Workload("fk", 1, 2, 2, 3, 100, 128, "bf16", causal=True, start_pos=97,
                          seed=9306), 0),
    ("window_lo", Workload("wl", 1, 4, 2, 4, 3000, 128, "bf16", causal=True, start_pos=2996,
                           window_lo=1500, seed=9307), 0),
    ("sliding_noncausal", Workload("sn", 1, 4, 2, 4, 3000, 64, "fp16", start_pos=1000,
                                   window_size=700, seed=9308), 0),
    ("chunked_prefill_tail", Workload("ct", 2, 2, 1, 7, 4099, 128, "bf16", causal=True,
                                      start_pos=2000, seed=9309), 0),
    ("long_cache", Workload("lc", 1, 8, 8, 1, 65536, 128, "fp16", causal=True, start_pos=65535,
                            seed=9310), 0),
]


@pytest.mark.parametrize("name,w,splits", CASES, ids=[c[0] for c in CASES])
def test_decode_kernel_against_oracle(name, w, splits):
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v, num_splits=splits)
    assert att.kernel_path == "decode"
    if splits:
        assert att.num_splits == splits
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro, name)
    check_lse(lse, rl, name)


def test_rows_that_see_no_key():
    # causal from position 0 with keys from 5 on: the rows at positions 0..4 see nothing
    w = Workload("empty", 1, 2, 2, 8, 300, 64, "bf16", causal=True, window_lo=5, seed=9320)
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v)
    assert att.kernel_path == "decode"
    assert np.all(o[:, :, :5] == 0) and np.all(lse[:, :, :5] == -math.inf)
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o, ro)
    check_lse(lse, rl)
    # no row sees any key: every output row is 0, lse -inf
    w = Workload("none", 1, 4, 2, 4, 300, 128, "fp16", causal=True, start_pos=50, window_lo=200,
                 seed=9321)
    q, k, v = make_qkv(w)
    o, lse, att = run_gpu(w, q, k, v)
    assert att.kernel_path == "decode"
    assert np.all(o == 0) and np.all(lse == -math.inf)


def test_single_pass_when_forced_and_split_merge_past_the_cluster_limit():
    w = Workload("paths", 1, 16, 8, 4, 4096, 128, "fp16", causal=True, start_pos=4092, seed=9322)
    q, k, v = make_qkv(w)
    ro, rl = oracle_for(w, q, k, v)
    for splits, path in ((1, "single_pass"), (32, "split_merge"), (16, "decode")):
        o, lse, att = run_gpu(w, q, k, v, num_splits=splits)
        assert att.kernel_path == path, (splits, att.kernel_path)
        check_exact(o, ro, path)
        check_lse(lse, rl, path)


def test_paged_cache_with_nan_past_the_end():
    """A paged cache whose positions past kv_len (in the last block) hold NaN: those
    keys are masked and their values must not reach O (0 * NaN is NaN)."""
    w = Workload("pn", 2, 16, 8, 4, 4133, 128, "bf16", causal=True, start_pos=4129, seed=9323)
    q, k, v = make_qkv(w)
    B, Hkv, S, D = k.shape
    nbt = -(-S // 128)
    g = torch.Generator().manual_seed(3)
    table = torch.randperm(B * nbt + 2, generator=g)[:B * nbt].reshape(B, nbt).to(torch.int32)
    kp = torch.full((B * nbt + 2, Hkv, 128, D), float("nan"), dtype=k.dtype)
    vp = torch.full_like(kp, float("nan"))
    for b in range(B):
        for t in range(nbt):
            m = min(128, S - 128 * t)
            kp[table[b, t], :, :m] = k[b, :, 128 * t:128 * t + m]
            vp[table[b, t], :, :m] = v[b, :, 128 * t:128 * t + m]
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype, causal=True, start_pos=w.start_pos)
    assert att.kernel_path == "decode"
    o, lse = att.forward_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), return_lse=True)
    att.check_error()
    assert torch.isfinite(o).all()
    ro, rl = oracle_for(w, q, torch.from_numpy(gather_paged(kp, table, S)),
                        torch.from_numpy(gather_paged(vp, table, S)))
    check_exact(o.double().cpu().numpy(), ro, "paged NaN")
    check_lse(lse.cpu().numpy(), rl, "paged NaN")


def test_decode_wait_timeout_is_reported_and_context_survives():
    """The test hook makes warp 0 of the first CTA never load its second key chunk:
    its wait runs out, the kernel records ATTN_ERR_TIMEOUT, every CTA still reaches
    the cluster barriers, and the next call on the same context is correct."""
    w = Workload("timeout_d", 1, 4, 2, 4, 4096, 128, "bf16", causal=True, start_pos=4092,
                 seed=9324)
    q, k, v = (t.cuda() for t in make_qkv(w))
    att = Attention(1, 4, 2, 4, 4096, 128, causal=True, start_pos=4092, num_splits=2)
    assert att.kernel_path == "decode"
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


def test_graph_captured_calls_then_destroy_leave_no_error():
    """A forward captured into a CUDA graph and replayed, then the context destroyed:
    the next context's calls report no error (the context's completion event is not
    recorded inside a capture, and destroying it leaves no pending CUDA error)."""
    w = WORKLOADS["decode"]
    q, k, v = (t.cuda() for t in make_qkv(w))
    ro, rl = oracle_for(w, *(t.cpu() for t in (q, k, v)))
    for splits in (0, 32):   # the decode kernel, then the split-KV kernel and its merge
        att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                        dtype=w.torch_dtype, causal=True, start_pos=w.start_pos,
                        num_splits=splits)
        out = torch.empty_like(q)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            att.forward(q, k, v, out=out)
            s.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                att.forward(q, k, v, out=out)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        att.check_error()
        check_exact(out.double().cpu().numpy(), ro, f"graph replay, num_splits={splits}")
        del g
        del att
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype, causal=True, start_pos=w.start_pos, num_splits=32)
    o, lse = att.forward(q, k, v, return_lse=True)
    att.check_error()
    check_exact(o.double().cpu().numpy(), ro, "after destroy")


@pytest.mark.parametrize("R_rope,inter,G,Sq", [(64, True, 2, 4), (128, False, 4, 3),
                                               (96, False, 1, 1)],
                         ids=["interleaved_partial_8rows", "half_12rows", "partial_1row"])
def test_decode_kernel_with_rope(R_rope, inter, G, Sq):
    """Q rotated in the decode kernel's staged rows (keys rotated once by the call):
    against float64 attention on float64-rotated Q and K, both pair layouts, a partial
    rotary width, the transposed (<= 8 rows) and the row-major (9..16 rows) products."""
    from oracle import apply_rope, rope_frequencies
    from oracle import rope_table as oracle_table
    w = Workload("dr", 2, 4 * G, 4, Sq, 3000, 128, "bf16", causal=True, start_pos=3000 - Sq,
                 seed=9330 + R_rope + G)
    q, k, v = make_qkv(w)
    theta = rope_frequencies(R_rope, scaling="ntk", factor=4.0)
    table = oracle_table(3000, theta)
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype, causal=True, start_pos=w.start_pos, rope_dim=R_rope,
                    rope_interleaved=inter, rope_table=torch.from_numpy(table))
    assert att.kernel_path == "decode"
    o = att.forward(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    layout = "interleaved" if inter else "half"
    qr = apply_rope(q.double().numpy(), w.start_pos + np.arange(Sq), theta, layout=layout)
    kr = apply_rope(k.double().numpy(), np.arange(3000), theta, layout=layout)
    from oracle import attention_f64
    ro, _ = attention_f64(qr, kr, v.double().numpy(), causal=True, start_pos=w.start_pos)
    check_exact(o.double().cpu().numpy(), ro, f"rope R={R_rope}")
