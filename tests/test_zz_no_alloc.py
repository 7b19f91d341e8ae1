"""The split-KV forward that allocates nothing, against the regular entry point.

``attn_forward_splitkv_noalloc`` is for callers that cannot call cudaMalloc
(device memory owned by another allocator, or a latency-critical decode step
that cannot take cudaMalloc's implicit synchronisation): it keeps its split
partials in a fixed array inside the library instead of a context workspace.
Its output must match the float64 oracle and ``attn_forward`` (through
``attn_create``) within the exact-mode tolerances the other tests use, on two
calls in a row with a different problem run through the same array in between
(the array keeps the previous call's contents).  This file is collected last.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention, _abi
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv
from oracle import attention_f64

pytestmark = pytest.mark.gpu

RMSE, MAXABS = 5e-3, 2e-2   # exact-mode tolerances of the parity tests


def _params(w, num_splits=0):
    return _abi.AttnParams(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                           w.start_pos, int(w.causal), w.window_lo, 0.0,
                           _abi.ATTN_FP16 if w.dtype == "fp16" else _abi.ATTN_BF16,
                           _abi.ATTN_EXACT, num_splits, w.window_size)


def _noalloc(w, q, k, v, err=None):
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream().cuda_stream
    _abi.attn_forward_splitkv_noalloc(_params(w), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      o.data_ptr(), lse.data_ptr(),
                                      err.data_ptr() if err is not None else None, stream)
    return o, lse


def _compare(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    e = np.linalg.norm(a - b) / np.linalg.norm(b)
    m = np.abs(a - b).max()
    assert e <= RMSE and m <= MAXABS, (e, m)


CASES = {
    "decode": WORKLOADS["decode"],
    "decode_window": WORKLOADS["decode_window"],
    "bf16_gqa": Workload("bf16_gqa", 2, 8, 2, 16, 3000, 64, "bf16", causal=True, start_pos=2984,
                         window_lo=100, seed=21),
    # per-row sliding window of 1000 positions over a 32768-key cache
    "sliding": Workload("sliding", 1, 8, 4, 3, 32768, 128, "fp16", causal=True, start_pos=32765,
                        window_size=1000, seed=23),
}
# a problem of another shape (more rows, more splits) run through the array between
# the two compared calls, so that its leftovers differ from what the next call writes
OTHER = {"decode": "bf16_gqa", "decode_window": "sliding", "bf16_gqa": "decode",
         "sliding": "decode_window"}


def _check(o, lse, ro, rl):
    _compare(o, torch.from_numpy(ro))
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(lse.cpu().numpy()), fin)
    assert np.abs(lse.cpu().numpy()[fin] - rl[fin]).max() <= 1e-3


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_oracle_and_attn_forward_on_two_calls(name):
    w = CASES[name]
    q, k, v = make_qkv(w)
    ro, rl = attention_f64(q, k, v, causal=w.causal, start_pos=w.start_pos,
                           window_lo=w.window_lo, window_size=w.window_size)
    q, k, v = (t.cuda() for t in (q, k, v))
    att = Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                    dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                    window_lo=w.window_lo, window_size=w.window_size)
    ref, ref_lse = att.forward(q, k, v, return_lse=True)
    att.check_error()
    wo = CASES[OTHER[name]]
    qo, ko, vo = (t.cuda() for t in make_qkv(wo.scaled(seed=wo.seed + 100)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = _noalloc(w, q, k, v, err)
    _noalloc(wo, qo, ko, vo, err)          # leaves another problem's partials behind
    o2, l2 = _noalloc(w, q, k, v, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for o, l in ((o1, l1), (o2, l2)):
        _check(o, l, ro, rl)               # against the float64 oracle
        _compare(o, ref)                   # and against attn_forward
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(l), fin)
        assert (l[fin] - ref_lse[fin]).abs().max().item() <= 1e-3
    # the later call saw another problem's leftovers in the array and does not depend on them
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_noalloc_rejects_problems_larger_than_its_array():
    w = Workload("big", 1, 64, 64, 128, 32768, 128, "bf16")
    q = torch.empty((1, 64, 128, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.empty((1, 64, 32768, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_abi.AttnError) as e:
        _noalloc(w, q, kv, kv)
    assert e.value.status == _abi.ATTN_ERR_UNSUPPORTED


def test_noalloc_rejects_the_quantised_mode():
    w = WORKLOADS["decode"]
    p = _params(w)
    p.precision = _abi.ATTN_INT8QK_FP8PV
    t = torch.empty(16, dtype=torch.float16, device="cuda")
    status = _abi.lib().attn_forward_splitkv_noalloc(ctypes.byref(p), t.data_ptr(), t.data_ptr(),
                                                     t.data_ptr(), t.data_ptr(), None, None, None)
    assert status == _abi.ATTN_ERR_UNSUPPORTED
