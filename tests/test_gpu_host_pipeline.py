"""The host-buffer entry point ``attn_forward_host`` against the device one.

``attn_forward_host`` copies Q, K and V from host memory, runs the same kernels
as ``attn_quantize_qk`` / ``attn_forward`` on contiguous ranges of units (batch
entry x kv head) and copies O and lse back, with the copies of one range
overlapping the kernels of its neighbours.  Each unit's rows are computed by the
same code whichever range it falls in, so its outputs must be bit-identical to
``attn_forward``'s on the same inputs, for every range count, in both modes and
on the split-KV path.  One case also goes to the oracle directly, and one runs
at the full size of the largest workload, in the launch configuration the
benchmark's end-to-end leg uses.
"""

import ctypes

import pytest
import torch

from attention_forward_flash_b200 import Attention, DeviceStaging, _abi
from attention_forward_flash_b200.inputs import WORKLOADS, Workload, make_qkv
from parity_util import check_exact, check_lse, oracle_for

pytestmark = pytest.mark.gpu


def _att(w, precision="exact", num_splits=0):
    return Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                     dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                     window_lo=w.window_lo, precision=precision, num_splits=num_splits,
                     window_size=w.window_size)


def _device_result(att, q, k, v):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    if att.precision == "quant":
        qb = att.quantize(qd, kd, vd)
        o, lse = att.forward(qbufs=qb, return_lse=True)
    else:
        qb = None
        o, lse = att.forward(qd, kd, vd, return_lse=True)
    att.check_error()
    return o.cpu(), lse.cpu(), qb


def _host_result(att, q, k, v, chunks, pin=True):
    if pin:
        q, k, v = (t.pin_memory() for t in (q, k, v))
    o = torch.empty(q.shape, dtype=q.dtype, pin_memory=pin)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=pin)
    st = DeviceStaging(att.params, att.dtype, torch.device("cuda"), att.precision == "quant",
                       True)
    # poison the staging and the host outputs: every byte must be written by the call
    for t in (st.o, st.lse, o, lse):
        t.view(torch.uint8).fill_(0xFF)
    att.forward_host(q, k, v, out=o, lse=lse, staging=st, chunks=chunks)
    att.check_error()
    return o, lse, st


def _same(a, b, what):
    assert a.shape == b.shape
    assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), what


SMALL = {
    # GQA, causal with a start position, a window, ragged key and query lengths
    "gqa_causal": Workload("gqa_causal", 4, 8, 2, 700, 1291, 128, "fp16", causal=True,
                           start_pos=591, window_lo=130, seed=4101),
    "mha_d64": Workload("mha_d64", 2, 10, 10, 1000, 1000, 64, "bf16", seed=4102),
}
# Both take the single-pass kernel (no key split), the path that is cut into ranges.
SINGLE_PASS = 1


@pytest.mark.parametrize("chunks", [0, 1, 2, 3, 5, 64])
@pytest.mark.parametrize("name", ["gqa_causal", "mha_d64"])
def test_exact_bit_identical_to_device_entry(name, chunks):
    w = SMALL[name]
    q, k, v = make_qkv(w)
    att = _att(w, num_splits=SINGLE_PASS)
    ro, rl, _ = _device_result(att, q, k, v)
    o, lse, _ = _host_result(att, q, k, v, chunks)
    _same(o, ro, f"{name} chunks={chunks}: O")
    _same(lse, rl, f"{name} chunks={chunks}: lse")


@pytest.mark.parametrize("chunks", [1, 3, 6])
def test_quant_bit_identical_to_device_entry(chunks):
    w = SMALL["gqa_causal"]
    q, k, v = make_qkv(w)
    att = _att(w, "quant", num_splits=SINGLE_PASS)
    ro, rl, rqb = _device_result(att, q, k, v)
    o, lse, st = _host_result(att, q, k, v, chunks)
    for f in ("q", "k", "q_scale", "k_scale", "v_t", "v_scale"):
        _same(getattr(st.qbufs, f).cpu(), getattr(rqb, f).cpu(), f"chunks={chunks}: {f}")
    _same(o, ro, f"chunks={chunks}: O")
    _same(lse, rl, f"chunks={chunks}: lse")


def test_split_path_and_pageable_memory():
    w = WORKLOADS["decode_window"]
    q, k, v = make_qkv(w)
    att = _att(w)
    assert att.num_splits > 1
    ro, rl, _ = _device_result(att, q, k, v)
    o, lse, _ = _host_result(att, q, k, v, chunks=4, pin=False)  # one range on this path
    _same(o, ro, "split path O")
    _same(lse, rl, "split path lse")


def test_against_oracle_through_the_wrapper():
    w = SMALL["gqa_causal"]
    q, k, v = make_qkv(w)
    att = _att(w)
    assert att.num_splits == 1
    o, lse = att.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), return_lse=True,
                              chunks=3)
    torch.cuda.current_stream().synchronize()
    ro, rl = oracle_for(w, q, k, v)
    check_exact(o.double().numpy(), ro, "forward_host")
    check_lse(lse.numpy(), rl, "forward_host")


def test_repeated_calls_reuse_the_pipeline():
    w = SMALL["mha_d64"]
    att = _att(w, num_splits=SINGLE_PASS)
    ref = None
    for seed in (4201, 4202, 4201):
        q, k, v = make_qkv(w.scaled(seed=seed))
        o = att.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), chunks=4)
        torch.cuda.current_stream().synchronize()
        if seed == 4201 and ref is None:
            ref = o.clone()
    _same(o, ref, "same inputs, same outputs after another call in between")


def test_argument_errors():
    w = SMALL["mha_d64"]
    att = _att(w)
    st = DeviceStaging(att.params, att.dtype, torch.device("cuda"), False, True)
    q, k, v = (torch.zeros(t.shape, dtype=t.dtype) for t in (st.q, st.k, st.v))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32)
    L = _abi.lib()
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731

    def call(chunks=0, lse_host=P(lse), lse_dev=P(st.lse), q_host=P(q), o_dev=P(st.o), qb=None):
        return L.attn_forward_host(att.ctx, q_host, P(k), P(v), P(o), lse_host, P(st.q), P(st.k),
                                   P(st.v), o_dev, lse_dev, qb, chunks, s)

    assert call(chunks=-1) == _abi.ATTN_ERR_INVALID_ARG
    assert call(chunks=65) == _abi.ATTN_ERR_INVALID_ARG
    assert call(lse_dev=None) == _abi.ATTN_ERR_INVALID_ARG
    assert call(lse_host=None) == _abi.ATTN_ERR_INVALID_ARG
    assert call(q_host=None) == _abi.ATTN_ERR_INVALID_ARG
    assert call(o_dev=P(st.o) + 8) == _abi.ATTN_ERR_INVALID_ARG
    qb = _abi.AttnQBufs(P(st.q), P(st.k), P(st.lse), P(st.lse), P(st.v), P(st.lse))
    assert call(qb=ctypes.byref(qb)) == _abi.ATTN_ERR_INVALID_ARG  # qb in exact mode
    assert call(chunks=2) == _abi.ATTN_OK
    att.check_error()


def test_full_size_video_default_chunks():
    """The largest workload, 1 GB of inputs, in the benchmark's end-to-end configuration."""
    w = WORKLOADS["video"]
    g = torch.Generator(device="cuda").manual_seed(4301)
    shape = (w.batch, w.n_q_heads, w.q_len, w.head_dim)
    qd, kd, vd = (torch.randn(shape, generator=g, device="cuda", dtype=torch.bfloat16)
                  for _ in range(3))
    att = _att(w)
    ro = att.forward(qd, kd, vd)
    att.check_error()
    q, k, v = (t.cpu().pin_memory() for t in (qd, kd, vd))
    del qd, kd, vd
    o = att.forward_host(q, k, v)
    torch.cuda.current_stream().synchronize()
    att.check_error()
    _same(o, ro.cpu(), "video O")


def test_sliding_window_bit_identical_to_device_entry():
    w = Workload("gqa_sliding", 4, 8, 2, 700, 1291, 128, "fp16", causal=True, start_pos=591,
                 window_size=200, seed=4103)
    q, k, v = make_qkv(w)
    att = _att(w, num_splits=SINGLE_PASS)
    ro, rl, _ = _device_result(att, q, k, v)
    o, lse, _ = _host_result(att, q, k, v, chunks=3)
    _same(o, ro, "sliding window O")
    _same(lse, rl, "sliding window lse")
