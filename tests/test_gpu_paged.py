"""The paged key/value cache (``attn_forward_paged``) against the dense entry point
and the oracle.

K and V of every (batch entry, kv head) are scattered into a pool of 128-position
blocks through a random block table, with spare blocks that nobody references and
large finite values past kv_len in each entry's last block.  Only the addresses
of the key/value tiles differ from ``attn_forward`` on the dense tensors, so the
outputs must be bit-identical to it; one case also goes to the oracle through its
own gather (``oracle.gather_paged``).
"""

import pytest
import torch

from attention_forward_flash_b200 import Attention, _abi
from attention_forward_flash_b200.inputs import Workload, make_qkv
from oracle import gather_paged
from parity_util import check_exact, check_lse, oracle_for

pytestmark = pytest.mark.gpu


def _att(w, precision="exact", num_splits=0):
    return Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                     dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                     window_lo=w.window_lo, precision=precision, num_splits=num_splits,
                     window_size=w.window_size)


def _paged(k, v, seed, spare=5):
    """Pool [blocks, Hkv, 128, D] and int32 table [B, ceil(S/128)] holding k, v."""
    B, Hkv, S, D = k.shape
    nbt = -(-S // 128)
    g = torch.Generator().manual_seed(seed)
    nblocks = B * nbt + spare
    table = torch.randperm(nblocks, generator=g)[:B * nbt].reshape(B, nbt).to(torch.int32)
    kp = torch.full((nblocks, Hkv, 128, D), 3e3, dtype=k.dtype)   # finite filler
    vp = torch.full((nblocks, Hkv, 128, D), -3e3, dtype=v.dtype)
    for b in range(B):
        for t in range(nbt):
            m = min(128, S - 128 * t)
            kp[table[b, t], :, :m] = k[b, :, 128 * t:128 * t + m]
            vp[table[b, t], :, :m] = v[b, :, 128 * t:128 * t + m]
    return kp, vp, table


def _same(a, b, what):
    assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), what


CASES = [
    # prefill, single pass, GQA, causal with a ragged key length
    Workload("paged_prefill", 2, 8, 2, 700, 1291, 128, "fp16", causal=True, start_pos=591,
             seed=7101),
    # head_dim 64, bf16, non-causal, window lower bound
    Workload("paged_d64", 3, 4, 4, 300, 1000, 64, "bf16", window_lo=77, seed=7102),
    # decode shape (split-KV path) on a long cache, with a sliding window
    Workload("paged_decode", 2, 16, 8, 4, 32768, 128, "fp16", causal=True, start_pos=32764,
             window_size=4096, seed=7103),
    # decode without a window, partial last block
    Workload("paged_decode_ragged", 1, 16, 8, 1, 4133, 128, "fp16", causal=True,
             start_pos=4132, seed=7104),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_paged_bit_identical_to_dense(w):
    q, k, v = make_qkv(w)
    kp, vp, table = _paged(k, v, w.seed)
    att = _att(w)
    qd = q.cuda()
    ro, rl = att.forward(qd, k.cuda(), v.cuda(), return_lse=True)
    o, lse = att.forward_paged(qd, kp.cuda(), vp.cuda(), table.cuda(), return_lse=True)
    att.check_error()
    _same(o.cpu(), ro.cpu(), f"{w.name}: O")
    _same(lse.cpu(), rl.cpu(), f"{w.name}: lse")


def test_paged_against_oracle_gather():
    w = CASES[0]
    q, k, v = make_qkv(w)
    kp, vp, table = _paged(k, v, w.seed)
    att = _att(w)
    o, lse = att.forward_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), return_lse=True)
    att.check_error()
    kg = torch.from_numpy(gather_paged(kp, table, w.kv_len))
    vg = torch.from_numpy(gather_paged(vp, table, w.kv_len))
    ro, rl = oracle_for(w, q, kg, vg)
    check_exact(o.double().cpu().numpy(), ro, "paged")
    check_lse(lse.cpu().numpy(), rl, "paged")


def test_paged_argument_errors():
    w = CASES[1]
    q, k, v = make_qkv(w)
    kp, vp, table = _paged(k, v, 1)
    L = _abi.lib()
    s = torch.cuda.current_stream().cuda_stream
    qd, kd, vd, td = q.cuda(), kp.cuda(), vp.cuda(), table.cuda()
    o = torch.empty_like(qd)
    att = _att(w)
    P = lambda t: t.data_ptr()  # noqa: E731
    assert L.attn_forward_paged(att.ctx, P(qd), P(kd), P(vd), None, kd.shape[0], P(o), None,
                                s) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_forward_paged(att.ctx, P(qd), P(kd), P(vd), P(td), 0, P(o), None,
                                s) == _abi.ATTN_ERR_INVALID_ARG
    attq = _att(w, precision="quant")
    assert L.attn_forward_paged(attq.ctx, P(qd), P(kd), P(vd), P(td), kd.shape[0], P(o), None,
                                s) == _abi.ATTN_ERR_UNSUPPORTED
    assert L.attn_forward_paged(att.ctx, P(qd), P(kd), P(vd), P(td), kd.shape[0], P(o), None,
                                s) == _abi.ATTN_OK
    att.check_error()


QUANT_CASES = [
    Workload("pq_gqa_causal", 2, 8, 2, 300, 1291, 128, "bf16", causal=True, start_pos=991,
             seed=7201),
    Workload("pq_d64", 1, 4, 4, 256, 1000, 64, "fp16", seed=7202),
    Workload("pq_decode", 2, 16, 8, 4, 4133, 128, "fp16", causal=True, start_pos=4129,
             seed=7203),
]


@pytest.mark.parametrize("w", QUANT_CASES, ids=[w.name for w in QUANT_CASES])
def test_paged_quantised_mode(w):
    """The INT8 mode on a paged cache: the quantisers read K and V through the block
    table (``attn_quantize_qk_paged``) and write the same codes and scales as on the
    gathered dense tensors, bit for bit (the pool's filler past kv_len is never read);
    the attention on them is identical and within the quantised mode's tolerance of
    the oracle."""
    from parity_util import QUANT_RMSE, rel_rmse
    q, k, v = make_qkv(w)
    kp, vp, table = _paged(k, v, w.seed)
    att = _att(w, precision="quant")
    qd = q.cuda()
    dense = att.quantize(qd, k.cuda(), v.cuda())
    paged = att.quantize_paged(qd, kp.cuda(), vp.cuda(), table.cuda())
    att.check_error()
    for f in ("q", "k", "q_scale", "k_scale", "v_t", "v_scale"):
        _same(getattr(paged, f).cpu(), getattr(dense, f).cpu(), f"{w.name}: {f}")
    o_p = att.forward(qbufs=paged)
    o_d = att.forward(qbufs=dense)
    att.check_error()
    _same(o_p.cpu(), o_d.cpu(), f"{w.name}: O")
    ro, _ = oracle_for(w, q, k, v)
    assert rel_rmse(o_p.double().cpu().numpy(), ro) <= QUANT_RMSE


def test_paged_quantiser_argument_errors():
    w = QUANT_CASES[1]
    q, k, v = make_qkv(w)
    kp, vp, table = _paged(k, v, 1)
    L = _abi.lib()
    s = torch.cuda.current_stream().cuda_stream
    qd, kd, vd, td = q.cuda(), kp.cuda(), vp.cuda(), table.cuda()
    att = _att(w, precision="quant")
    qb = att.quantize(qd, k.cuda(), v.cuda())
    P = lambda t: t.data_ptr()  # noqa: E731
    import ctypes
    qbs = qb.struct()
    st = ctypes.byref(qbs)
    assert L.attn_quantize_qk_paged(att.ctx, P(qd), P(kd), P(vd), None, kd.shape[0], st,
                                    s) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_quantize_qk_paged(att.ctx, P(qd), P(kd), P(vd), P(td), 0, st,
                                    s) == _abi.ATTN_ERR_INVALID_ARG
    exact = _att(w)
    assert L.attn_quantize_qk_paged(exact.ctx, P(qd), P(kd), P(vd), P(td), kd.shape[0], st,
                                    s) == _abi.ATTN_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        exact.quantize_paged(qd, kd, vd, td)
    # the binding checks q and the caller's output buffers before any call
    with pytest.raises(ValueError):
        att.quantize_paged(qd[:, :1], kd, vd, td)
    with pytest.raises(ValueError):
        exact.forward_paged(qd, kd, vd, td, out=torch.empty_like(qd, dtype=torch.float32))
    with pytest.raises(ValueError):
        att.forward(qbufs=qb, lse=torch.empty(1, device="cuda"))
    assert L.attn_quantize_qk_paged(att.ctx, P(qd), P(kd), P(vd), P(td), kd.shape[0], st,
                                    s) == _abi.ATTN_OK
    att.check_error()
    # a table entry past the pool is read as block 0 and reported by attn_get_error
    bad = td.clone()
    bad[0, 0] = kd.shape[0]
    assert L.attn_quantize_qk_paged(att.ctx, P(qd), P(kd), P(vd), P(bad), kd.shape[0], st,
                                    s) == _abi.ATTN_OK
    assert L.attn_get_error(att.ctx, s) == _abi.ATTN_ERR_INVALID_ARG
    assert L.attn_get_error(att.ctx, s) == _abi.ATTN_OK
    bad[0, 0] = -1
    assert L.attn_quantize_qk_paged(att.ctx, P(qd), P(kd), P(vd), P(bad), kd.shape[0], st,
                                    s) == _abi.ATTN_OK
    assert L.attn_get_error(att.ctx, s) == _abi.ATTN_ERR_INVALID_ARG
    att.check_error()
