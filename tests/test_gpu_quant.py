"""The GPU quantisers (called through the C ABI) against the reference
quantiser of the oracle: INT8 codes, E4M3 codes and float32 scales must be
identical byte for byte."""

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention
from attention_forward_flash_b200.inputs import WORKLOADS, make_qkv
from oracle import quantize_qk_int8, quantize_v_fp8

pytestmark = pytest.mark.gpu


def _check_quant(q, k, v, dtype):
    B, Hq, Sq, D = q.shape
    Hk, Sk = k.shape[1], k.shape[2]
    att = Attention(B, Hq, Hk, Sq, Sk, D, dtype=dtype, precision="quant")
    qb = att.quantize(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    rq, rqs = quantize_qk_int8(q.float().numpy())
    rk, rks = quantize_qk_int8(k.float().numpy())
    rv, rvs = quantize_v_fp8(v.float().numpy())
    assert np.array_equal(qb.q_scale.cpu().numpy().view(np.uint32), rqs.view(np.uint32))
    assert np.array_equal(qb.k_scale.cpu().numpy().view(np.uint32), rks.view(np.uint32))
    assert np.array_equal(qb.v_scale.cpu().numpy().view(np.uint32), rvs.view(np.uint32))
    gq, gk, gv = qb.q.cpu().numpy(), qb.k.cpu().numpy(), qb.v_t.cpu().numpy()
    for name, g, r in (("q", gq, rq), ("k", gk, rk), ("v_t", gv, rv)):
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)
            i = tuple(bad[0])
            raise AssertionError(f"{name}: {len(bad)} codes differ, first at {i}: "
                                 f"gpu {g[i]} oracle {r[i]}")


@pytest.mark.parametrize("shape,dtype", [
    ((1, 2, 1, 256, 256, 64), torch.bfloat16),
    ((2, 4, 2, 300, 300, 128), torch.float16),
    ((1, 16, 8, 4, 4133, 128), torch.float16),
    ((1, 2, 1, 129, 1, 64), torch.bfloat16),
])
def test_quantiser_bit_exact_random(shape, dtype):
    B, Hq, Hk, Sq, Sk, D = shape
    g = torch.Generator().manual_seed(5)
    q = (torch.randn(B, Hq, Sq, D, generator=g) * 3).to(dtype)
    k = (torch.randn(B, Hk, Sk, D, generator=g) * 0.01).to(dtype)
    v = torch.randn(B, Hk, Sk, D, generator=g).to(dtype)
    _check_quant(q, k, v, dtype)


def test_quantiser_ties_zero_blocks_and_signed_zero():
    D = 64
    q = torch.zeros(1, 1, 300, D)
    # block 0: amax 127 -> s = 1; half-integers exercise round-half-even
    q[0, 0, 0, 0] = 127.0
    q[0, 0, 1, :8] = torch.tensor([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -126.5])
    # block 1 stays all zero; block 2 (partial, 44 tokens) has amax 254 -> s = 2
    q[0, 0, 256, 0] = 254.0
    q[0, 0, 257, :3] = torch.tensor([1.0, 3.0, 5.0])
    k = q.clone()
    v = torch.zeros(1, 1, 300, D)
    v[0, 0, 0, :] = 448.0                       # s = 1 on every channel
    mids = torch.tensor([1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, -1.0625, 2.0 ** -11,
                         -(2.0 ** -11), 0.0])
    v[0, 0, 1, :8] = mids                       # ties, a value that rounds to -0
    v[0, 0, 2, :] = -0.0
    v[0, 0, :, 63] = 0.0                        # an all-zero channel
    _check_quant(q.bfloat16(), k.bfloat16(), v.bfloat16(), torch.bfloat16)


@pytest.mark.parametrize("name", ["image", "video"])
def test_quantiser_bit_exact_full_workloads(name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    _check_quant(q, k, v, w.torch_dtype)


def test_quantiser_wait_timeout_is_reported_and_context_survives():
    """A block copy that never arrives (test hook: the Q quantiser's first CTA skips
    its second block) ends in a bounded wait: ATTN_ERR_TIMEOUT is reported, nothing
    hangs, and the next call on the same context is bit-exact again."""
    from attention_forward_flash_b200 import _abi
    B, Hq, Hk, S, D = 1, 32, 8, 4096, 128   # 1024 Q blocks: more than the quantiser CTAs
    g = torch.Generator().manual_seed(21)
    q, k, v = (torch.randn(B, h, S, D, generator=g).to(torch.bfloat16) for h in (Hq, Hk, Hk))
    att = Attention(B, Hq, Hk, S, S, D, precision="quant")
    _abi.attn_debug_set(att.ctx, 2)
    att.quantize(q.cuda(), k.cuda(), v.cuda())
    with pytest.raises(_abi.AttnError) as e:
        att.check_error()
    assert e.value.status == _abi.ATTN_ERR_TIMEOUT
    _abi.attn_debug_set(att.ctx, 0)
    qb = att.quantize(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    rq, rqs = quantize_qk_int8(q.float().numpy())
    assert np.array_equal(qb.q_scale.cpu().numpy().view(np.uint32), rqs.view(np.uint32))
    assert np.array_equal(qb.q.cpu().numpy(), rq)
