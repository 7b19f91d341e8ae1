"""RoPE on the GPU path against the oracle.

* ``attn_rope_apply`` (the stand-alone pass: keys for a cache, the exact mode's
  keys) is bit-exact against the oracle's float32 rotation rounded to 16 bits,
  on the same table (the oracle's, passed in as the input it is).
* The quantised mode rotates Q and K inside its quantiser: the INT8 codes and
  scales are bit-exact against the oracle's quantiser applied to the oracle's
  float32 rotation.
* Attention with RoPE, exact and quantised, single-pass and split-KV kernels,
  both pair layouts, partial rotary widths, NTK and YaRN frequencies, against
  float64 attention on the float64-rotated inputs at the usual tolerances (the
  oracle's table as input; one case with the library's own table); keys rotated
  once into a cache (rope_keys_rotated) and a paged cache give the same bits as
  rotating inside the forward; the INT8 mode on such a cache rotates only Q, dense
  and paged alike; the host-buffer pipeline is bit-identical.
"""

import numpy as np
import pytest
import torch

from attention_forward_flash_b200 import Attention, rope_table
from attention_forward_flash_b200.inputs import Workload, make_qkv
from oracle import (apply_rope, apply_rope_f32, attention_f64, quantize_qk_int8, rope_frequencies,
                    yarn_attention_factor)
from oracle import rope_table as oracle_table
from parity_util import QUANT_RMSE, check_exact, check_lse, rel_rmse

pytestmark = pytest.mark.gpu


def _att(w, precision="exact", num_splits=0, R=128, inter=False, keys_rotated=False, table=None):
    return Attention(w.batch, w.n_q_heads, w.n_kv_heads, w.q_len, w.kv_len, w.head_dim,
                     dtype=w.torch_dtype, causal=w.causal, start_pos=w.start_pos,
                     window_lo=w.window_lo, window_size=w.window_size, precision=precision,
                     num_splits=num_splits, rope_dim=R, rope_interleaved=inter,
                     rope_keys_rotated=keys_rotated, rope_table=table)


def _theta_m(R, scaling, factor=4.0, original_len=4096):
    theta = rope_frequencies(R, scaling=scaling, factor=factor,
                             original_len=original_len if scaling == "yarn" else None)
    m = yarn_attention_factor(factor) if scaling == "yarn" else 1.0
    return theta, m


def _oracle_rope_attention(w, q, k, v, theta, m, inter, rows=None, table16=None):
    """float64 attention on float64-rotated Q and K (the definition); with table16 (a
    float32 table), on Q and K rotated by the oracle's float32 form and rounded to the
    inputs' 16-bit type, i.e. the values the exact-mode kernel multiplies."""
    layout = "interleaved" if inter else "half"
    qpos = w.start_pos + np.arange(w.q_len)
    kpos = np.arange(w.kv_len)
    if table16 is None:
        qr = apply_rope(q.double().numpy(), qpos, theta, layout=layout, mscale=m)
        kr = apply_rope(k.double().numpy(), kpos, theta, layout=layout, mscale=m)
    else:
        qr, kr = (torch.from_numpy(apply_rope_f32(x.float().numpy(), pos, table16, layout=layout))
                  .to(w.torch_dtype).double().numpy() for x, pos in ((q, qpos), (k, kpos)))
    return attention_f64(qr, kr, v.double().numpy(), causal=w.causal, start_pos=w.start_pos,
                         window_lo=w.window_lo, window_size=w.window_size, rows=rows)


@pytest.mark.parametrize("D,R,inter,dtype", [(128, 128, False, "bf16"), (128, 128, True, "fp16"),
                                             (128, 64, False, "bf16"), (64, 64, True, "bf16"),
                                             (64, 32, False, "fp16")])
def test_rope_apply_bit_exact(D, R, inter, dtype):
    w = Workload("ra", 2, 3, 3, 5, 300, D, dtype, seed=8100 + R)
    _, x, _ = make_qkv(w)
    pos0 = 1234
    theta, _ = _theta_m(R, "yarn")
    table = oracle_table(pos0 + 300, theta, mscale=1.25)
    att = _att(w, R=R, inter=inter, table=torch.from_numpy(table))
    y = att.rope_apply(x.cuda(), pos0=pos0)
    att.check_error()
    ref = apply_rope_f32(x.float().numpy(), pos0 + np.arange(300), table,
                         layout="interleaved" if inter else "half")
    ref16 = torch.from_numpy(ref).to(w.torch_dtype)      # round to nearest even
    assert torch.equal(y.cpu().view(torch.int16), ref16.view(torch.int16))
    # in place gives the same bits
    xi = x.cuda().clone()
    att.rope_apply(xi, out=xi, pos0=pos0)
    assert torch.equal(xi.cpu(), y.cpu())


@pytest.mark.parametrize("D,R,inter", [(128, 128, False), (128, 128, True), (128, 64, False),
                                       (64, 64, False), (64, 48, True)])
def test_quantiser_codes_of_rotated_qk_bit_exact(D, R, inter):
    w = Workload("rq", 1, 4, 2, 300, 777, D, "bf16", causal=True, start_pos=477, seed=8200 + R,
                 k_outlier_frac=0.01, k_outlier_mult=20.0)
    q, k, v = make_qkv(w)
    theta, m = _theta_m(R, "ntk", factor=8.0)
    table = oracle_table(w.start_pos + w.q_len, theta, mscale=m)
    att = _att(w, precision="quant", R=R, inter=inter, table=torch.from_numpy(table))
    qb = att.quantize(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    layout = "interleaved" if inter else "half"
    qr = apply_rope_f32(q.float().numpy(), w.start_pos + np.arange(w.q_len), table, layout=layout)
    kr = apply_rope_f32(k.float().numpy(), np.arange(w.kv_len), table, layout=layout)
    for got_c, got_s, x in ((qb.q, qb.q_scale, qr), (qb.k, qb.k_scale, kr)):
        codes, scales = quantize_qk_int8(x)
        assert np.array_equal(got_c.cpu().numpy(), codes)
        assert np.array_equal(got_s.cpu().numpy(), scales)


ATT_CASES = [
    # name, workload, R, interleaved, scaling
    ("prefill_half", Workload("p", 1, 4, 4, 700, 700, 128, "bf16", seed=8301), 128, False, None),
    ("causal_gqa_yarn", Workload("c", 2, 8, 2, 600, 900, 128, "bf16", causal=True, start_pos=300,
                                 seed=8302), 128, False, "yarn"),
    ("interleaved_ntk", Workload("i", 1, 4, 2, 513, 1111, 128, "fp16", seed=8303), 128, True,
     "ntk"),
    ("partial_64", Workload("r", 1, 4, 4, 400, 400, 128, "bf16", causal=True, seed=8304), 64,
     False, None),
    ("d64", Workload("d", 1, 4, 4, 500, 500, 64, "bf16", seed=8305), 64, False, "yarn"),
    ("sliding", Workload("s", 1, 4, 2, 700, 1291, 128, "bf16", causal=True, start_pos=591,
                         window_size=256, seed=8306), 128, False, None),
    ("decode_split", Workload("t", 1, 16, 8, 4, 4096, 128, "fp16", causal=True, start_pos=4092,
                              seed=8307), 128, False, "yarn"),
]


@pytest.mark.parametrize("name,w,R,inter,scaling", ATT_CASES, ids=[c[0] for c in ATT_CASES])
def test_exact_attention_with_rope(name, w, R, inter, scaling):
    """O against the float64 definition at the exact-mode tolerances.  lse against
    float64 attention on the 16-bit rotated Q and K that the kernel multiplies (the
    rounding of the rotated values moves scores by ~2^-9 relative, which lse
    carries one for one), at the exact-mode lse tolerance."""
    q, k, v = make_qkv(w)
    theta, m = _theta_m(R, scaling)
    n_pos = max(w.start_pos + w.q_len, w.kv_len)
    table = oracle_table(n_pos, theta, mscale=m)
    att = _att(w, R=R, inter=inter, table=torch.from_numpy(table))
    o, lse = att.forward(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    att.check_error()
    if name == "decode_split":
        assert att.num_splits > 1
    ro, _ = _oracle_rope_attention(w, q, k, v, theta, m, inter)
    check_exact(o.double().cpu().numpy(), ro, name)
    _, rl16 = _oracle_rope_attention(w, q, k, v, theta, m, inter, table16=table)
    check_lse(lse.cpu().numpy(), rl16, name)


def test_exact_attention_with_the_librarys_own_table():
    _, w, R, inter, scaling = ATT_CASES[1]
    q, k, v = make_qkv(w)
    theta, m = _theta_m(R, scaling)
    table = rope_table(R, max(w.start_pos + w.q_len, w.kv_len), scaling=scaling, factor=4.0,
                       original_len=4096)
    att = _att(w, R=R, inter=inter, table=table)
    o = att.forward(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    ro, _ = _oracle_rope_attention(w, q, k, v, theta, m, inter)
    check_exact(o.double().cpu().numpy(), ro, "library table")


@pytest.mark.parametrize("name", ["causal_gqa_yarn", "interleaved_ntk", "decode_split"])
def test_quantised_attention_with_rope(name):
    _, w, R, inter, scaling = next(c for c in ATT_CASES if c[0] == name)
    q, k, v = make_qkv(w)
    theta, m = _theta_m(R, scaling)
    n_pos = max(w.start_pos + w.q_len, w.kv_len)
    table = torch.from_numpy(oracle_table(n_pos, theta, mscale=m))
    att = _att(w, precision="quant", R=R, inter=inter, table=table)
    o = att.forward(q.cuda(), k.cuda(), v.cuda())
    att.check_error()
    ro, _ = _oracle_rope_attention(w, q, k, v, theta, m, inter)
    e = rel_rmse(o.double().cpu().numpy(), ro)
    assert e <= QUANT_RMSE, f"{name}: {e:.3e}"


def test_keys_rotated_once_into_a_cache_and_paged():
    """A decode step on a cache of keys rotated once through attn_rope_apply
    (rope_keys_rotated): the same bits as rotating inside the forward, dense and
    paged."""
    w = Workload("cache", 2, 16, 8, 4, 2000, 128, "bf16", causal=True, start_pos=1996, seed=8400)
    q, k, v = (t.cuda() for t in make_qkv(w))
    table = rope_table(128, 2000, scaling="yarn", factor=4.0, original_len=1024)
    full = _att(w, table=table)
    o_ref = full.forward(q, k, v)
    full.check_error()
    cached = _att(w, keys_rotated=True, table=table)
    k_rot = cached.rope_apply(k, pos0=0)                 # written once, as a cache would be
    o = cached.forward(q, k_rot, v)
    cached.check_error()
    assert torch.equal(o, o_ref)
    # the same cache as a paged pool (blocks of 128 positions, shuffled)
    nblk = (2000 + 127) // 128
    g = torch.Generator().manual_seed(5)
    perm = torch.randperm(w.batch * nblk, generator=g)
    pool_k = torch.zeros((w.batch * nblk + 3, 8, 128, 128), dtype=k.dtype, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    table_b = perm.view(w.batch, nblk).int().cuda()
    for b in range(w.batch):
        for t in range(nblk):
            n = min(128, 2000 - 128 * t)
            pool_k[table_b[b, t], :, :n] = k_rot[b, :, 128 * t:128 * t + n]
            pool_v[table_b[b, t], :, :n] = v[b, :, 128 * t:128 * t + n]
    o_p = cached.forward_paged(q, pool_k, pool_v, table_b)
    cached.check_error()
    assert torch.equal(o_p, o_ref)


def test_quantised_mode_on_keys_rotated_once_dense_and_paged():
    """INT8 mode on a cache of keys rotated once (rope_keys_rotated): the quantiser
    rotates Q only and takes the cached keys as they are.  Q's codes and scales are
    those of the mode that rotates both; K's are the oracle quantiser's on the cached
    keys; the paged quantiser's buffers equal the dense ones bit for bit; the attention
    is within the quantised tolerance of the float64 definition."""
    w = Workload("cacheq", 2, 16, 8, 4, 2000, 128, "bf16", causal=True, start_pos=1996,
                 seed=8401)
    q, k, v = make_qkv(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    table = rope_table(128, 2000, scaling="yarn", factor=4.0, original_len=1024)
    both = _att(w, precision="quant", table=table)
    qb_both = both.quantize(qd, kd, vd)
    both.check_error()
    cached = _att(w, precision="quant", keys_rotated=True, table=table)
    k_rot = cached.rope_apply(kd, pos0=0)
    dense = cached.quantize(qd, k_rot, vd)
    cached.check_error()
    assert torch.equal(dense.q, qb_both.q) and torch.equal(dense.q_scale, qb_both.q_scale)
    rk, rks = quantize_qk_int8(k_rot.float().cpu().numpy())
    assert np.array_equal(dense.k.cpu().numpy(), rk)
    assert np.array_equal(dense.k_scale.cpu().numpy().view(np.uint32), rks.view(np.uint32))
    # the same cache as a paged pool (blocks of 128 positions, shuffled)
    nblk = (2000 + 127) // 128
    perm = torch.randperm(w.batch * nblk, generator=torch.Generator().manual_seed(6))
    pool_k = torch.zeros((w.batch * nblk + 3, 8, 128, 128), dtype=k.dtype, device="cuda")
    pool_v = torch.zeros_like(pool_k)
    table_b = perm.view(w.batch, nblk).int().cuda()
    for b in range(w.batch):
        for t in range(nblk):
            n = min(128, 2000 - 128 * t)
            pool_k[table_b[b, t], :, :n] = k_rot[b, :, 128 * t:128 * t + n]
            pool_v[table_b[b, t], :, :n] = vd[b, :, 128 * t:128 * t + n]
    paged = cached.quantize_paged(qd, pool_k, pool_v, table_b)
    cached.check_error()
    for f in ("q", "k", "q_scale", "k_scale", "v_t", "v_scale"):
        assert torch.equal(getattr(paged, f), getattr(dense, f)), f
    o = cached.forward(qbufs=paged)
    cached.check_error()
    assert torch.equal(o, cached.forward(qbufs=dense))
    theta, m = _theta_m(128, "yarn", original_len=1024)
    ro, _ = _oracle_rope_attention(w, q, k, v, theta, m, False)
    e = rel_rmse(o.double().cpu().numpy(), ro)
    assert e <= QUANT_RMSE, f"{e:.3e}"


@pytest.mark.parametrize("precision", ["exact", "quant"])
def test_host_pipeline_with_rope_is_bit_identical(precision):
    w = Workload("hp", 1, 8, 2, 1000, 1000, 128, "bf16", causal=True, seed=8500)
    q, k, v = make_qkv(w)
    table = rope_table(128, 1000, scaling="ntk", factor=2.0)
    att = _att(w, precision=precision, table=table)
    ref = att.forward(q.cuda(), k.cuda(), v.cuda())
    out = att.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), chunks=2)
    torch.cuda.synchronize()
    att.check_error()
    assert torch.equal(out, ref.cpu())


def test_rope_without_a_table_is_rejected():
    from attention_forward_flash_b200 import _abi
    w = Workload("nt", 1, 2, 2, 128, 128, 128, "bf16", seed=1)
    q, k, v = (t.cuda() for t in make_qkv(w))
    att = _att(w)
    with pytest.raises(_abi.AttnError) as e:
        att.forward(q, k, v)
    assert e.value.status == _abi.ATTN_ERR_INVALID_ARG
    small = torch.zeros((10, 2, 64), dtype=torch.float32)   # too few positions
    with pytest.raises(_abi.AttnError):
        att.set_rope_table(small)
