"""Torch-facing convenience wrapper over the C ABI.

Torch provides device memory and streams only; every computation runs in the
library's kernels.  Shapes: q [B, Hq, Sq, D], k/v [B, Hkv, Skv, D], contiguous
CUDA tensors of the context's dtype.
"""

from __future__ import annotations

import torch

from . import _abi
from ._abi import (ATTN_BF16, ATTN_EXACT, ATTN_FP16, ATTN_INT8QK_FP8PV, ATTN_MIXED_DIAG,
                   ATTN_MXFP4QK_FP8PV, ATTN_ROPE_NTK,
                   ATTN_ROPE_PLAIN, ATTN_ROPE_YARN, AttnParams, AttnQBufs, AttnRopeFreq)

_SCALINGS = {None: ATTN_ROPE_PLAIN, "ntk": ATTN_ROPE_NTK, "yarn": ATTN_ROPE_YARN}


def rope_table(rope_dim, n_pos, *, base=10000.0, scaling=None, factor=1.0, original_len=0,
               beta_fast=32.0, beta_slow=1.0):
    """The library's cos/sin table (``attn_rope_table``) as a CPU float32 tensor
    [n_pos, 2, rope_dim / 2]; ``scaling`` is None, "ntk" or "yarn"."""
    t = torch.empty((n_pos, 2, rope_dim // 2), dtype=torch.float32)
    f = AttnRopeFreq(base, _SCALINGS[scaling], factor, original_len, beta_fast, beta_slow)
    _abi.attn_rope_table(rope_dim, n_pos, f, t.data_ptr())
    return t

# "mixed": the quantised mode with 16-bit Q K^T on the causal diagonal band tiles;
# "fp4": MXFP4 Q K^T (block-scaled MMA) with FP8 P V, head_dim 64
_PRECISIONS = {"exact": ATTN_EXACT, "quant": ATTN_INT8QK_FP8PV, "mixed": ATTN_MIXED_DIAG,
               "fp4": ATTN_MXFP4QK_FP8PV}


def _stream_handle(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class QuantBuffers:
    """Device buffers of the quantised modes (see ``attn_qbufs`` in include/attn.h).

    FP4 mode: ``q``/``k`` hold packed E2M1 codes ([..., D/2] bytes), ``q_sf``/``k_sf``
    the E8M0 scale chunks, and there are no FP32 Q/K scales."""

    def __init__(self, params: AttnParams, device):
        B, Hq, Hk = params.batch, params.n_q_heads, params.n_kv_heads
        Sq, Sk, D = params.q_len, params.kv_len, params.head_dim
        nbq, nbk = (Sq + 127) // 128, (Sk + 127) // 128
        fp4 = params.precision == ATTN_MXFP4QK_FP8PV
        w = D // 2 if fp4 else D
        self.q = torch.empty((B, Hq, Sq, w), dtype=torch.uint8 if fp4 else torch.int8,
                             device=device)
        self.k = torch.empty((B, Hk, Sk, w), dtype=torch.uint8 if fp4 else torch.int8,
                             device=device)
        self.q_scale = None if fp4 else torch.empty((B, Hq, nbq), dtype=torch.float32,
                                                    device=device)
        self.k_scale = None if fp4 else torch.empty((B, Hk, nbk), dtype=torch.float32,
                                                    device=device)
        self.v_t = torch.empty((B, Hk, D, nbk * 128), dtype=torch.uint8, device=device)
        self.v_scale = torch.empty((B, Hk, D), dtype=torch.float32, device=device)
        self.q_sf = self.k_sf = None
        if fp4:
            nq, nk = _abi.attn_qbufs_sf_sizes(params)
            self.q_sf = torch.empty(max(nq, 16), dtype=torch.uint8, device=device)
            self.k_sf = torch.empty(max(nk, 16), dtype=torch.uint8, device=device)

    def struct(self):
        ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
        return AttnQBufs(self.q.data_ptr(), self.k.data_ptr(), ptr(self.q_scale),
                         ptr(self.k_scale), self.v_t.data_ptr(), self.v_scale.data_ptr(),
                         ptr(self.q_sf), ptr(self.k_sf))


class DeviceStaging:
    """Device buffers that ``Attention.forward_host`` copies through (full problem size)."""

    def __init__(self, params: AttnParams, dtype, device, quant, with_lse):
        B, Hq, Hk = params.batch, params.n_q_heads, params.n_kv_heads
        Sq, Sk, D = params.q_len, params.kv_len, params.head_dim
        self.q = torch.empty((B, Hq, Sq, D), dtype=dtype, device=device)
        self.k = torch.empty((B, Hk, Sk, D), dtype=dtype, device=device)
        self.v = torch.empty((B, Hk, Sk, D), dtype=dtype, device=device)
        self.o = torch.empty((B, Hq, Sq, D), dtype=dtype, device=device)
        self.lse = (torch.empty((B, Hq, Sq), dtype=torch.float32, device=device)
                    if with_lse else None)
        self.qbufs = QuantBuffers(params, device) if quant else None


class Attention:
    """One attention problem shape bound to a library context."""

    def __init__(self, batch, n_q_heads, n_kv_heads, q_len, kv_len, head_dim, *,
                 dtype=torch.bfloat16, causal=False, start_pos=0, window_lo=0, scale=0.0,
                 precision="exact", num_splits=0, window_size=0, rope_dim=0,
                 rope_interleaved=False, rope_keys_rotated=False, rope_table=None):
        """``rope_dim`` > 0 turns on RoPE over the first rope_dim channels; its
        cos/sin table is ``rope_table`` (a float32 tensor [n_pos, 2, rope_dim / 2],
        e.g. from ``rope_table()``; copied to the device if it is on the CPU) and
        can also be given later with ``set_rope_table``."""
        if dtype not in (torch.bfloat16, torch.float16):
            raise ValueError("dtype must be torch.bfloat16 or torch.float16")
        self.dtype = dtype
        self.precision = precision
        self.params = AttnParams(batch, n_q_heads, n_kv_heads, q_len, kv_len, head_dim, start_pos,
                                 int(bool(causal)), window_lo, float(scale),
                                 ATTN_FP16 if dtype == torch.float16 else ATTN_BF16,
                                 _PRECISIONS[precision], num_splits, window_size, rope_dim,
                                 int(bool(rope_interleaved)), int(bool(rope_keys_rotated)))
        self.ctx = _abi.attn_create(self.params)
        self._rope_table = None
        if rope_table is not None:
            self.set_rope_table(rope_table)

    def set_rope_table(self, table, device=None):
        """Gives the context its RoPE table (kept alive by this object)."""
        if table.dtype != torch.float32 or table.dim() != 3 or table.shape[1] != 2:
            raise ValueError("rope table: expected float32 [n_pos, 2, rope_dim / 2]")
        if not table.is_cuda:
            dev = device if device is not None else torch.device("cuda",
                                                                 torch.cuda.current_device())
            table = table.to(dev)
        table = table.contiguous()
        _abi.attn_set_rope_table(self.ctx, table.data_ptr(), table.shape[0])
        self._rope_table = table

    def rope_apply(self, x, out=None, pos0=0, stream=None):
        """RoPE of x [batch, heads, len, head_dim] (positions pos0 + t) through
        ``attn_rope_apply``; ``out`` may be x itself."""
        out = torch.empty_like(x) if out is None else out
        _abi.attn_rope_apply(self.ctx, x.data_ptr(), out.data_ptr(), x.shape[1], x.shape[2], pos0,
                             _stream_handle(stream))
        return out

    @property
    def num_splits(self):
        return _abi.attn_num_splits(self.ctx)

    @property
    def kernel_path(self):
        """``"single_pass"``, ``"single_pass_tail"``, ``"split_merge"`` or ``"decode"``
        (``attn_kernel_path``)."""
        return {_abi.ATTN_PATH_SINGLE_PASS: "single_pass", _abi.ATTN_PATH_SPLIT_MERGE:
                "split_merge", _abi.ATTN_PATH_DECODE: "decode",
                _abi.ATTN_PATH_SINGLE_PASS_TAIL: "single_pass_tail"}[
                    _abi.attn_kernel_path(self.ctx)]

    def _check_tensor(self, name, t, shape, dtype, on_cuda=True):
        where = "CUDA" if on_cuda else "host"
        if (tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous()
                or t.is_cuda != on_cuda):
            raise ValueError(f"{name}: expected contiguous {where} {dtype} of shape "
                             f"{shape}, got {t.dtype} {tuple(t.shape)} on {t.device}")

    def _check_inputs(self, q, k, v, on_cuda=True):
        p = self.params
        want_q = (p.batch, p.n_q_heads, p.q_len, p.head_dim)
        want_kv = (p.batch, p.n_kv_heads, p.kv_len, p.head_dim)
        for name, t, shape in (("q", q, want_q), ("k", k, want_kv), ("v", v, want_kv)):
            self._check_tensor(name, t, shape, self.dtype, on_cuda)

    def _check_outputs(self, out, lse, on_cuda=True):
        """A caller's O [B, Hq, Sq, D] (the context's dtype) and lse [B, Hq, Sq] (float32)."""
        p = self.params
        if out is not None:
            self._check_tensor("out", out, (p.batch, p.n_q_heads, p.q_len, p.head_dim),
                               self.dtype, on_cuda)
        if lse is not None:
            self._check_tensor("lse", lse, (p.batch, p.n_q_heads, p.q_len), torch.float32,
                               on_cuda)

    def quantize(self, q, k, v, qbufs=None, stream=None):
        if self.precision == "exact":
            raise ValueError("quantize() needs a quantised precision ('quant', 'mixed', 'fp4')")
        self._check_inputs(q, k, v)
        qbufs = qbufs if qbufs is not None else QuantBuffers(self.params, q.device)
        _abi.attn_quantize_qk(self.ctx, q.data_ptr(), k.data_ptr(), v.data_ptr(), qbufs.struct(),
                              _stream_handle(stream))
        return qbufs

    def _check_pools(self, q, k_pool, v_pool, block_table):
        p = self.params
        self._check_tensor("q", q, (p.batch, p.n_q_heads, p.q_len, p.head_dim), self.dtype)
        want = (p.n_kv_heads, 128, p.head_dim)
        for name, t in (("k_pool", k_pool), ("v_pool", v_pool)):
            if (t.dim() != 4 or tuple(t.shape[1:]) != want or t.dtype != self.dtype
                    or not t.is_contiguous() or not t.is_cuda):
                raise ValueError(f"{name}: expected contiguous CUDA {self.dtype} "
                                 f"[blocks, {want[0]}, {want[1]}, {want[2]}]")
        if v_pool.shape[0] != k_pool.shape[0]:
            raise ValueError("k_pool and v_pool must hold the same number of blocks")
        nbt = (p.kv_len + 127) // 128
        if (block_table.dtype != torch.int32 or tuple(block_table.shape) != (p.batch, nbt)
                or not block_table.is_contiguous() or not block_table.is_cuda):
            raise ValueError(f"block_table: expected contiguous CUDA int32 [{p.batch}, {nbt}]")

    def quantize_paged(self, q, k_pool, v_pool, block_table, qbufs=None, stream=None):
        """INT8 mode: the quantisers with K and V read from a paged cache
        (``attn_quantize_qk_paged``); returns the dense ``QuantBuffers`` that
        ``forward(qbufs=...)`` takes."""
        if self.precision != "quant":
            raise ValueError("quantize_paged() needs precision='quant'")
        self._check_pools(q, k_pool, v_pool, block_table)
        qbufs = qbufs if qbufs is not None else QuantBuffers(self.params, q.device)
        _abi.attn_quantize_qk_paged(self.ctx, q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                    block_table.data_ptr(), k_pool.shape[0], qbufs.struct(),
                                    _stream_handle(stream))
        return qbufs

    def forward(self, q=None, k=None, v=None, *, qbufs=None, out=None, lse=None, return_lse=False,
                stream=None):
        p = self.params
        device = (q if q is not None else qbufs.q).device
        self._check_outputs(out, lse)
        if out is None:
            out = torch.empty((p.batch, p.n_q_heads, p.q_len, p.head_dim), dtype=self.dtype,
                              device=device)
        if lse is None and return_lse:
            lse = torch.empty((p.batch, p.n_q_heads, p.q_len), dtype=torch.float32, device=device)
        st = _stream_handle(stream)
        lse_ptr = lse.data_ptr() if lse is not None else None
        if self.precision in ("quant", "fp4"):
            if qbufs is None:
                qbufs = self.quantize(q, k, v, stream=stream)
            _abi.attn_forward(self.ctx, None, None, None, qbufs.struct(), out.data_ptr(), lse_ptr, st)
        elif self.precision == "mixed":   # the band tiles read the 16-bit q and k
            self._check_inputs(q, k, v)
            if qbufs is None:
                qbufs = self.quantize(q, k, v, stream=stream)
            _abi.attn_forward(self.ctx, q.data_ptr(), k.data_ptr(), None, qbufs.struct(),
                              out.data_ptr(), lse_ptr, st)
        else:
            self._check_inputs(q, k, v)
            _abi.attn_forward(self.ctx, q.data_ptr(), k.data_ptr(), v.data_ptr(), None,
                              out.data_ptr(), lse_ptr, st)
        return (out, lse) if return_lse else out

    __call__ = forward

    def forward_paged(self, q, k_pool, v_pool, block_table, *, out=None, lse=None,
                      return_lse=False, stream=None):
        """Exact-mode forward over a paged key/value cache (``attn_forward_paged``).

        k_pool, v_pool: [num_blocks, n_kv_heads, 128, head_dim] CUDA tensors of the
        context's dtype; block_table: int32 CUDA tensor [batch, ceil(kv_len / 128)].
        """
        p = self.params
        if self.precision != "exact":
            raise ValueError("forward_paged() needs precision='exact' (the INT8 mode: "
                             "quantize_paged(), then forward(qbufs=...))")
        self._check_pools(q, k_pool, v_pool, block_table)
        self._check_outputs(out, lse)
        if out is None:
            out = torch.empty((p.batch, p.n_q_heads, p.q_len, p.head_dim), dtype=self.dtype,
                              device=q.device)
        if lse is None and return_lse:
            lse = torch.empty((p.batch, p.n_q_heads, p.q_len), dtype=torch.float32,
                              device=q.device)
        _abi.attn_forward_paged(self.ctx, q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                block_table.data_ptr(), k_pool.shape[0], out.data_ptr(),
                                lse.data_ptr() if lse is not None else None,
                                _stream_handle(stream))
        return (out, lse) if return_lse else out

    def forward_host(self, q, k, v, *, out=None, lse=None, return_lse=False, staging=None,
                     chunks=0, stream=None, device=None):
        """End-to-end forward from host tensors through ``attn_forward_host``.

        q, k, v: contiguous CPU tensors (page-locked ones let the copies overlap the
        kernels).  out / lse: CPU tensors to write (page-locked ones are allocated if
        None).  staging: the ``DeviceStaging`` to copy through; one is allocated on
        ``device`` (default: the current CUDA device) and kept for later calls if
        None.  Calls that share a staging must be ordered (one stream).  The call is
        asynchronous on ``stream``: synchronise it before reading the outputs.
        """
        p = self.params
        self._check_inputs(q, k, v, on_cuda=False)
        self._check_outputs(out, lse, on_cuda=False)
        want_lse = return_lse or lse is not None
        if staging is None:
            cached = getattr(self, "_staging", None)
            if cached is None or (want_lse and cached.lse is None):
                dev = (device if device is not None
                       else torch.device("cuda", torch.cuda.current_device()))
                cached = DeviceStaging(p, self.dtype, dev, self.precision != "exact", want_lse)
                self._staging = cached
            staging = cached
        if out is None:
            out = torch.empty((p.batch, p.n_q_heads, p.q_len, p.head_dim), dtype=self.dtype,
                              pin_memory=True)
        if lse is None and return_lse:
            lse = torch.empty((p.batch, p.n_q_heads, p.q_len), dtype=torch.float32,
                              pin_memory=True)
        if lse is not None and staging.lse is None:
            raise ValueError("lse requested but the staging has no lse buffer")
        lse_host = lse.data_ptr() if lse is not None else None
        lse_dev = staging.lse.data_ptr() if lse is not None else None
        qb = staging.qbufs.struct() if staging.qbufs is not None else None
        _abi.attn_forward_host(self.ctx, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse_host, staging.q.data_ptr(), staging.k.data_ptr(),
                               staging.v.data_ptr(), staging.o.data_ptr(), lse_dev, qb, chunks,
                               _stream_handle(stream))
        return (out, lse) if return_lse else out

    def check_error(self, stream=None):
        """Synchronise and raise AttnError if a kernel recorded a failed wait."""
        status = _abi.attn_get_error(self.ctx, _stream_handle(stream))
        if status != _abi.ATTN_OK:
            raise _abi.AttnError(status, "device")

    def close(self):
        if getattr(self, "ctx", None) is not None and self.ctx.value:
            _abi.attn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
