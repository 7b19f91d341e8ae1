"""ctypes declarations of the C ABI in ``include/attn.h`` (marshalling only)."""

from __future__ import annotations

import ctypes
import os

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_OOM, \
    ATTN_ERR_TIMEOUT = range(6)
ATTN_BF16, ATTN_FP16 = 0, 1
ATTN_EXACT, ATTN_INT8QK_FP8PV, ATTN_MIXED_DIAG, ATTN_MXFP4QK_FP8PV = 0, 1, 2, 3
ATTN_ROPE_PLAIN, ATTN_ROPE_NTK, ATTN_ROPE_YARN = 0, 1, 2
ATTN_PATH_SINGLE_PASS, ATTN_PATH_SPLIT_MERGE, ATTN_PATH_DECODE, ATTN_PATH_SINGLE_PASS_TAIL = \
    1, 2, 3, 4

EXPORTED = ("attn_create", "attn_quantize_qk", "attn_forward", "attn_get_error", "attn_destroy",
            "attn_status_string", "attn_qbufs_sizes", "attn_num_splits", "attn_debug_set",
            "attn_debug_exp2", "attn_forward_splitkv_noalloc", "attn_forward_host",
            "attn_forward_paged", "attn_rope_table", "attn_set_rope_table", "attn_rope_apply",
            "attn_qbufs_sf_sizes", "attn_kernel_path", "attn_plan_for", "attn_quantize_qk_paged")

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path():
    return os.path.join(_HERE, "libattn.so")


class AttnParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("q_len", ctypes.c_int), ("kv_len", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("start_pos", ctypes.c_int), ("causal", ctypes.c_int), ("window_lo", ctypes.c_int),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int), ("precision", ctypes.c_int),
                ("num_splits", ctypes.c_int), ("window_size", ctypes.c_int),
                ("rope_dim", ctypes.c_int), ("rope_interleaved", ctypes.c_int),
                ("rope_keys_rotated", ctypes.c_int)]


class AttnRopeFreq(ctypes.Structure):
    _fields_ = [("base", ctypes.c_float), ("scaling", ctypes.c_int), ("factor", ctypes.c_float),
                ("original_len", ctypes.c_int), ("beta_fast", ctypes.c_float),
                ("beta_slow", ctypes.c_float)]


class AttnQBufs(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_t", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("q_sf", ctypes.c_void_p),
                ("k_sf", ctypes.c_void_p)]


class AttnError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {attn_status_string(status)} ({status})")


_LIB = None


def lib():
    """Load ``libattn.so`` (raises OSError if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise OSError(f"{path} is missing: build it with "
                          "`python -m attention_forward_flash_b200.build`")
        L = ctypes.CDLL(path)
        vp, c_int = ctypes.c_void_p, ctypes.c_int
        L.attn_create.argtypes = [ctypes.POINTER(AttnParams), ctypes.POINTER(vp)]
        L.attn_create.restype = c_int
        L.attn_quantize_qk.argtypes = [vp, vp, vp, vp, ctypes.POINTER(AttnQBufs), vp]
        L.attn_quantize_qk.restype = c_int
        L.attn_forward.argtypes = [vp, vp, vp, vp, ctypes.POINTER(AttnQBufs), vp, vp, vp]
        L.attn_forward.restype = c_int
        L.attn_get_error.argtypes = [vp, vp]
        L.attn_get_error.restype = c_int
        L.attn_destroy.argtypes = [vp]
        L.attn_destroy.restype = None
        L.attn_status_string.argtypes = [c_int]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_qbufs_sizes.argtypes = [ctypes.POINTER(AttnParams), ctypes.POINTER(ctypes.c_size_t)]
        L.attn_qbufs_sizes.restype = c_int
        L.attn_qbufs_sf_sizes.argtypes = [ctypes.POINTER(AttnParams),
                                          ctypes.POINTER(ctypes.c_size_t)]
        L.attn_qbufs_sf_sizes.restype = c_int
        L.attn_num_splits.argtypes = [vp]
        L.attn_num_splits.restype = c_int
        L.attn_kernel_path.argtypes = [vp]
        L.attn_kernel_path.restype = c_int
        L.attn_plan_for.argtypes = [ctypes.POINTER(AttnParams), c_int, ctypes.POINTER(AttnPlan)]
        L.attn_plan_for.restype = c_int
        L.attn_debug_set.argtypes = [vp, ctypes.c_uint]
        L.attn_debug_set.restype = c_int
        L.attn_debug_exp2.argtypes = [vp, vp, ctypes.c_size_t, vp]
        L.attn_debug_exp2.restype = c_int
        L.attn_forward_splitkv_noalloc.argtypes = [ctypes.POINTER(AttnParams), vp, vp, vp, vp, vp,
                                                   vp, vp]
        L.attn_forward_splitkv_noalloc.restype = c_int
        L.attn_forward_host.argtypes = [vp] * 11 + [ctypes.POINTER(AttnQBufs), c_int, vp]
        L.attn_forward_host.restype = c_int
        L.attn_forward_paged.argtypes = [vp, vp, vp, vp, vp, c_int, vp, vp, vp]
        L.attn_forward_paged.restype = c_int
        L.attn_quantize_qk_paged.argtypes = [vp, vp, vp, vp, vp, c_int, ctypes.POINTER(AttnQBufs),
                                             vp]
        L.attn_quantize_qk_paged.restype = c_int
        L.attn_rope_table.argtypes = [c_int, c_int, ctypes.POINTER(AttnRopeFreq), vp]
        L.attn_rope_table.restype = c_int
        L.attn_set_rope_table.argtypes = [vp, vp, c_int]
        L.attn_set_rope_table.restype = c_int
        L.attn_rope_apply.argtypes = [vp, vp, vp, c_int, c_int, c_int, vp]
        L.attn_rope_apply.restype = c_int
        _LIB = L
    return _LIB


def attn_status_string(status):
    return lib().attn_status_string(int(status)).decode()


def _check(status, what):
    if status != ATTN_OK:
        raise AttnError(status, what)


def attn_create(params: AttnParams):
    ctx = ctypes.c_void_p()
    _check(lib().attn_create(ctypes.byref(params), ctypes.byref(ctx)), "attn_create")
    return ctx


def attn_quantize_qk(ctx, q, k, v, qbufs: AttnQBufs, stream):
    _check(lib().attn_quantize_qk(ctx, q, k, v, ctypes.byref(qbufs), stream), "attn_quantize_qk")


def attn_quantize_qk_paged(ctx, q, k_pool, v_pool, block_table, num_blocks, qbufs: AttnQBufs,
                           stream):
    _check(lib().attn_quantize_qk_paged(ctx, q, k_pool, v_pool, block_table, num_blocks,
                                        ctypes.byref(qbufs), stream), "attn_quantize_qk_paged")


def attn_forward(ctx, q, k, v, qbufs, o, lse, stream):
    qb = ctypes.byref(qbufs) if qbufs is not None else None
    _check(lib().attn_forward(ctx, q, k, v, qb, o, lse, stream), "attn_forward")


def attn_get_error(ctx, stream):
    return lib().attn_get_error(ctx, stream)


def attn_destroy(ctx):
    lib().attn_destroy(ctx)


def attn_qbufs_sizes(params: AttnParams):
    sizes = (ctypes.c_size_t * 6)()
    _check(lib().attn_qbufs_sizes(ctypes.byref(params), sizes), "attn_qbufs_sizes")
    return list(sizes)


def attn_qbufs_sf_sizes(params: AttnParams):
    sizes = (ctypes.c_size_t * 2)()
    _check(lib().attn_qbufs_sf_sizes(ctypes.byref(params), sizes), "attn_qbufs_sf_sizes")
    return list(sizes)


def attn_num_splits(ctx):
    return lib().attn_num_splits(ctx)


def attn_kernel_path(ctx):
    return lib().attn_kernel_path(ctx)


class AttnPlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("path", "splits", "tiles_per_split", "ctas",
                                            "tail_items", "tail_splits", "decode_chunk",
                                            "decode_chunks")]


def attn_plan_for(params, num_sms):
    """The kernel choice for ``params`` (an AttnParams) on ``num_sms`` SMs, as a dict."""
    out = AttnPlan()
    _check(lib().attn_plan_for(ctypes.byref(params), num_sms, ctypes.byref(out)), "attn_plan_for")
    return {n: getattr(out, n) for n, _ in AttnPlan._fields_}


def attn_debug_set(ctx, flags):
    _check(lib().attn_debug_set(ctx, flags), "attn_debug_set")


def attn_debug_exp2(x, y, n, stream):
    _check(lib().attn_debug_exp2(x, y, n, stream), "attn_debug_exp2")


def attn_forward_splitkv_noalloc(params: AttnParams, q, k, v, o, lse, err, stream):
    _check(lib().attn_forward_splitkv_noalloc(ctypes.byref(params), q, k, v, o, lse, err, stream),
           "attn_forward_splitkv_noalloc")


def attn_forward_host(ctx, q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev,
                      lse_dev, qbufs, chunks, stream):
    qb = ctypes.byref(qbufs) if qbufs is not None else None
    _check(lib().attn_forward_host(ctx, q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev,
                                   v_dev, o_dev, lse_dev, qb, chunks, stream),
           "attn_forward_host")


def attn_forward_paged(ctx, q, k_pool, v_pool, block_table, num_blocks, o, lse, stream):
    _check(lib().attn_forward_paged(ctx, q, k_pool, v_pool, block_table, num_blocks, o, lse,
                                    stream), "attn_forward_paged")


def attn_rope_table(rope_dim, n_pos, freq: AttnRopeFreq, table_host_ptr):
    _check(lib().attn_rope_table(rope_dim, n_pos, ctypes.byref(freq), table_host_ptr),
           "attn_rope_table")


def attn_set_rope_table(ctx, table_dev_ptr, n_pos):
    _check(lib().attn_set_rope_table(ctx, table_dev_ptr, n_pos), "attn_set_rope_table")


def attn_rope_apply(ctx, x, y, n_heads, length, pos0, stream):
    _check(lib().attn_rope_apply(ctx, x, y, n_heads, length, pos0, stream), "attn_rope_apply")
