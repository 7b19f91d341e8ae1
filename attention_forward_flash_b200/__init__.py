"""B200-native fused attention forward (sm_100a): thin Python binding of ``libattn.so``.

The functions named after the C ABI (``attn_create``, ``attn_quantize_qk``,
``attn_forward``, ``attn_get_error``, ``attn_destroy``) only marshal
arguments; every step of the computation runs in the library's CUDA kernels.
``Attention`` is a convenience wrapper that allocates outputs with torch.
There is no fallback: if the library is missing, loading it raises.
"""

from ._abi import (  # noqa: F401
    ATTN_BF16,
    ATTN_EXACT,
    ATTN_FP16,
    ATTN_INT8QK_FP8PV,
    AttnError,
    AttnParams,
    AttnQBufs,
    AttnRopeFreq,
    attn_create,
    attn_debug_set,
    attn_destroy,
    attn_forward,
    attn_forward_splitkv_noalloc,
    attn_get_error,
    attn_num_splits,
    attn_qbufs_sizes,
    attn_quantize_qk,
    attn_status_string,
    lib,
    lib_path,
)
from .api import Attention, DeviceStaging, QuantBuffers, rope_table  # noqa: F401
