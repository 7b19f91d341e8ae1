"""Reference quantisers for the opt-in reduced-precision attention mode.

TEST INFRASTRUCTURE ONLY (imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path).  Shares no
code with the CUDA library.

The reduced-precision mode is the "SageAttention 2 INT8 QK · FP8 PV" row of the
table in section "1 · Только ядро" of the page "Ядра attention на домашней RTX
5080": Q and K are quantised to INT8 per block with FP32 scales, the product
P·V runs in FP8 E4M3.  The page gives only that description.  The granularity
is one scale per 128-token block per head for Q/K (the block size of the key tile
the kernels stream) and one scale per head and channel for V.  This and everything
else below is a reading of the plainest kind:

* Q/K block = 128 consecutive tokens x all D channels of one (b, h); the last
  block of a sequence may be partial.
* amax = max |x| over the block (exact, order-free);  s = amax / 127 in fp32;
  q = clamp(round_half_even(x / s), -127, 127) with ``x / s`` an fp32
  division; amax == 0 gives s = 0 and all codes 0.
* V channel c of one (b, hkv): s_c = amax_c / 448 in fp32 (448 is the largest
  finite E4M3 value); code = e4m3(V / s_c) rounded to nearest-even with
  saturation to +-448; s_c == 0 gives code 0.  V codes are stored transposed,
  ``[B, Hkv, D, S_pad]`` with ``S_pad`` = ``S`` rounded up to 128, padding 0.

Each operation is one correctly rounded IEEE binary32 operation, so the GPU
quantiser must match these bytes exactly.
"""

from __future__ import annotations

import numpy as np

QK_BLOCK = 128
INT8_MAX = 127.0
E4M3_MAX = 448.0


# --------------------------------------------------------------------------
# FP8 E4M3 (OCP 8-bit floating point, the "FN" variant: 4 exponent bits with
# bias 7, 3 mantissa bits, subnormals, no infinities, S.1111.111 is NaN).
# --------------------------------------------------------------------------

def fp8_e4m3_decode(codes):
    """Value of each E4M3 code, from the format definition (float64; NaN codes -> nan)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, e - 7)
    subnormal = np.ldexp(m / 8.0, -6)
    val = np.where(e == 0, subnormal, normal)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def fp8_e4m3_encode(x):
    """Round float32 values to E4M3 codes: nearest, ties to even, saturating.

    Finite magnitudes above 448 (and +-inf) become +-448; NaN becomes 0x7F with
    the sign bit of the input.  The sign of a zero result is the input's sign.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)  # exact widening
    neg = np.signbit(x)
    isnan = np.isnan(x)
    a = np.where(isnan, 0.0, np.abs(x))
    a = np.minimum(a, E4M3_MAX)
    # Binade of a: a in [2^E, 2^(E+1)).  Below 2^-6 the spacing is fixed at 2^-9.
    _, e = np.frexp(a)
    E = np.maximum(e - 1, -6)
    quantum = np.ldexp(1.0, E - 3)            # spacing of 3-bit mantissas
    r = np.rint(a / quantum) * quantum        # exact scaling; rint is half-to-even
    r = np.minimum(r, E4M3_MAX)
    # Encode the representable value r.
    _, er = np.frexp(r)
    Er = er - 1
    is_sub = (r < 2.0 ** -6)
    sub_code = np.rint(r / 2.0 ** -9)
    exp_field = Er + 7
    man_field = np.rint(np.ldexp(r, -Er) * 8.0 - 8.0)
    code = np.where(is_sub, sub_code, exp_field * 8 + man_field)
    code = np.where(isnan, 0x7F, code).astype(np.int64)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------
# INT8 per-block quantiser for Q and K.
# --------------------------------------------------------------------------

def quantize_qk_int8(x):
    """Quantise Q or K, ``[B, H, S, D]`` (values exactly representable in fp32).

    Returns ``(codes int8 [B, H, S, D], scales float32 [B, H, ceil(S/128)])``.
    """
    x = np.asarray(x, dtype=np.float32)
    B, H, S, D = x.shape
    nblk = (S + QK_BLOCK - 1) // QK_BLOCK
    codes = np.zeros((B, H, S, D), dtype=np.int8)
    scales = np.zeros((B, H, nblk), dtype=np.float32)
    for t in range(nblk):
        blk = x[:, :, t * QK_BLOCK:(t + 1) * QK_BLOCK, :]
        amax = np.max(np.abs(blk), axis=(2, 3)).astype(np.float32)        # [B, H]
        s = (amax / np.float32(INT8_MAX)).astype(np.float32)               # fp32 division
        scales[:, :, t] = s
        s_b = s[:, :, None, None]
        safe = np.where(s_b > 0, s_b, np.float32(1.0)).astype(np.float32)
        r = (blk / safe).astype(np.float32)                                # fp32 division
        qv = np.clip(np.rint(r), -INT8_MAX, INT8_MAX)                      # half-to-even
        qv = np.where(s_b > 0, qv, 0.0)
        codes[:, :, t * QK_BLOCK:(t + 1) * QK_BLOCK, :] = qv.astype(np.int8)
    return codes, scales


# --------------------------------------------------------------------------
# FP8 per-channel quantiser for V (transposed output).
# --------------------------------------------------------------------------

def padded_len(S):
    """Sequence length rounded up to the 128-token block."""
    return (S + QK_BLOCK - 1) // QK_BLOCK * QK_BLOCK


def quantize_v_fp8(v):
    """Quantise V, ``[B, Hkv, S, D]``.

    Returns ``(codes uint8 [B, Hkv, D, S_pad], scales float32 [B, Hkv, D])``.
    """
    v = np.asarray(v, dtype=np.float32)
    B, H, S, D = v.shape
    amax = np.max(np.abs(v), axis=2).astype(np.float32)                   # [B, H, D]
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)                  # fp32 division
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    r = (v / safe[:, :, None, :]).astype(np.float32)                      # fp32 division
    codes = fp8_e4m3_encode(r)
    codes = np.where((s > 0)[:, :, None, :], codes, np.uint8(0)).astype(np.uint8)
    out = np.zeros((B, H, D, padded_len(S)), dtype=np.uint8)
    out[:, :, :, :S] = np.transpose(codes, (0, 1, 3, 2))
    return out, s


def dequantize_qk(codes, scales):
    """float64 values represented by INT8 codes and their per-block scales."""
    codes = np.asarray(codes).astype(np.float64)
    scales = np.asarray(scales).astype(np.float64)
    S = codes.shape[2]
    s_tok = np.repeat(scales, QK_BLOCK, axis=2)[:, :, :S]
    return codes * s_tok[..., None]


def dequantize_v(codes_t, scales, S):
    """float64 V ``[B, Hkv, S, D]`` represented by transposed E4M3 codes."""
    vals = fp8_e4m3_decode(codes_t[:, :, :, :S])                           # [B, H, D, S]
    vals = vals * np.asarray(scales, dtype=np.float64)[:, :, :, None]
    return np.transpose(vals, (0, 1, 3, 2))
