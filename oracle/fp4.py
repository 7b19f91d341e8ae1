"""Reference MXFP4 quantiser (FP4 E2M1 elements, one E8M0 scale per 32 elements).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  The page "Transformers Get a
Turbo Boost with Mixed-Precision Magic" names the microscaling floating-point (MXFP)
formats for low-bit attention on B200, and the page "Ядра attention на домашней RTX
5080" lists SageAttention 3's FP4 path; neither defines the formats.  This module
restates the OCP Microscaling Formats (MX) specification v1.0:

* E2M1 element: sign, 2 exponent bits (bias 1), 1 mantissa bit, no Inf or NaN.
  Exponent 0 is subnormal (0.m x 2^0); the finite magnitudes are
  0, 0.5, 1, 1.5, 2, 3, 4, 6.
* E8M0 scale: an unsigned 8-bit biased exponent e, value 2^(e - 127); 0xFF is NaN.
* Conversion of a block of 32 values V: X = 2^(floor(log2(max|V|)) - 2) (2 is the
  largest E2M1 exponent), then each element is V / X rounded to the nearest E2M1
  value, ties to the even code, and saturated to +-6.  An all-zero block takes the
  smallest scale and zero codes.

Parity status: pinned by tests/test_oracle_fp4.py; the CUDA path has no FP4 mode yet.
"""

from __future__ import annotations

import numpy as np

MX_BLOCK = 32
E2M1_EMAX = 2
E2M1_MAX = 6.0


def e2m1_decode(code):
    """Float64 values of 4-bit E2M1 codes (bit 3 sign, bits 2..1 exponent, bit 0 mantissa)."""
    code = np.asarray(code, dtype=np.int64) & 0xF
    sign = np.where(code & 0x8, -1.0, 1.0)
    e = (code >> 1) & 0x3
    m = (code & 0x1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, (1.0 + 0.5 * m) * 2.0 ** (e - 1))
    return sign * mag


def e2m1_encode(x):
    """Nearest E2M1 code of each value, ties to the even code, saturating at +-6.

    Written as a search over the eight magnitudes: the candidate with the smallest
    distance wins, and of two equally distant candidates the one with the even
    (mantissa bit 0) code.  Zero keeps its sign bit.
    """
    x = np.asarray(x, dtype=np.float64)
    mags = e2m1_decode(np.arange(8))                      # 0, 0.5, 1, 1.5, 2, 3, 4, 6
    a = np.minimum(np.abs(x), E2M1_MAX)
    d = np.abs(a[..., None] - mags)                       # [..., 8]
    best = np.min(d, axis=-1, keepdims=True)
    cand = d == best
    # among ties prefer the even code (mantissa bit 0), i.e. the even index
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    return (code | np.where(np.signbit(x), 0x8, 0)).astype(np.uint8)


def mxfp4_quantize(x, block=MX_BLOCK):
    """Quantises the last axis in blocks of ``block`` values.

    Returns (codes uint8 [..., n], scale_exp uint8 [..., n / block]) with the E8M0
    scale of each block as its biased exponent.
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    assert n % block == 0
    xb = x.reshape(x.shape[:-1] + (n // block, block))
    amax = np.max(np.abs(xb), axis=-1)
    with np.errstate(divide="ignore"):
        e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - E2M1_EMAX,
                     -127.0)
    e = np.clip(e, -127, 127)
    scale = 2.0 ** e
    codes = e2m1_encode(xb / scale[..., None]).reshape(x.shape)
    return codes, (e + 127).astype(np.uint8)


def mxfp4_dequantize(codes, scale_exp, block=MX_BLOCK):
    """Float64 values of MXFP4 codes and their E8M0 block scales."""
    codes = np.asarray(codes)
    n = codes.shape[-1]
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (n // block, block))
    scale = 2.0 ** (np.asarray(scale_exp, dtype=np.float64) - 127.0)
    return (vals * scale[..., None]).reshape(codes.shape)
