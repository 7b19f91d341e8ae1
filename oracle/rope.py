"""FP64 rotary position embedding (RoPE) with NTK-aware and YaRN frequency scaling.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).  The page "Ядра attention на
домашней RTX 5080" (section "Планы · Rigsy Kernel") plans RoPE "with NTK / YaRN
scaling" inside the attention kernel instead of a separate pass; it gives no
formulas.  These are the published definitions, restated:

* RoPE (Su et al., "RoFormer"): channel pair i of a head of width D rotates by the
  angle ``p * theta_i`` at position p, with ``theta_i = base ** (-2 i / D)``,
  i = 0 .. D/2 - 1.
* NTK-aware scaling (the "NTK-aware scaled RoPE" proposal): the base becomes
  ``base * alpha ** (D / (D - 2))`` for a context-extension factor alpha.
* YaRN (Peng et al., "YaRN: Efficient Context Window Extension of Large Language
  Models"): with scale s and original context length L, pair i has wavelength
  ``2 pi / theta_i`` and ratio ``r_i = L * theta_i / (2 pi)``; the ramp
  ``g_i = clamp((r_i - beta_slow) / (beta_fast - beta_slow), 0, 1)`` blends the
  interpolated and the original frequency, ``theta'_i = (1 - g_i) theta_i / s +
  g_i theta_i``, and the logits are scaled by ``(0.1 ln s + 1) ** 2`` (each of q
  and k carries one factor ``0.1 ln s + 1``).

Pair layouts: "half" pairs channel i with channel i + R/2; "interleaved" pairs
2i with 2i + 1, over the first R = rotary_dim channels (R = D unless a partial
rotary width is given; the channels past R pass through unchanged, as in models
that rotate only part of each head).

Two forms:

* ``apply_rope``: the definition in float64 (angles, cosines and sines in float64).
* ``apply_rope_f32``: the rotation as single correctly rounded float32 operations
  on a float32 table of cosines and sines -- for a pair (a, b) with table entries
  (c, s): a' = RN(RN(a c) - RN(b s)), b' = RN(RN(a s) + RN(b c)).  The pages
  give no precision for RoPE; this float32 form is the reading under which the
  quantised mode's INT8 codes of rotated Q and K are reproducible bit for bit
  (the table is an input shared by value, the operations are fixed).
  ``rope_table`` builds the table from the definition (float64, then rounded).

Parity status: pinned by tests/test_oracle_rope.py (closed forms, invariants,
hand-worked cases, the float32 form against the float64 one within its rounding
bound).
"""

from __future__ import annotations

import math

import numpy as np


def rope_frequencies(D, *, base=10000.0, scaling=None, factor=1.0, original_len=None,
                     beta_fast=32.0, beta_slow=1.0):
    """theta_i (float64, length D/2) for ``scaling`` in (None, "ntk", "yarn")."""
    assert D % 2 == 0 and D >= 2
    i = np.arange(D // 2, dtype=np.float64)
    if scaling == "ntk":
        base = base * factor ** (D / (D - 2))
    theta = base ** (-2.0 * i / D)
    if scaling == "yarn":
        assert original_len is not None and beta_fast > beta_slow
        r = original_len * theta / (2.0 * math.pi)
        g = np.clip((r - beta_slow) / (beta_fast - beta_slow), 0.0, 1.0)
        theta = (1.0 - g) * theta / factor + g * theta
    elif scaling not in (None, "ntk"):
        raise ValueError(f"unknown scaling {scaling!r}")
    return theta


def yarn_attention_factor(factor):
    """Per-tensor multiplier 0.1 ln s + 1 (q and k each carry one; 1 for s <= 1)."""
    return 0.1 * math.log(factor) + 1.0 if factor > 1.0 else 1.0


def apply_rope(x, positions, theta, *, layout="half", mscale=1.0):
    """Rotates the last axis of ``x`` [..., S, D] by position (float64 result).

    positions: [S] absolute positions of the S rows; theta: [R/2] for a rotary
    width R <= D (R = 2 * len(theta)); channels R .. D-1 are returned unchanged
    (times mscale, which multiplies the whole vector as the YaRN attention factor).
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    R = 2 * theta.shape[0]
    assert theta.ndim == 1 and 2 <= R <= D and R % 2 == 0
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]   # [S, R/2]
    c, s = np.cos(ang), np.sin(ang)
    out = x.copy()
    if layout == "half":
        a, b = x[..., : R // 2], x[..., R // 2:R]
        out[..., : R // 2] = a * c - b * s
        out[..., R // 2:R] = a * s + b * c
    elif layout == "interleaved":
        a, b = x[..., 0:R:2], x[..., 1:R:2]
        out[..., 0:R:2] = a * c - b * s
        out[..., 1:R:2] = a * s + b * c
    else:
        raise ValueError(f"unknown layout {layout!r}")
    return out * mscale


def rope_table(n_pos, theta, mscale=1.0):
    """float32 table [n_pos, 2, R/2]: cos and sin of p * theta_i for p = 0 .. n_pos-1,
    each times mscale, computed in float64 and rounded once to float32."""
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * np.asarray(theta, np.float64)[None, :]
    return np.stack([np.cos(ang) * mscale, np.sin(ang) * mscale], axis=1).astype(np.float32)


def apply_rope_f32(x, positions, table, *, layout="half"):
    """RoPE as float32 operations on a float32 table (see the module docstring).

    x: [..., S, D] float32-representable values; positions: [S]; table: float32
    [n_pos, 2, R/2] (cos, then sin; the YaRN factor, if any, already folded in).
    Returns float32.  Channels R .. D-1 are returned unchanged (no factor: a table
    with mscale != 1 is meant for R = D).
    """
    x = np.asarray(x, dtype=np.float32)
    table = np.asarray(table, dtype=np.float32)
    D = x.shape[-1]
    R = 2 * table.shape[2]
    assert 2 <= R <= D
    pos = np.asarray(positions, dtype=np.int64)
    c = table[pos, 0, :]                                   # [S, R/2]
    s = table[pos, 1, :]
    out = x.copy()
    if layout == "half":
        a, b = x[..., : R // 2], x[..., R // 2:R]
    elif layout == "interleaved":
        a, b = x[..., 0:R:2], x[..., 1:R:2]
    else:
        raise ValueError(f"unknown layout {layout!r}")
    # every product and sum is one float32 operation (numpy rounds each one)
    lo = np.subtract(np.multiply(a, c, dtype=np.float32), np.multiply(b, s, dtype=np.float32),
                     dtype=np.float32)
    hi = np.add(np.multiply(a, s, dtype=np.float32), np.multiply(b, c, dtype=np.float32),
                dtype=np.float32)
    if layout == "half":
        out[..., : R // 2] = lo
        out[..., R // 2:R] = hi
    else:
        out[..., 0:R:2] = lo
        out[..., 1:R:2] = hi
    return out
