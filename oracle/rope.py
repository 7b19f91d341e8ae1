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

Pair layouts: "half" pairs channel i with channel i + D/2; "interleaved" pairs
2i with 2i + 1.  Parity status: pinned by tests/test_oracle_rope.py (closed
forms, invariants, a hand-worked case); the CUDA path has no RoPE yet.
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

    positions: [S] absolute positions of the S rows; theta: [D/2].
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    assert theta.shape == (D // 2,)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]   # [S, D/2]
    c, s = np.cos(ang), np.sin(ang)
    if layout == "half":
        a, b = x[..., : D // 2], x[..., D // 2:]
        out = np.concatenate([a * c - b * s, a * s + b * c], axis=-1)
    elif layout == "interleaved":
        a, b = x[..., 0::2], x[..., 1::2]
        out = np.empty_like(x)
        out[..., 0::2] = a * c - b * s
        out[..., 1::2] = a * s + b * c
    else:
        raise ValueError(f"unknown layout {layout!r}")
    return out * mscale
