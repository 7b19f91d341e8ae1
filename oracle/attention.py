"""FP64 CPU oracle for the fused attention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: it
is used by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``.  It shares no code with the CUDA library.

What it computes is the plain definition of scaled-dot-product attention, the
computation all the source pages turn on:

    O = softmax(scale * Q K^T + mask) V

* "Performance evidence" of the page "perf(metal): widen four-row flash KV
  tiles - #89" fixes the problem statement: query rows, ``n_head`` query heads
  sharing ``n_kv`` key/value heads, ``head_dim``, ``kv_len``, a start position
  ``pos`` of query row 0 and a causal mask.
* "Summary" of the same page adds a sliding-window lower bound on the keys.
* Table "1 · Только ядро" of the page "Ядра attention на домашней RTX 5080"
  gives the SDPA workload (1 x 40 heads x 32760 tokens x 128, bf16) against
  which reduced-precision kernels are judged by their relative difference to
  the full-precision result.

The flash method (online softmax over key tiles) reaches exactly this result up
to rounding order, so the oracle is the definition written out, with a library
matmul as the only primitive and no tiling.

Readings taken where the pages are silent:

* layout ``[B, H, S, D]`` contiguous;
* query head ``hq`` reads key/value head ``hq // (Hq // Hkv)`` (contiguous
  groups);
* query row ``i`` sits at absolute position ``start_pos + i``; with ``causal``
  it sees keys ``j <= start_pos + i``;
* ``window_lo`` is an inclusive absolute lower bound on the key index, applied
  with or without ``causal``;
* ``window_size`` W > 0 adds a per-row sliding window: row ``i`` (position
  ``p = start_pos + i``) sees keys ``j >= p - W + 1``, i.e. the last W positions
  up to its own when causal.  The pages name only a window lower bound (the
  "Summary" above) and position/window test cases ("round 21 track b -- qsa2",
  section "experiment contract"); the per-row form is the usual sliding window
  read from that lower bound, applied together with ``window_lo`` (the larger
  bound wins);
* a row that sees no key returns O = 0 and lse = -inf;
* ``scale`` defaults to ``1/sqrt(D)``.
"""

from __future__ import annotations

import math

import numpy as np


def visible_range(i, *, kv_len, start_pos=0, causal=False, window_lo=0, window_size=0):
    """Inclusive key range ``[lo, hi]`` seen by query row ``i`` (empty if lo > hi).

    Row ``i`` is at absolute position ``start_pos + i`` (the ``pos`` of
    "Performance evidence", page "perf(metal): widen four-row flash KV tiles").
    ``window_size`` W > 0 keeps only keys ``j >= start_pos + i - W + 1``.
    """
    lo = max(int(window_lo), 0)
    if window_size > 0:
        lo = max(lo, int(start_pos) + int(i) - int(window_size) + 1)
    hi = kv_len - 1
    if causal:
        hi = min(hi, int(start_pos) + int(i))
    return lo, hi


def gather_paged(pool, block_table, kv_len):
    """Dense keys (or values) ``[B, Hkv, kv_len, D]`` of a paged cache.

    ``pool`` is ``[num_blocks, Hkv, 128, D]`` and ``block_table`` is ``[B, ceil(kv_len / 128)]``:
    position ``128 t + r`` of batch entry ``b`` is ``pool[block_table[b, t], :, r, :]``.  The
    pages show no cache layout; this is the block-table reading of the qsa2 audit's
    32768-cell KV cache ("round 21 track b -- qsa2", section "build and reproduction").
    """
    pool = _as_f64(pool)
    table = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table,
                       dtype=np.int64)
    B, nbt = table.shape
    _, Hkv, bs, D = pool.shape
    assert bs == 128 and nbt * 128 >= kv_len
    out = np.empty((B, Hkv, kv_len, D), dtype=np.float64)
    for b in range(B):
        for t in range(nbt):
            n = min(128, kv_len - 128 * t)
            out[b, :, 128 * t:128 * t + n, :] = pool[table[b, t], :, :n, :]
    return out


def _as_f64(x):
    """Widen a torch tensor (bf16/fp16/fp32, any device) or array to float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself only needs numpy

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attention_f64(q, k, v, *, scale=None, causal=False, start_pos=0, window_lo=0,
                  window_size=0, rows=None, return_probs=False):
    """Attention forward in float64.

    Arguments
      q : [B, Hq, Sq, D];  k, v : [B, Hkv, Skv, D]  (any float dtype; widened exactly)
      scale : multiplier of Q K^T (default 1/sqrt(D))
      causal, start_pos, window_lo, window_size : mask parameters, see ``visible_range``
      rows : optional 1-D index array of query rows to evaluate (same rows for
             every (b, hq)); default all rows
      return_probs : also return the softmax matrix P [B, Hq, len(rows), Skv]

    Returns (O [B, Hq, R, D] float64, lse [B, Hq, R] float64[, P]) where
    lse = natural-log of sum_j exp(scale * q.k_j) over the visible keys.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    assert Bk == B and Dk == D and v.shape == k.shape
    assert Hq % Hkv == 0, "GQA needs n_q_heads to be a multiple of n_kv_heads"
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if rows is None:
        rows = np.arange(Sq)
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]

    # Visibility of key j for row i: lo_i <= j <= hi_i.
    lo = np.empty(R, dtype=np.int64)
    hi = np.empty(R, dtype=np.int64)
    for n, i in enumerate(rows):
        lo[n], hi[n] = visible_range(int(i), kv_len=Skv, start_pos=start_pos,
                                     causal=causal, window_lo=window_lo,
                                     window_size=window_size)
    j = np.arange(Skv)
    vis = (j[None, :] >= lo[:, None]) & (j[None, :] <= hi[:, None])  # [R, Skv]
    any_vis = vis.any(axis=1)
    # O sums over each row's visible keys only.  P is 0 at masked keys, and a key
    # that no evaluated row sees is also removed from V, so that a non-finite value
    # there (0 * inf or 0 * nan) cannot reach the product.
    seen = vis.any(axis=0)                                            # [Skv]

    out = np.zeros((B, Hq, R, D), dtype=np.float64)
    lse = np.full((B, Hq, R), -np.inf, dtype=np.float64)
    probs = np.zeros((B, Hq, R, Skv), dtype=np.float64) if return_probs else None

    for b in range(B):
        for hq in range(Hq):
            hk = hq // group
            if Skv == 0:                                    # no key at all: every row is empty
                continue
            s = scale * (q[b, hq, rows, :] @ k[b, hk].T)  # [R, Skv] scores
            s = np.where(vis, s, -np.inf)                  # masked keys
            m = np.max(s, axis=1)                           # row max (-inf if none)
            m_safe = np.where(any_vis, m, 0.0)
            p = np.where(vis, np.exp(s - m_safe[:, None]), 0.0)
            l = p.sum(axis=1)
            l_safe = np.where(any_vis, l, 1.0)
            p = p / l_safe[:, None]                         # softmax rows
            out[b, hq] = p @ np.where(seen[:, None], v[b, hk], 0.0)
            lse[b, hq] = np.where(any_vis, m_safe + np.log(l_safe), -np.inf)
            if return_probs:
                probs[b, hq] = p
    if return_probs:
        return out, lse, probs
    return out, lse


def attention_flops(B, Hq, Sq, Skv, D, *, causal=False):
    """Work count of the headline metric: 4*B*Hq*Sq*Skv*D, halved for causal.

    The 4 = 2 (multiply-add) x 2 (Q K^T and P V).  The same count reproduces the
    "≈ 520 TOPS" the page "Ядра attention на домашней RTX 5080" quotes for a
    42 ms kernel at 1 x 40 x 32760 x 128 (section "1 · Только ядро").
    """
    f = 4.0 * B * Hq * Sq * Skv * D
    return f / 2.0 if causal else f


def visible_pairs(Sq, Skv, *, start_pos=0, causal=False, window_lo=0, window_size=0):
    """Exact number of visible (query, key) pairs of one head."""
    n = 0
    for i in range(Sq):
        lo, hi = visible_range(i, kv_len=Skv, start_pos=start_pos, causal=causal,
                               window_lo=window_lo, window_size=window_size)
        n += max(0, hi - lo + 1)
    return n


def diagonal_band_start(i, hq, *, Sq, n_q_heads, n_kv_heads, start_pos=0, causal=True,
                        query_tile=256, key_tile=128):
    """First key of the causal diagonal band of query row ``i`` of head ``hq``.

    The diagonal-tiled mixed precision of the page "Transformers Get a Turbo Boost
    with Mixed-Precision Magic" chooses the arithmetic per tile; the page does not
    say which tiles are "diagonal".  Reading: the query rows of a unit (the
    ``G = n_q_heads / n_kv_heads`` heads sharing a kv head, stacked head-major,
    ``G * Sq`` rows) are cut into tiles of ``query_tile`` rows; the band of a query
    tile is every ``key_tile``-key tile that some row of it must partly mask for
    causality, i.e. the key tiles from the one holding the smallest position
    among its rows.  Without a causal mask there is no band (returns a key index
    past any sequence).
    """
    if not causal:
        return np.iinfo(np.int64).max
    G = n_q_heads // n_kv_heads
    r = (hq % G) * Sq + int(i)                      # stacked row within the unit
    t0 = (r // query_tile) * query_tile
    t1 = min(t0 + query_tile, G * Sq)
    stacked = np.arange(t0, t1)
    pos_min = int(start_pos) + int((stacked % Sq).min())
    # key tile jt is in the band when jt * key_tile + key_tile - 1 > pos_min
    return key_tile * ((pos_min + 1) // key_tile)


def attention_f64_mixed(q, k, q_low, k_low, v, *, scale=None, causal=False, start_pos=0,
                        rows=None, query_tile=256, key_tile=128):
    """Float64 attention whose scores come from (q, k) on each row's causal diagonal
    band (``diagonal_band_start``) and from (q_low, k_low) on every other key: the
    definition of the diagonal-tiled mixed precision mode, with the low-precision
    operands given as the values they represent (e.g. dequantised INT8 codes).
    Same conventions and returns as ``attention_f64`` (no sliding window)."""
    q, k, ql, kl, v = (_as_f64(x) for x in (q, k, q_low, k_low, v))
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    assert ql.shape == q.shape and kl.shape == k.shape and v.shape == k.shape
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((B, Hq, len(rows), D))
    lse = np.full((B, Hq, len(rows)), -np.inf)
    j = np.arange(Skv)
    for b in range(B):
        for hq in range(Hq):
            hk = hq // group
            for n, i in enumerate(rows):
                lo, hi = visible_range(int(i), kv_len=Skv, start_pos=start_pos, causal=causal)
                if hi < lo:
                    continue
                band = diagonal_band_start(i, hq, Sq=Sq, n_q_heads=Hq, n_kv_heads=Hkv,
                                           start_pos=start_pos, causal=causal,
                                           query_tile=query_tile, key_tile=key_tile)
                keys = j[lo:hi + 1]
                s = np.where(keys >= band, k[b, hk, lo:hi + 1] @ q[b, hq, i],
                             kl[b, hk, lo:hi + 1] @ ql[b, hq, i]) * scale
                m = s.max()
                p = np.exp(s - m)
                out[b, hq, n] = (p / p.sum()) @ v[b, hk, lo:hi + 1]
                lse[b, hq, n] = m + math.log(p.sum())
    return out, lse
