"""Seeded synthetic workloads, shared by the tests, the bench and the smoke check.

This module only draws random numbers and casts them; it holds none of the
attention arithmetic, so both the CUDA path and the float64 oracle can be fed
from it without sharing any of the method.

Shapes mirror the pages' workloads:

* ``decode``: "Performance evidence" of the page "perf(metal): widen four-row
  flash KV tiles - #89" -- 4 query rows at position 4092, 16 query heads over 8
  key/value heads, head_dim 128, kv_len 4096, f16, causal; ``decode_window``
  adds the page's non-aligned last KV chunk and a window lower bound inside the
  first chunk (its "Summary").
* ``video``: section "1 · Только ядро" of the page "Ядра attention на домашней
  RTX 5080" -- 1 x 40 heads x 32760 tokens x 128, bf16.
* ``image``: a 64x64-latent diffusion self-attention (the page "Shmoosh update"
  works on 1024px image diffusion), with a per-channel offset on K that gives
  the channel outliers per-block INT8 quantisation has to cope with.
* ``llm``: a causal GQA prefill with 1% of K entries scaled by 20.
* ``llm_window``: the same shape with a per-row sliding window of 1024 positions
  (each query row sees the last 1024 keys up to its own).
* ``video_rope`` / ``llm_rope``: the video and causal GQA prefill shapes with
  rotary position embedding on all head_dim channels (the RoPE "inside the
  kernel" planned in section "Планы · Rigsy Kernel" of the RTX 5080 page).
* ``tiny``: a small exact case the oracle finishes in well under a second.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws float32
standard normals in the order Q, K, V, then the perturbation; the results are
cast to bf16/fp16 with round-to-nearest-even.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    q_len: int
    kv_len: int
    head_dim: int
    dtype: str = "bf16"          # "bf16" | "fp16"
    causal: bool = False
    start_pos: int = 0
    window_lo: int = 0
    window_size: int = 0                 # sliding window W (0: none)
    modes: tuple = ("exact",)    # precision modes this workload is run in
    seed: int = 1000
    k_channel_offset_var: float = 0.0   # per-(b,h) channel offset ~ N(0, var) added to K
    k_outlier_frac: float = 0.0         # fraction of K entries multiplied by k_outlier_mult
    k_outlier_mult: float = 1.0
    oracle_rows: int = 0                 # 0: every row; else a seeded subset per head
    rope_dim: int = 0                    # rotary channels (0: no RoPE)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    def shapes(self):
        return ((self.batch, self.n_q_heads, self.q_len, self.head_dim),
                (self.batch, self.n_kv_heads, self.kv_len, self.head_dim))

    def flops(self):
        """Headline work count: 4*B*Hq*Sq*Skv*D, halved for causal."""
        f = 4.0 * self.batch * self.n_q_heads * self.q_len * self.kv_len * self.head_dim
        return f / 2 if self.causal else f

    def scaled(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 256, 64, "bf16", seed=1000),
    "decode": Workload("decode", 1, 16, 8, 4, 4096, 128, "fp16", causal=True, start_pos=4092,
                       seed=1001),
    "decode_window": Workload("decode_window", 1, 16, 8, 4, 4133, 128, "fp16", causal=True,
                              start_pos=4129, window_lo=40, seed=1011),
    "image": Workload("image", 2, 10, 10, 4096, 4096, 64, "bf16",
                      modes=("exact", "quant", "fp4"),
                      seed=1002, k_channel_offset_var=2.0),
    "video": Workload("video", 1, 40, 40, 32760, 32760, 128, "bf16", modes=("exact", "quant"),
                      seed=1003, oracle_rows=256),
    "llm": Workload("llm", 4, 32, 8, 8192, 8192, 128, "bf16", causal=True,
                    modes=("exact", "quant", "mixed"), seed=1004, k_outlier_frac=0.01,
                    k_outlier_mult=20.0, oracle_rows=256),
    # the causal GQA prefill with a 1024-position sliding window per row
    "llm_window": Workload("llm_window", 4, 32, 8, 8192, 8192, 128, "bf16", causal=True,
                           window_size=1024, modes=("exact", "quant"), seed=1005,
                           oracle_rows=256),
    # rotary position embedding on every channel (plain frequencies, base 10000)
    "video_rope": Workload("video_rope", 1, 40, 40, 32760, 32760, 128, "bf16",
                           modes=("exact", "quant"), seed=1006, oracle_rows=256, rope_dim=128),
    "llm_rope": Workload("llm_rope", 4, 32, 8, 8192, 8192, 128, "bf16", causal=True,
                         modes=("exact", "quant"), seed=1007, oracle_rows=256, rope_dim=128),
}


def make_qkv(w: Workload, device="cpu"):
    """Draw (q, k, v) for workload ``w`` on the CPU, then move them to ``device``."""
    g = torch.Generator().manual_seed(w.seed)
    qs, ks = w.shapes()
    q = torch.randn(qs, generator=g, dtype=torch.float32)
    k = torch.randn(ks, generator=g, dtype=torch.float32)
    v = torch.randn(ks, generator=g, dtype=torch.float32)
    if w.k_channel_offset_var > 0:
        off = torch.randn((w.batch, w.n_kv_heads, 1, w.head_dim), generator=g,
                          dtype=torch.float32) * math.sqrt(w.k_channel_offset_var)
        k += off
    if w.k_outlier_frac > 0:
        sel = torch.rand(ks, generator=g, dtype=torch.float32) < w.k_outlier_frac
        k = torch.where(sel, k * w.k_outlier_mult, k)
    dt = w.torch_dtype
    out = tuple(t.to(dt) for t in (q, k, v))
    if device != "cpu":
        out = tuple(t.to(device) for t in out)
    return out


def make_qkv_device(w: Workload, device):
    """Same recipe as ``make_qkv`` but drawn by a generator on ``device``.

    Used where only the distribution matters (timing); the random stream differs
    from the CPU one, so parity tests use ``make_qkv``.
    """
    g = torch.Generator(device=device).manual_seed(w.seed)
    qs, ks = w.shapes()
    dt = w.torch_dtype
    q = torch.randn(qs, generator=g, device=device, dtype=torch.float32).to(dt)
    k = torch.randn(ks, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(ks, generator=g, device=device, dtype=torch.float32).to(dt)
    if w.k_channel_offset_var > 0:
        k += torch.randn((w.batch, w.n_kv_heads, 1, w.head_dim), generator=g, device=device,
                         dtype=torch.float32) * math.sqrt(w.k_channel_offset_var)
    if w.k_outlier_frac > 0:
        sel = torch.rand(ks, generator=g, device=device, dtype=torch.float32) < w.k_outlier_frac
        k = torch.where(sel, k * w.k_outlier_mult, k)
    return q, k.to(dt), v


def sample_rows(w: Workload, n=None, seed=None):
    """Seeded subset of query rows (sorted) evaluated by the oracle on large workloads."""
    n = w.oracle_rows if n is None else n
    if n <= 0 or n >= w.q_len:
        return torch.arange(w.q_len)
    g = torch.Generator().manual_seed(w.seed + 7 if seed is None else seed)
    idx = torch.randperm(w.q_len, generator=g)[:n]
    # always include the first and the last (ragged) rows
    idx = torch.unique(torch.cat([idx[:n - 2], torch.tensor([0, w.q_len - 1])]))
    return idx.sort().values
