"""Plain, slow, obviously correct CPU oracle (float64 attention, reference quantisers).

TEST INFRASTRUCTURE ONLY: ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / ``--impl reference`` legs of ``bench.py`` may import it; the
product library never does.  It shares no code, headers or tables with the CUDA
path in ``attention_forward_flash_b200/``.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against hand-worked examples, brute force, closed forms and library special
cases.
"""

from .attention import (  # noqa: F401
    attention_f64,
    attention_f64_mixed,
    diagonal_band_start,
    attention_flops,
    gather_paged,
    visible_pairs,
    visible_range,
)
from .rope import (  # noqa: F401
    apply_rope,
    apply_rope_f32,
    rope_frequencies,
    rope_table,
    yarn_attention_factor,
)
from .quant import (  # noqa: F401
    E4M3_MAX,
    QK_BLOCK,
    dequantize_qk,
    dequantize_v,
    fp8_e4m3_decode,
    fp8_e4m3_encode,
    padded_len,
    quantize_qk_int8,
    quantize_v_fp8,
)
