"""fp64 CPU oracle for exact IO-aware attention.

This package is TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it. The product package (``io_aware_exact_27_b200``) never imports it, shares no
code with it, and fails loudly instead of falling back to it.

Sources (the web pages this library restates):
  * "Dao and colleagues: IO-aware exact attention with FlashAttention"
    (catalogue record, fields ``summary`` and ``boundary``): exact attention,
    computed tile by tile with recomputation, the full attention matrix never
    materialised; the dense algorithm changes memory access, not the result.
  * "Flash Attention and Efficient Transformer Mechanisms" (topic page, opening
    paragraphs): blocks of Q, K, V read into SRAM, partial attention outputs,
    "without approximation".
  * Dao-AILab flash-attention repository overview (architecture paragraph):
    online softmax with rescaling, tiled attention, varlen API.
  * "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
    Low-precision" (summary, contribution 3): FP8 GEMMs in the forward pass.

The pages print no formula, so the plain definition of scaled dot-product
attention with a causal mask, a per-row log-sum-exp and the analytic gradient is
written out here (``attention.py``); the tiled online-softmax algorithm the
pages describe in words is restated separately (``tiled.py``) and pinned to the
plain definition by the tests. Parity of every function here is pinned by
``tests/test_oracle_pins.py`` (closed forms, invariants, brute force, finite
differences and an independent library routine).
"""

from .attention import (  # noqa: F401
    kv_head_of,
    attention_head,
    attn_fwd,
    attn_fwd_rows,
    attn_fwd_varlen,
    attn_bwd,
    attn_bwd_varlen,
    attn_bwd_rows,
    attn_bwd_block,
    attn_fwd_kvcache,
    attn_fwd_blocksparse,
    attn_bwd_blocksparse,
    merge_partials,
    dequantize_blockscaled,
)
from .tiled import attn_head_tiled  # noqa: F401
from .quant import hadamard, fwht_f32, rotate_f32, quantize_blockscaled, dequantize_f32  # noqa: F401
from .metrics import max_abs, rel_rms  # noqa: F401
