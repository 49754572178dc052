"""CPU oracle for the joint video+audio attention path (float64, NumPy).

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check in
``__graft_entry__.smoke`` and the benchmark's CPU-baseline leg may import
this package. The product path (the CUDA library and its Python binding)
never imports, links or calls it, and shares no code with it.

What it computes, and the passages it follows:

* ``positions``   -- per-token (t, h, w) rotary positions on the shared
  audio/video temporal clock, built in float64 and rounded once to float32
  ("MiniMax-H3 Reference" Space README, section "References": ordered
  references advance the shared audio/video rotary clock; "MiniMax H3 on
  Moore Threads MUSA", section "MUSA validation": FP64 position metadata is
  cast to FP32 before device arithmetic).
* ``rope``        -- 3-axis rotary embedding of q and k ("Day 0 Support for
  MiniMax-H3 on AMD Instinct GPUs", section "The diffusion transformer
  (DiT)": position encoding is Rotary (RoPE)).
* ``attention``   -- non-causal softmax attention inside each packed
  segment ("MiniMax H3" vLLM-Omni recipe, section "Step execution and
  continuous batching": one attention document per packed request).
* ``skip_softmax`` -- the lossy Skip-Softmax variant that drops negligible
  key tiles ("MiniMax H3" vLLM-Omni recipe, section "Attention Backends").
* ``qkv_rope``    -- the qkv projection with RoPE applied to q and k in its
  epilogue ("MiniMax-H3 Reference" Space README, section "AoTI-compiled
  blocks": rotary epilogues around the block's matmuls).
* ``sage``        -- the lossy SAGE-style FP8 attention: e4m3 Q/K with
  per-token and per-16-key scales, FP8 P and V ("MiniMax H3" vLLM-Omni
  recipe, section "Attention Backends"), with its e4m3 codec.

Readings where the pages say nothing (pair layout, frequency schedule,
audio-token clock, reference layout) are listed in the design notes of the
repository; each function's docstring names the one it relies on.

Pins: every function here is checked by ``tests/test_oracle.py`` against
brute force, closed forms and invariants, not against itself. The rotary
pair layout and per-axis frequency schedule are a documented reading:
"parity unpinned" against the real model, which the pages never print.
"""

from .bf16 import bf16_bits_to_f64  # noqa: F401
from .positions import segment_positions, packed_positions  # noqa: F401
from .rope import rope_ref, rope_inv_freq  # noqa: F401
from .attention import (  # noqa: F401
    attention_ref,
    attention_dense_bruteforce,
    attention_rows_ref,
)
from .skip_softmax import attention_skip_ref, attention_skip_rows_ref  # noqa: F401
from .qkv_rope import qkv_rope_ref  # noqa: F401
from .sage import (  # noqa: F401
    e4m3_decode,
    e4m3_encode,
    e4m3_round,
    sage_quantize,
    sage_attention_ref,
    sage_attention_rows_ref,
)
