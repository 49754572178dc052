"""Seeded synthetic inputs for the joint video+audio attention path.

This package is shared by the tests, the benchmark and the oracle's checks.
It holds workload *descriptions* (segment layouts, head counts, head dim,
rotary split, seeds) and the seeded random draws of q/k/v as bf16 bit
patterns. It holds none of the method's arithmetic: token positions, the
rotary embedding and attention are computed separately by the oracle
(``oracle/``) and by the CUDA library, each from its own code.
"""

from .configs import (  # noqa: F401
    SegmentLayout,
    Workload,
    WORKLOADS,
    workload,
    draw_qkv,
    draw_random_case,
    draw_group_case,
    f32_to_bf16_bits,
    cu_seqlens_of,
    QkvProjection,
    QKV_PROJECTION,
    draw_linear_case,
)
