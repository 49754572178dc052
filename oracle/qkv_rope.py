"""QKV projection with the rotary embedding applied to its q and k outputs, float64.

"MiniMax-H3 Reference" Space README, section "AoTI-compiled blocks": the
norm / rotary / AdaLN epilogues run around the block's matmuls; "MiniMax H3"
vLLM-Omni recipe, section "Online FP8 quantization": the attention's qkv
projection is one of the DiT's linears. Definition:
    Y = X W^T                  (X [N, K], W [3 H D, K])
    q = Y[:, 0:HD], k = Y[:, HD:2HD], v = Y[:, 2HD:3HD]   (each [N, H, D])
    q, k <- RoPE(q, pos), RoPE(k, pos)   (oracle.rope, same reading)
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64
from .rope import rope_ref


def qkv_rope_ref(x, w, heads, head_dim, pos=None, split=None, theta=10000.0,
                 pair_layout="interleaved", rows=None):
    """Returns (q, k, v) float64 [n, H, D]; ``rows`` selects token rows."""
    X = _as_f64(x if rows is None else np.asarray(x)[rows])
    W = _as_f64(w)
    Y = X @ W.T
    HD = heads * head_dim
    q = Y[:, :HD].reshape(-1, heads, head_dim)
    k = Y[:, HD:2 * HD].reshape(-1, heads, head_dim)
    v = Y[:, 2 * HD:].reshape(-1, heads, head_dim)
    if pos is not None:
        P = np.asarray(pos) if rows is None else np.asarray(pos)[rows]
        q = rope_ref(q, P, split, theta, pair_layout)
        k = rope_ref(k, P, split, theta, pair_layout)
    return q, k, v
