"""3-axis rotary position embedding (RoPE), float64.

Follows "Day 0 Support for MiniMax-H3 on AMD Instinct GPUs", section "The
diffusion transformer (DiT)" (position encoding: Rotary (RoPE)), applied on
the (t, h, w) positions of the joint sequence.

Readings (the pages do not print the rotation):
* the head dimension D is split into contiguous axis chunks of widths
  (d_t, d_h, d_w), in that order, each even, summing to D;
* inside an axis chunk of width d_a starting at channel c_a, pair j
  (j < d_a/2) is rotated by the angle p_a * omega_j with
  omega_j = theta ** (-2 j / d_a);
* pair layout "interleaved": pair j is channels (c_a+2j, c_a+2j+1), the
  rotary embedding's original formulation; "half" (channels c_a+j and
  c_a+j+d_a/2) is kept as a switch so the reading can change in one place;
* the rotation of (x0, x1) by phi is (x0 cos phi - x1 sin phi,
  x0 sin phi + x1 cos phi).
Positions arrive as float32 values and are used exactly (widened to
float64); the angle, cos and sin are float64.
"""

from __future__ import annotations

import numpy as np


def rope_inv_freq(d_a: int, theta: float) -> np.ndarray:
    """omega_j = theta ** (-2 j / d_a) for j < d_a / 2, float64."""
    j = np.arange(d_a // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * j / np.float64(d_a))


def _pair_channels(c_a: int, d_a: int, pair_layout: str):
    j = np.arange(d_a // 2)
    if pair_layout == "interleaved":
        return c_a + 2 * j, c_a + 2 * j + 1
    if pair_layout == "half":
        return c_a + j, c_a + j + d_a // 2
    raise ValueError(pair_layout)


def rope_ref(x: np.ndarray, pos: np.ndarray, split, theta: float,
             pair_layout: str = "interleaved") -> np.ndarray:
    """Rotate x [N, H, D] (float64) by positions pos [N, 3]; returns float64.

    ``split`` = (d_t, d_h, d_w). Values are not rounded.
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos).astype(np.float64)
    N, H, D = x.shape
    if sum(split) != D or any(d % 2 for d in split):
        raise ValueError("split must be even widths summing to D")
    out = x.copy()
    c_a = 0
    for a, d_a in enumerate(split):
        if d_a == 0:
            continue
        omega = rope_inv_freq(d_a, theta)                     # [d_a/2]
        phi = pos[:, a:a + 1] * omega[None, :]                 # [N, d_a/2]
        cos = np.cos(phi)[:, None, :]
        sin = np.sin(phi)[:, None, :]
        i0, i1 = _pair_channels(c_a, d_a, pair_layout)
        x0 = x[:, :, i0]
        x1 = x[:, :, i1]
        out[:, :, i0] = x0 * cos - x1 * sin
        out[:, :, i1] = x0 * sin + x1 * cos
        c_a += d_a
    return out
