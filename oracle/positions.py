"""Per-token (t, h, w) positions on the shared audio/video clock.

Follows:
* "MiniMax-H3 Reference" Space README, section "References": references are
  read in order and that order advances the shared audio/video rotary clock.
* "MiniMax-H3 Reference" Space README, section "AoTI-compiled blocks": the
  reference rows are packed in front of the generated rows.
* "MiniMax H3 on Moore Threads MUSA", section "MUSA validation": position
  metadata is FP64 on the host and cast to FP32 before device arithmetic.
* "MiniMax H3" vLLM-Omni recipe, section "Step execution and continuous
  batching": each packed request is its own attention document, so each
  segment's clock restarts at zero.

Readings (the pages print no formula):
* video token (tau, h, w) of a T x Hg x Wg grid starting at clock t0 sits at
  (t0 + tau, h, w), row-major order;
* audio-tail token i of n spans the video grid's T frames: t = t0 + i*T/n,
  h = w = 0;
* an image reference is one Hg x Wg frame at t0 and advances the clock by 1;
* an audio reference of len tokens at rate r tokens per clock unit puts
  token i at t0 + i/r (h = w = 0) and advances the clock by len/r;
* order inside a segment: image refs, audio refs, video grid, audio tail.
* latent continuation ("MiniMax H3" vLLM-Omni recipe, section "Long video and
  driving audio": continuation chunks use global temporal RoPE positions): a
  segment may start its clock at an origin t_origin instead of 0; every
  position of the segment is then formed from t0 = t_origin.
Every value is formed in float64 with the operation order written here and
rounded once to float32.
"""

from __future__ import annotations

import numpy as np


def segment_positions(layout, t_origin: float = 0.0) -> np.ndarray:
    """Positions of one segment as float32 [L, 3] (t, h, w), its clock
    starting at ``t_origin``.

    ``layout`` has the attributes of ``synth.SegmentLayout``: video (T, Hg,
    Wg), audio_tail, image_refs, image_grid (ih, iw), audio_refs,
    audio_ref_len, audio_rate.
    """
    rows: list[tuple[float, float, float]] = []
    t0 = float(t_origin)
    ih, iw = layout.image_grid
    for _ in range(layout.image_refs):
        for h in range(ih):
            for w in range(iw):
                rows.append((t0, float(h), float(w)))
        t0 = t0 + 1.0
    for _ in range(layout.audio_refs):
        n, r = layout.audio_ref_len, layout.audio_rate
        for i in range(n):
            rows.append((t0 + float(i) / float(r), 0.0, 0.0))
        t0 = t0 + float(n) / float(r)
    T, Hg, Wg = layout.video
    for tau in range(T):
        for h in range(Hg):
            for w in range(Wg):
                rows.append((t0 + float(tau), float(h), float(w)))
    n = layout.audio_tail
    for i in range(n):
        rows.append((t0 + (float(i) * float(T)) / float(n), 0.0, 0.0))
    if not rows:
        return np.zeros((0, 3), dtype=np.float32)
    return np.asarray(rows, dtype=np.float64).astype(np.float32)


def packed_positions(layouts, t_origins=None) -> np.ndarray:
    """Positions of consecutive packed segments, float32 [N, 3]; segment s's
    clock starts at t_origins[s] (0 for all when None)."""
    origins = [0.0] * len(layouts) if t_origins is None else list(t_origins)
    parts = [segment_positions(l, o) for l, o in zip(layouts, origins)]
    if not parts:
        return np.zeros((0, 3), dtype=np.float32)
    return np.concatenate(parts, axis=0)
