"""Workload descriptions and seeded bf16 draws.

The five workloads stand in for the joint video+audio sequences of the
MiniMax-H3 denoiser ("Day 0 Support for MiniMax-H3 on AMD Instinct GPUs",
section "The diffusion transformer (DiT)": video and audio latents flattened
into one token sequence; "MiniMax H3" vLLM-Omni recipe, section "Step
execution and continuous batching": co-batched requests packed into one
sequence with one attention document each). No public benchmark or dataset
exists for this path; every input is drawn here from a fixed seed.

Nothing in this module computes positions, rotations or attention.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Sequence

import numpy as np


@dataclass(frozen=True)
class SegmentLayout:
    """Token composition of one packed segment (one attention document).

    Order inside the segment: ``image_refs`` single-frame reference grids,
    then ``audio_refs`` audio-reference runs, then the ``video`` latent grid
    (T, Hg, Wg) in row-major (t, h, w) order, then ``audio_tail`` audio
    tokens that share the video grid's temporal span.
    ``audio_rate`` is the number of audio-reference tokens per unit of the
    temporal clock.
    """

    video: tuple[int, int, int]
    audio_tail: int = 0
    image_refs: int = 0
    image_grid: tuple[int, int] = (24, 42)
    audio_refs: int = 0
    audio_ref_len: int = 256
    audio_rate: int = 32

    def n_tokens(self) -> int:
        T, Hg, Wg = self.video
        ih, iw = self.image_grid
        return (self.image_refs * ih * iw + self.audio_refs * self.audio_ref_len
                + T * Hg * Wg + self.audio_tail)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    segments: tuple[SegmentLayout, ...]
    heads: int
    head_dim: int
    split: tuple[int, int, int]
    theta: float = 10000.0
    k_head_offset_std: float = 0.0
    description: str = ""
    seed: int = field(default=-1)

    @property
    def seg_lens(self) -> list[int]:
        return [s.n_tokens() for s in self.segments]

    @property
    def n_tokens(self) -> int:
        return int(sum(self.seg_lens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seg_lens))

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    @property
    def the_seed(self) -> int:
        return self.seed if self.seed >= 0 else 1000 + self.index

    def flops(self) -> float:
        """Algorithmic forward FLOPs: 4 * L^2 * H * D per segment (QK^T and PV)."""
        return float(sum(4.0 * L * L * self.heads * self.head_dim for L in self.seg_lens))


def _grid(T, H, W, tail=0, **kw):
    return SegmentLayout(video=(T, H, W), audio_tail=tail, **kw)


WORKLOADS: tuple[Workload, ...] = (
    Workload("tiny", 0,
             (_grid(4, 4, 4, 16), _grid(4, 4, 4, 16)),
             heads=2, head_dim=64, split=(16, 24, 24),
             description="2 packed segments of a 4x4x4 grid + 16 audio tokens"),
    Workload("single", 1,
             (_grid(8, 24, 42, 256),),
             heads=24, head_dim=128, split=(32, 48, 48),
             description="one clip: T8x24x42 grid + 256 audio tokens"),
    Workload("long", 2,
             (_grid(32, 24, 42, 1024),),
             heads=40, head_dim=128, split=(32, 48, 48), k_head_offset_std=0.5,
             description="one long clip: T32x24x42 grid + 1024 audio tokens, "
                         "k offset by a per-head constant"),
    Workload("packed", 3,
             (_grid(3, 24, 42, 1088, image_refs=1, audio_refs=0),
              _grid(8, 24, 42, 944, image_refs=3, audio_refs=1),
              _grid(13, 24, 42, 816, image_refs=6, audio_refs=2),
              _grid(22, 24, 42, 1008, image_refs=9, audio_refs=3)),
             heads=40, head_dim=128, split=(32, 48, 48),
             description="4 packed segments with image and audio references in front"),
    Workload("max", 4,
             (_grid(60, 24, 42, 1800), _grid(16, 24, 42, 0)),
             heads=48, head_dim=128, split=(32, 48, 48),
             description="T60x24x42 grid + 1800 audio tokens, plus a packed T16 grid"),
)


def workload(name_or_index) -> Workload:
    for w in WORKLOADS:
        if w.name == name_or_index or w.index == name_or_index:
            return w
    raise KeyError(name_or_index)


def cu_seqlens_of(seg_lens: Sequence[int]) -> np.ndarray:
    """Segment boundaries [0, L0, L0+L1, ...] as int32."""
    cu = np.zeros(len(seg_lens) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(seg_lens, dtype=np.int64))
    return cu.astype(np.int32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16. Inputs are finite draws.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def _normal_chunks(rng: np.random.Generator, shape, chunk_tokens: int = 1 << 14):
    """Yield (start, end, float32 standard normals) over token chunks.

    Drawing in fixed chunks bounds host memory at the largest sizes; the
    chunk size is part of the recipe, so the stream is reproducible.
    """
    N = shape[0]
    for s in range(0, N, chunk_tokens):
        e = min(N, s + chunk_tokens)
        yield s, e, rng.standard_normal((e - s,) + tuple(shape[1:]), dtype=np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    for s, e, x in _normal_chunks(rng, shape):
        out[s:e] = f32_to_bf16_bits(x)
    return out


def draw_qkv(w: Workload, seed: int | None = None):
    """q, k, v bf16 bit patterns [N, H, D] for workload ``w``.

    Recipe: ``numpy.random.default_rng(seed)`` with seed ``1000 + index``;
    q, then k, then v, each standard normal float32 drawn in chunks of 16384
    tokens and rounded to bf16 (round to nearest even). If the workload asks
    for a per-head key offset, one more standard normal per head, times
    ``k_head_offset_std``, is drawn after v and added in float32 to every
    element of that head's k before k is rounded to bf16.
    """
    seed = w.the_seed if seed is None else seed
    N, H, D = w.n_tokens, w.heads, w.head_dim
    rng = np.random.default_rng(seed)
    q = _normal_bf16(rng, (N, H, D))
    if w.k_head_offset_std > 0.0:
        k32 = np.empty((N, H, D), dtype=np.float32)
        for s, e, x in _normal_chunks(rng, (N, H, D)):
            k32[s:e] = x
        v = _normal_bf16(rng, (N, H, D))
        c = rng.standard_normal(H, dtype=np.float32) * np.float32(w.k_head_offset_std)
        k32 += c[None, :, None]
        k = f32_to_bf16_bits(k32)
        del k32
    else:
        k = _normal_bf16(rng, (N, H, D))
        v = _normal_bf16(rng, (N, H, D))
    return q, k, v


def draw_random_case(seg_lens: Sequence[int], heads: int, head_dim: int, seed: int,
                     pos_range: float = 64.0, std: float = 1.0):
    """A small random case for edge tests: q, k, v bf16 bits and fp32 positions.

    Positions are drawn uniformly in [0, pos_range) per token and axis and
    passed to both sides as inputs (they are data here, not computed).
    """
    N = int(sum(seg_lens))
    rng = np.random.default_rng(seed)
    q = f32_to_bf16_bits(rng.standard_normal((N, heads, head_dim), dtype=np.float32) * np.float32(std))
    k = f32_to_bf16_bits(rng.standard_normal((N, heads, head_dim), dtype=np.float32) * np.float32(std))
    v = f32_to_bf16_bits(rng.standard_normal((N, heads, head_dim), dtype=np.float32))
    pos = (rng.random((N, 3), dtype=np.float32) * np.float32(pos_range)).astype(np.float32)
    return q, k, v, pos, cu_seqlens_of(seg_lens)


def draw_group_case(seg_lens: Sequence[int], heads: int, head_dim: int, group_len: int,
                    amp: float, eps: float, seed: int):
    """Inputs with frame-group locality for the skip-softmax variant.

    Token i of a segment belongs to group g = i // group_len (counted from the
    segment start); its q and k are amp * e_(g mod head_dim) plus eps * N(0,1)
    noise per channel, v is N(0,1). Same-group scores are ~amp^2 and all others
    ~0, so a key tile either matters to a query or is clearly negligible.
    Recipe: default_rng(seed), noise for q, then k, then v, float32, rounded to
    bf16 (RNE). Returns q, k, v bits and cu_seqlens.
    """
    N = int(sum(seg_lens))
    rng = np.random.default_rng(seed)
    code = np.zeros((N, head_dim), dtype=np.float32)
    start = 0
    for L in seg_lens:
        g = (np.arange(L) // group_len) % head_dim
        code[start + np.arange(L), g] = np.float32(amp)
        start += L
    out = []
    for _ in range(2):
        x = rng.standard_normal((N, heads, head_dim), dtype=np.float32) * np.float32(eps)
        x += code[:, None, :]
        out.append(f32_to_bf16_bits(x))
    v = f32_to_bf16_bits(rng.standard_normal((N, heads, head_dim), dtype=np.float32))
    return out[0], out[1], v, cu_seqlens_of(seg_lens)


@dataclass(frozen=True)
class QkvProjection:
    """Shape of the DiT attention's input projection, the step that produces
    this path's q, k, v: hidden size 5376 and 56 heads of 128 ("Day 0 Support
    for MiniMax-H3 on AMD Instinct GPUs", section "The diffusion transformer
    (DiT)"), rotary split (32, 48, 48) as for the attention workloads."""

    hidden: int = 5376
    heads: int = 56
    head_dim: int = 128
    split: tuple = (32, 48, 48)
    theta: float = 10000.0

    @property
    def out_features(self) -> int:
        return 3 * self.heads * self.head_dim


QKV_PROJECTION = QkvProjection()


def draw_linear_case(n_rows: int, k: int, out_features: int, seed: int):
    """Activations and weights of one linear layer as bf16 bit patterns.

    Recipe: ``numpy.random.default_rng(seed)``; x [n_rows, k] standard normal
    float32 drawn in chunks of 16384 rows, then w [out_features, k] standard
    normal float32 times 1/sqrt(k) (so every output is ~N(0, 1)), each rounded
    to bf16 (round to nearest even).
    """
    rng = np.random.default_rng(seed)
    x = _normal_bf16(rng, (n_rows, k))
    w32 = rng.standard_normal((out_features, k), dtype=np.float32)
    w32 *= np.float32(1.0 / np.sqrt(k))
    return x, f32_to_bf16_bits(w32)
