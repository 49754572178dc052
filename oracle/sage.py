"""SAGE-style FP8 attention (a lossy variant of the path), float64 with the
quantisation decisions taken in float32.

"MiniMax H3" vLLM-Omni recipe, section "Attention Backends": the TRTLLM
backend's SAGE quantisation runs Q and K in fp8_e4m3 with q_block_size 1 and
k_block_size 16, and P and V are always FP8 in that kernel. The pages give no
formulas; the reading used here (R18):

  * e4m3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
    largest finite 448, subnormals m/8 * 2^-6; conversion rounds to nearest
    (ties to even) and saturates to +-448.
  * Q~ = RoPE(q), K~ = RoPE(k) (oracle.rope) in float32.
  * Q: one scale per (token, head): a = max_d |Q~|, s_q = a / 448,
    code = e4m3(Q~ * (448 / a)) (float32 division and product; a = 0 gives
    s_q = 0 and zero codes).
  * K: one scale per (16-key block, head); blocks start at the segment start
    (a block never straddles two segments); same formulas over the block.
  * V: one scale per (segment, head, channel) over the segment's tokens.
  * Scores: x = (q8 . k8) * s_q * s_k * scale * log2(e) (log2 domain).
  * Online softmax over key tiles of 128 from the segment start, in order,
    with a lazily updated reference max m (log2 domain): the first tile sets
    m to its max; a later tile raises m to the running max only when its own
    max exceeds m by more than tau = 2 (the accumulator and the row sum are
    then rescaled by 2^(m_old - m_new)). Hence 2^(x - m) <= 2^tau and
    P8 = e4m3(448 * 2^-tau * 2^(x - m)) = e4m3(112 * 2^(x - m)) <= 448; the
    row sum l adds the unquantised 112 * 2^(x - m). tau = 0 is the eager
    update (every rise of the max rescales).
  * O = s_v * (sum_j P8_j v8_j) / l, LSE = ln(sum_j e^(scale q~.k~)) from the
    same quantities: (m + log2(l / 112)) * ln 2.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import _as_f64
from .rope import rope_ref

E4M3_MAX = 448.0
LAZY_LOG2 = 2.0
_LOG2E = 1.0 / math.log(2.0)


# ------------------------------------------------------------------ e4m3 codec

def e4m3_decode(codes) -> np.ndarray:
    """uint8 codes -> float64 values (0x7F / 0xFF decode to NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_round(x) -> np.ndarray:
    """Nearest e4m3 value (ties to even), saturated to +-448; float64 in, out."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # exponent of the binade: a in [2^e, 2^(e+1)); below 2^-6 the quantum is 2^-9
    _, fe = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(fe - 1, -6)
    quantum = np.ldexp(1.0, e - 3)
    r = np.round(a / quantum) * quantum          # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x) -> np.ndarray:
    """float values -> uint8 codes of e4m3_round(x) (-0 encodes as 0x80)."""
    r = e4m3_round(x)
    a = np.abs(r)
    _, fe = np.frexp(np.where(a > 0, a, 1.0))
    e = fe - 1
    normal = a >= 2.0 ** -6
    ebits = np.where(normal, e + 7, 0)
    mbits = np.where(normal, np.round((a / np.ldexp(1.0, e) - 1.0) * 8.0),
                     np.round(a / 2.0 ** -9))
    code = (ebits.astype(np.int64) << 3) | mbits.astype(np.int64)
    code = np.where(a == 0, 0, code)
    code = code | np.where(np.signbit(r), 0x80, 0)
    return code.astype(np.uint8)


# ---------------------------------------------------------------- quantisation

def _quant_rows(X32: np.ndarray):
    """X32 float32 [..., n]: one scale over the last axis. Returns (codes as
    float64 e4m3 values, dequant scale float32)."""
    amax = np.max(np.abs(X32), axis=-1).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0)).astype(np.float32)
    y = (X32 * inv[..., None]).astype(np.float32)
    codes = e4m3_round(y)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return codes, scale


def sage_quantize(q, k, v, cu_seqlens, pos=None, split=None, theta=10000.0,
                  pair_layout="interleaved", k_block=16):
    """Returns dict with q8, k8, v8 (float64 e4m3 values [N, H, D]), s_q [H, N],
    s_k [H, N] (each token carries its block's scale), s_v [nseg, H, D]
    (float32 dequantisation scales)."""
    Q, K, V = _as_f64(q), _as_f64(k), _as_f64(v)
    if pos is not None:
        Q = rope_ref(Q, pos, split, theta, pair_layout)
        K = rope_ref(K, pos, split, theta, pair_layout)
    Q32, K32, V32 = Q.astype(np.float32), K.astype(np.float32), V.astype(np.float32)
    N, H, D = Q.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nseg = len(cu) - 1
    q8, sq = _quant_rows(Q32)                                    # [N, H, D], [N, H]
    k8 = np.zeros((N, H, D))
    sk = np.zeros((N, H), dtype=np.float32)
    v8 = np.zeros((N, H, D))
    sv = np.zeros((nseg, H, D), dtype=np.float32)
    for s in range(nseg):
        a, e = int(cu[s]), int(cu[s + 1])
        for b0 in range(a, e, k_block):
            b1 = min(e, b0 + k_block)
            blk = K32[b0:b1].transpose(1, 0, 2).reshape(H, -1)   # [H, n*D]
            codes, scale = _quant_rows(blk)
            k8[b0:b1] = codes.reshape(H, b1 - b0, D).transpose(1, 0, 2)
            sk[b0:b1] = scale[None, :]
        if e > a:
            Vs = V32[a:e].transpose(1, 2, 0)                     # [H, D, L]
            codes, scale = _quant_rows(Vs)
            v8[a:e] = codes.transpose(2, 0, 1)
            sv[s] = scale
    return {"q8": q8, "s_q": sq.T.copy(), "k8": k8, "s_k": sk.T.copy(), "v8": v8, "s_v": sv}


# ------------------------------------------------------------------- attention

def p_scale(tau: float) -> float:
    """The P8 scale 448 * 2^-tau of the module docstring."""
    return E4M3_MAX * 2.0 ** -tau


def _online_rows(xs, v8, kv_tile, tau):
    """xs [R, L] scores (log2 domain), v8 [L, D] codes -> (acc [R, D], l [R], m [R])
    following the online algorithm of the module docstring."""
    R, L = xs.shape
    acc = np.zeros((R, v8.shape[1]))
    l = np.zeros(R)
    m = np.full(R, -np.inf)
    ps = p_scale(tau)
    for j0 in range(0, L, kv_tile):
        x = xs[:, j0:j0 + kv_tile]
        tmax = x.max(axis=1)
        first = ~np.isfinite(m)
        raise_ = first | (tmax > m + tau)
        m_new = np.where(first, tmax, np.where(raise_, np.maximum(m, tmax), m))
        f = np.where(first, 0.0, np.exp2(np.where(first, 0.0, m - m_new)))
        acc *= f[:, None]
        l *= f
        m = m_new
        p = ps * np.exp2(x - m[:, None])
        acc += e4m3_round(p) @ v8[j0:j0 + kv_tile]
        l += p.sum(axis=1)
    return acc, l, m


def sage_attention_ref(q, k, v, cu_seqlens, scale, pos=None, split=None, theta=10000.0,
                       pair_layout="interleaved", kv_tile=128, quant=None, tau=LAZY_LOG2):
    """Returns (O [N, H, D], LSE [H, N]) of the SAGE reading; ``quant`` may pass
    a precomputed ``sage_quantize`` result."""
    qz = quant if quant is not None else sage_quantize(q, k, v, cu_seqlens, pos, split, theta,
                                                         pair_layout)
    q8, k8, v8 = qz["q8"], qz["k8"], qz["v8"]
    sq, sk, sv = qz["s_q"].astype(np.float64), qz["s_k"].astype(np.float64), qz["s_v"]
    N, H, D = q8.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    O = np.zeros((N, H, D))
    LSE = np.zeros((H, N))
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        if e <= a:
            continue
        for h in range(H):
            raw = q8[a:e, h] @ k8[a:e, h].T                    # exact (e4m3 products)
            xs = raw * sq[h, a:e, None] * sk[h, None, a:e] * (scale * _LOG2E)
            acc, l, m = _online_rows(xs, v8[a:e, h], kv_tile, tau)
            O[a:e, h] = acc * sv[s, h][None, :].astype(np.float64) / l[:, None]
            LSE[h, a:e] = (m + np.log2(l / p_scale(tau))) * math.log(2.0)
    return O, LSE


def sage_attention_rows_ref(q, k, v, cu_seqlens, scale, rows, heads, pos=None, split=None,
                            theta=10000.0, pair_layout="interleaved", kv_tile=128,
                            k_block=16, tau=LAZY_LOG2):
    """``sage_attention_ref`` for selected query rows and heads (any size):
    quantises only the rows' own Q and their segments' K and V for those heads."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    D = np.asarray(v).shape[2]
    O = np.zeros((len(rows), len(heads), D))
    LSE = np.zeros((len(heads), len(rows)))
    seg_of = np.searchsorted(cu, rows, side="right") - 1
    for s in np.unique(seg_of):
        a, e = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(seg_of == s)[0]
        r = rows[sel]
        for hi, h in enumerate(heads):
            hs = slice(h, h + 1)
            P = None if pos is None else np.asarray(pos)[a:e]
            qz = sage_quantize(np.asarray(q)[a:e, hs], np.asarray(k)[a:e, hs],
                               np.asarray(v)[a:e, hs], np.array([0, e - a]), P, split, theta,
                               pair_layout, k_block)
            q8, k8, v8 = qz["q8"][r - a, 0], qz["k8"][:, 0], qz["v8"][:, 0]
            sq = qz["s_q"][0, r - a].astype(np.float64)
            sk = qz["s_k"][0].astype(np.float64)
            xs = (q8 @ k8.T) * sq[:, None] * sk[None, :] * (scale * _LOG2E)
            acc, l, m = _online_rows(xs, v8, kv_tile, tau)
            O[sel, hi] = acc * qz["s_v"][0, 0][None, :].astype(np.float64) / l[:, None]
            LSE[hi, sel] = (m + np.log2(l / p_scale(tau))) * math.log(2.0)
    return O, LSE
