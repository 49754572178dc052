"""Packed variable-length joint self-attention, float64.

Follows:
* "Day 0 Support for MiniMax-H3 on AMD Instinct GPUs", section "The
  diffusion transformer (DiT)": video and audio latents form one token
  sequence that is attended jointly (non-causal);
* "MiniMax H3" vLLM-Omni recipe, section "Step execution and continuous
  batching": co-batched requests are packed into one sequence that keeps one
  attention document per request, i.e. a block-diagonal mask given by the
  segment boundaries cu_seqlens;
* the same recipe, section "Attention Backends", and "MiniMax H3 on Moore
  Threads MUSA", section "MUSA validation": the backends are packed
  variable-length attention.

Definition, per segment s = [cu[s], cu[s+1]) and head h, with q and k
rotated by RoPE (``oracle.rope``) when positions are given:
    S = scale * Q K^T,  P = softmax_row(S),  O = P V,
    LSE = max_row(S) + log(sum_row(exp(S - max_row(S)))).
The softmax subtracts the row maximum (a rearrangement that leaves the
result unchanged). Query rows are processed in blocks of ``block`` rows so
that no L x L matrix is held; each block is the plain formula above.
"""

from __future__ import annotations

import numpy as np

from .bf16 import bf16_bits_to_f64
from .rope import rope_ref


def _as_f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


def _softmax_attention_rows(Qs, Ks, Vs, scale, block=256):
    """Qs [Lq, D], Ks and Vs [L, D] -> O [Lq, D], LSE [Lq] (float64)."""
    Lq = Qs.shape[0]
    O = np.empty((Lq, Vs.shape[1]), dtype=np.float64)
    lse = np.empty(Lq, dtype=np.float64)
    for b in range(0, Lq, block):
        S = scale * (Qs[b:b + block] @ Ks.T)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        O[b:b + block] = (P @ Vs) / l
        lse[b:b + block] = (m + np.log(l))[:, 0]
    return O, lse


def attention_ref(q, k, v, cu_seqlens, scale, pos=None, split=None, theta=10000.0,
                  pair_layout="interleaved", block=256):
    """Full oracle. q, k, v: [N, H, D] as bf16 bit patterns (uint16) or floats.

    Returns (O [N, H, D] float64, LSE [H, N] float64).
    """
    Q, K, V = _as_f64(q), _as_f64(k), _as_f64(v)
    if pos is not None:
        Q = rope_ref(Q, pos, split, theta, pair_layout)
        K = rope_ref(K, pos, split, theta, pair_layout)
    N, H, D = Q.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    O = np.zeros((N, H, D), dtype=np.float64)
    LSE = np.zeros((H, N), dtype=np.float64)
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        if e <= a:
            continue
        for h in range(H):
            o, l = _softmax_attention_rows(Q[a:e, h], K[a:e, h], V[a:e, h], scale, block)
            O[a:e, h] = o
            LSE[h, a:e] = l
    return O, LSE


def attention_rows_ref(q, k, v, cu_seqlens, scale, rows, heads, pos=None, split=None,
                       theta=10000.0, pair_layout="interleaved", block=256):
    """Oracle outputs for selected query rows and heads only.

    ``rows``: global token indices; ``heads``: head indices. Returns
    (O [len(rows), len(heads), D], LSE [len(heads), len(rows)]) in float64.
    Only the slices of the segments that hold the rows are widened and
    rotated, so this runs at any N.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    heads = list(int(h) for h in heads)
    D = np.asarray(v).shape[2]
    O = np.zeros((len(rows), len(heads), D), dtype=np.float64)
    LSE = np.zeros((len(heads), len(rows)), dtype=np.float64)
    seg_of = np.searchsorted(cu, rows, side="right") - 1
    for s in np.unique(seg_of):
        a, e = int(cu[s]), int(cu[s + 1])
        sel = np.nonzero(seg_of == s)[0]
        r = rows[sel]
        for hi, h in enumerate(heads):
            Qs = _as_f64(np.asarray(q)[r, h:h + 1])
            Ks = _as_f64(np.asarray(k)[a:e, h:h + 1])
            Vs = _as_f64(np.asarray(v)[a:e, h])
            if pos is not None:
                Qs = rope_ref(Qs, np.asarray(pos)[r], split, theta, pair_layout)
                Ks = rope_ref(Ks, np.asarray(pos)[a:e], split, theta, pair_layout)
            o, l = _softmax_attention_rows(Qs[:, 0], Ks[:, 0], Vs, scale, block)
            O[sel, hi] = o
            LSE[hi, sel] = l
    return O, LSE


def attention_dense_bruteforce(q, k, v, cu_seqlens, scale, pos=None, split=None,
                               theta=10000.0, pair_layout="interleaved"):
    """Independent check for tiny inputs: one N x N score matrix per head with
    an explicit block-diagonal mask (-inf outside the segment), softmax over
    the whole packed row, computed with plain Python loops over scalars."""
    import math
    Q, K, V = _as_f64(q), _as_f64(k), _as_f64(v)
    if pos is not None:
        Q = rope_ref(Q, pos, split, theta, pair_layout)
        K = rope_ref(K, pos, split, theta, pair_layout)
    N, H, D = Q.shape
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    seg = [0] * N
    for s in range(len(cu) - 1):
        for n in range(cu[s], cu[s + 1]):
            seg[n] = s
    O = np.zeros((N, H, D), dtype=np.float64)
    LSE = np.zeros((H, N), dtype=np.float64)
    for h in range(H):
        for i in range(N):
            scores = []
            for j in range(N):
                if seg[j] != seg[i]:
                    scores.append(-math.inf)
                    continue
                scores.append(scale * math.fsum(Q[i, h, d] * K[j, h, d] for d in range(D)))
            mx = max(scores)
            w = [math.exp(s - mx) if s != -math.inf else 0.0 for s in scores]
            tot = math.fsum(w)
            for d in range(D):
                O[i, h, d] = math.fsum(w[j] * V[j, h, d] for j in range(N)) / tot
            LSE[h, i] = mx + math.log(tot)
    return O, LSE
