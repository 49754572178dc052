"""Skip-softmax sparse attention, float64 (a lossy variant of the path).

Follows "MiniMax H3" vLLM-Omni recipe, section "Attention Backends": the
Skip-Softmax option skips attention tiles whose softmax contribution is
below a direct threshold (0.05 in the pages' example), keeping early
high-noise steps dense (that timestep gate is the caller's choice of dense
or sparse per call).

Reading (the pages give no formula): keys are processed per segment in tiles
of 128 starting at the segment start, in order; queries in blocks of 32 rows
inside 128-row tiles starting at the segment start. For a query block and a
key tile j > 0 let m_tile(r) be row r's largest score in the tile and m_run(r)
the largest score of row r over the tiles processed so far (skipped tiles
never raise it). The block skips the tile when, for every row of the block,
exp(m_tile(r) - m_run(r)) < threshold (scores include the softmax scale).
Skipped tiles contribute nothing; the first tile is never skipped. The
result is softmax attention over the keys of the tiles that were kept.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import _as_f64
from .rope import rope_ref


def attention_skip_ref(q, k, v, cu_seqlens, scale, threshold, pos=None, split=None,
                       theta=10000.0, pair_layout="interleaved", q_tile=128, row_block=32,
                       kv_tile=128):
    """Returns (O [N, H, D], LSE [H, N], skipped) with ``skipped`` the number of
    (row block, key tile) pairs that were skipped."""
    Q, K, V = _as_f64(q), _as_f64(k), _as_f64(v)
    if pos is not None:
        Q = rope_ref(Q, pos, split, theta, pair_layout)
        K = rope_ref(K, pos, split, theta, pair_layout)
    N, H, D = Q.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    O = np.zeros((N, H, D))
    LSE = np.zeros((H, N))
    log_thr = math.log(threshold) if threshold > 0 else -math.inf
    skipped = 0
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        L = e - a
        if L <= 0:
            continue
        n_kv = (L + kv_tile - 1) // kv_tile
        for h in range(H):
            S = scale * (Q[a:e, h] @ K[a:e, h].T)             # [L, L]
            keep = np.zeros((L, n_kv), dtype=bool)            # per row: tiles kept
            for r0 in range(0, L, row_block):
                # a row block never crosses a 128-row query tile (both start at a)
                rows = slice(r0, min(L, r0 + row_block))
                m_run = None
                for j in range(n_kv):
                    cols = slice(j * kv_tile, min(L, (j + 1) * kv_tile))
                    m_tile = S[rows, cols].max(axis=1)
                    if j > 0 and np.all(m_tile - m_run < log_thr):
                        skipped += 1
                        continue
                    keep[rows, j] = True
                    m_run = m_tile if m_run is None else np.maximum(m_run, m_tile)
            col_keep = np.repeat(keep, kv_tile, axis=1)[:, :L]
            Sm = np.where(col_keep, S, -np.inf)
            m = Sm.max(axis=1, keepdims=True)
            P = np.exp(Sm - m)
            l = P.sum(axis=1, keepdims=True)
            O[a:e, h] = (P @ V[a:e, h]) / l
            LSE[h, a:e] = (m + np.log(l))[:, 0]
    return O, LSE, skipped


def attention_skip_rows_ref(q, k, v, cu_seqlens, scale, threshold, rows, heads, pos=None,
                            split=None, theta=10000.0, pair_layout="interleaved",
                            row_block=32, kv_tile=128):
    """``attention_skip_ref`` for selected query rows and heads only: each
    row's whole 32-row block is evaluated (the decision is per block), so this
    runs at any sequence length. Returns (O [len(rows), len(heads), D],
    LSE [len(heads), len(rows)])."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    D = np.asarray(v).shape[2]
    O = np.zeros((len(rows), len(heads), D))
    LSE = np.zeros((len(heads), len(rows)))
    log_thr = math.log(threshold) if threshold > 0 else -math.inf
    seg_of = np.searchsorted(cu, rows, side="right") - 1
    for i, row in enumerate(rows):
        s = int(seg_of[i])
        a, e = int(cu[s]), int(cu[s + 1])
        L = e - a
        r0 = a + ((row - a) // row_block) * row_block
        blk = np.arange(r0, min(e, r0 + row_block))
        n_kv = (L + kv_tile - 1) // kv_tile
        for hi, h in enumerate(heads):
            Qb = _as_f64(np.asarray(q)[blk, h:h + 1])
            Ks = _as_f64(np.asarray(k)[a:e, h:h + 1])
            Vs = _as_f64(np.asarray(v)[a:e, h])
            if pos is not None:
                Qb = rope_ref(Qb, np.asarray(pos)[blk], split, theta, pair_layout)
                Ks = rope_ref(Ks, np.asarray(pos)[a:e], split, theta, pair_layout)
            S = scale * (Qb[:, 0] @ Ks[:, 0].T)
            keep = np.zeros(n_kv, dtype=bool)
            m_run = None
            for j in range(n_kv):
                m_tile = S[:, j * kv_tile:min(L, (j + 1) * kv_tile)].max(axis=1)
                if j > 0 and np.all(m_tile - m_run < log_thr):
                    continue
                keep[j] = True
                m_run = m_tile if m_run is None else np.maximum(m_run, m_tile)
            col_keep = np.repeat(keep, kv_tile)[:L]
            srow = np.where(col_keep, S[row - r0], -np.inf)
            m = srow.max()
            p_ = np.exp(srow - m)
            l_ = p_.sum()
            O[i, hi] = (p_ @ Vs) / l_
            LSE[hi, i] = m + np.log(l_)
    return O, LSE
