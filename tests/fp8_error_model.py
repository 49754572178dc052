"""First-order error model of attention computed from e4m3-rounded Q, K, P
and V, used to bound the SAGE-style FP8 path against EXACT attention.

Nothing here depends on how an FP8 kernel tiles, schedules or scales its
work: only on the e4m3 format and on the exact float64 quantities of
softmax attention. Test infrastructure; it calls ``oracle.rope_ref`` and
``oracle.bf16_bits_to_f64`` and nothing else of the method.

Model. e4m3 keeps 3 mantissa bits, so rounding x to nearest on a scale s
(the value stored is x / s) changes it by at most 2^-4 |x| while x / s is a
normal number (|x| >= 2^-6 s) and by at most half the subnormal spacing,
2^-10 s, below that: |error| <= max(2^-4 |x|, 2^-10 s) = 2^-4 max(|x|, 2^-6 s).
The scale is only assumed to map the largest magnitude of its group into the
top two binades of the format, [112, 448], so s <= (group max) / 112; the
model uses the largest group each operand can have: the token's own row of
q, the whole segment's k (per head) and v (per head and channel), and the
row's largest softmax weight for p. Each of q_d, k_jd, p_j and v_jc is
rounded once; the roundings are treated as independent with zero mean and
variance at most b^2 / 3 for a bound b (a uniform error on [-b, b]); write
x'^2 = max(x^2, (2^-6 s)^2) and sigma2 = (2^-4)^2 / 3. To first order the
output O_c = sum_j w_j v_jc (w the exact softmax weights, sum 1) moves by

  Q:  scale * sum_d dq_d C_dc,   C = sum_j w_j k_j (v_j - O)^T
      (one rounding per query channel, shared by every key)
  K:  sum_j w_j (v_jc - O_c) * scale * sum_d q_d dk_jd
  P:  sum_j dw_j v_jc   (P rounded, the row sum kept exact)
  V:  sum_j w_j dv_jc

so its variance is at most
  sigma2 * [ scale^2 sum_d q'_d^2 C_dc^2
             + scale^2 sum_j w_j^2 (v_jc - O_c)^2 sum_d q_d^2 k'_jd^2
             + sum_j w'_j^2 v_jc^2 + sum_j w_j^2 v'_jc^2 ].
``sigma_rows`` returns the square root of that bound for each output
element, together with the exact output.
"""

from __future__ import annotations

import numpy as np

SIGMA2 = (2.0 ** -4) ** 2 / 3.0


def sigma_rows(q, k, v, cu, scale, rows, head, pos=None, split=None, theta=10000.0,
               parts=False):
    """Exact O [R, D] and the model's standard-deviation bound [R, D] for
    query rows ``rows`` (all in one segment) of head ``head``; with
    ``parts`` the bound of each rounding alone instead, as a dict with keys
    "q", "k", "p", "v"."""
    import oracle
    cu = np.asarray(cu, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    s = int(np.searchsorted(cu, rows[0], side="right") - 1)
    a, e = int(cu[s]), int(cu[s + 1])
    assert np.all((rows >= a) & (rows < e)), "rows of one segment"
    Q = oracle.bf16_bits_to_f64(np.asarray(q)[rows, head:head + 1])
    K = oracle.bf16_bits_to_f64(np.asarray(k)[a:e, head:head + 1])
    V = oracle.bf16_bits_to_f64(np.asarray(v)[a:e, head])
    if pos is not None:
        Q = oracle.rope_ref(Q, np.asarray(pos)[rows], split, theta)
        K = oracle.rope_ref(K, np.asarray(pos)[a:e], split, theta)
    Q, K = Q[:, 0], K[:, 0]
    S = scale * (Q @ K.T)
    W = np.exp(S - S.max(axis=1, keepdims=True))
    W /= W.sum(axis=1, keepdims=True)
    O = W @ V

    def floored_sq(x, group_max):
        return np.maximum(x * x, (2.0 ** -6 * group_max / 112.0) ** 2)

    Qf = floored_sq(Q, np.abs(Q).max(axis=1, keepdims=True))
    Kf = floored_sq(K, np.abs(K).max())
    Vf = floored_sq(V, np.abs(V).max(axis=0, keepdims=True))
    Wf = floored_sq(W, W.max(axis=1, keepdims=True))
    W2 = W * W
    V2 = V * V
    # K term: t_j = sum_d q_d^2 k'_jd^2
    T = (Q * Q) @ Kf.T
    WT = W2 * T
    var_k = scale * scale * (WT @ V2 - 2.0 * O * (WT @ V) + O * O * WT.sum(axis=1)[:, None])
    var_p = Wf @ V2
    var_v = W2 @ Vf
    var_q = np.empty_like(O)
    for r in range(len(rows)):
        C = (K * W[r][:, None]).T @ V - np.outer(K.T @ W[r], O[r])
        var_q[r] = scale * scale * (Qf[r] @ (C * C))
    var_k = np.maximum(var_k, 0.0)
    if parts:
        return O, {"q": np.sqrt(SIGMA2 * var_q), "k": np.sqrt(SIGMA2 * var_k),
                   "p": np.sqrt(SIGMA2 * var_p), "v": np.sqrt(SIGMA2 * var_v)}
    return O, np.sqrt(SIGMA2 * (var_q + var_k + var_p + var_v))
