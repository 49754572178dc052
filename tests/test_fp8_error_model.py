"""Pins of the first-order FP8 error model (tests/fp8_error_model.py) that
bounds the SAGE-style FP8 path against exact attention.

1. Against real rounding: Q, K, P and V are rounded to e4m3 (the oracle's
   codec, itself pinned code by code in test_oracle_sage.py) after a random
   rescaling per trial (a factor in one octave, undone after rounding), so
   that the rounding errors behave like independent draws; the output
   errors, each divided by the model's bound for its element, must have an
   RMS below 1 and not far below it (the bound assumes the largest variance
   an error of at most 2^-4 can have; e4m3's actual relative errors are
   smaller, about 0.7 of it in standard deviation), and none beyond 6.
2. The SAGE reading (oracle/sage.py, per-token / per-16-key / per-channel
   scales, lazily raised reference max) stays inside the model's bound
   against exact attention on the path's own input distribution.
"""

import math

import numpy as np

import oracle
import synth
from fp8_error_model import sigma_rows


def _rounded_attention(Q, K, V, scale, rng, which="qkpv"):
    """Attention with the operands named in ``which`` (of Q, K, P, V)
    rounded to e4m3 once each, after random rescalings (undone exactly
    afterwards); the row sum of P stays exact."""
    # each operand's largest magnitude lands at a random place in [112, 448)
    u = 2.0 ** rng.uniform(0.0, 2.0, size=4)
    rnd = {c: (lambda x, f: oracle.e4m3_round(x * f) / f) if c in which else (lambda x, f: x)
           for c in "qkpv"}
    Qr = rnd["q"](Q, u[0] * 112.0 / np.abs(Q).max())
    Kr = rnd["k"](K, u[1] * 112.0 / np.abs(K).max())
    Vr = rnd["v"](V, u[3] * 112.0 / np.abs(V).max())
    S = scale * (Qr @ Kr.T)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    l = P.sum(axis=1, keepdims=True)
    Pr = rnd["p"](P, u[2] * 112.0)   # the row maximum of P is 1
    return (Pr @ Vr) / l


def test_model_bounds_the_spread_of_real_e4m3_rounding():
    q, k, v, pos, cu = synth.draw_random_case([400], 1, 128, seed=501, pos_range=64.0)
    scale = 1.0 / math.sqrt(128)
    rows = np.arange(0, 400, 50)
    O, sig = sigma_rows(q, k, v, cu, scale, rows, 0)
    Q = oracle.bf16_bits_to_f64(q[rows, 0])
    K = oracle.bf16_bits_to_f64(k[:, 0])
    V = oracle.bf16_bits_to_f64(v[:, 0])
    _, part = sigma_rows(q, k, v, cu, scale, rows, 0, parts=True)
    rng = np.random.default_rng(502)
    # each rounding alone against its own term, then all four together
    for which, s in [("q", part["q"]), ("k", part["k"]), ("p", part["p"]), ("v", part["v"]),
                     ("qkpv", sig)]:
        z = np.stack([(_rounded_attention(Q, K, V, scale, rng, which) - O) / s
                      for _ in range(60)])
        # normalised errors over elements and trials: spread below the bound,
        # and not far below it (a term dropped from the total, or a wrong
        # factor in one, leaves this window); no outlier beyond the 6-sigma
        # the GPU tests use
        rms = float(np.sqrt((z ** 2).mean()))
        assert 0.6 < rms < 0.8, (which, rms)
        assert np.abs(z).max() <= 6.0, (which, np.abs(z).max())


def test_model_bounds_the_sage_reading_against_exact_attention():
    seg = [700, 333]
    q, k, v, pos, cu = synth.draw_random_case(seg, 2, 128, seed=503, pos_range=64.0)
    scale = 1.0 / math.sqrt(128)
    split = (32, 48, 48)
    Os, _ = oracle.sage_attention_ref(q, k, v, cu, scale, pos, split)
    zs, errs, sigs = [], [], []
    for h in range(2):
        for s in range(2):
            rows = np.arange(int(cu[s]), int(cu[s + 1]))
            O, sig = sigma_rows(q, k, v, cu, scale, rows, h, pos, split)
            e = np.abs(Os[rows, h] - O)
            zs.append(e / (sig + 2.0 ** -9 * np.abs(O)))
            errs.append(e.ravel())
            sigs.append(sig.ravel())
    z = np.concatenate([x.ravel() for x in zs])
    assert z.max() <= 6.0, z.max()
    assert np.concatenate(errs).mean() <= np.concatenate(sigs).mean()


def test_model_reduces_to_closed_forms():
    # one key: the softmax weight is exactly 1 and O = v; the Q and K terms
    # vanish (v - O = 0), the P term is SIGMA2 v^2 and the V term SIGMA2
    # max(v^2, (2^-6 max|v| / 112)^2)
    from fp8_error_model import SIGMA2
    q, k, v, _, cu = synth.draw_random_case([1], 1, 64, seed=504)
    O, sig = sigma_rows(q, k, v, cu, 0.3, [0], 0)
    V = oracle.bf16_bits_to_f64(v[:, 0])
    np.testing.assert_allclose(O, V, rtol=0, atol=1e-15)
    floor = (2.0 ** -6 * np.abs(V).max(axis=0) / 112.0) ** 2
    np.testing.assert_allclose(sig ** 2, SIGMA2 * (V ** 2 + np.maximum(V ** 2, floor)),
                               rtol=1e-12, atol=0)
    # identical keys: the weights are uniform whatever the scores, the K and
    # Q terms vanish with the key-independent scores (v_j - O averages to
    # zero against identical k_j), and the P and V terms are 2 SIGMA2 sum v^2 / L^2
    q, k, v, _, cu = synth.draw_random_case([50], 1, 64, seed=505)
    k = np.repeat(k[:1], 50, axis=0)
    O, sig = sigma_rows(q, k, v, cu, 0.2, [3], 0)
    V = oracle.bf16_bits_to_f64(v[:, 0])
    np.testing.assert_allclose(O[0], V.mean(0), rtol=0, atol=1e-14)
    vf = np.maximum(V ** 2, (2.0 ** -6 * np.abs(V).max(axis=0) / 112.0) ** 2)
    want_pv = SIGMA2 * ((V ** 2).sum(0) + vf.sum(0)) / 50 ** 2
    K = oracle.bf16_bits_to_f64(k[:, 0])
    Q = oracle.bf16_bits_to_f64(q[3:4, 0])
    kf = np.maximum(K[0] ** 2, (2.0 ** -6 * np.abs(K).max() / 112.0) ** 2)
    t = (Q[0] ** 2) @ kf
    want_k = SIGMA2 * 0.2 ** 2 * t * ((V - V.mean(0)) ** 2).sum(0) / 50 ** 2
    np.testing.assert_allclose(sig[0] ** 2, want_pv + want_k, rtol=1e-9, atol=1e-30)
