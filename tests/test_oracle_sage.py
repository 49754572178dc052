"""Pins of the SAGE-style FP8 attention oracle (oracle/sage.py) against what the
e4m3 format definition and the mathematics fix: code values, round-to-nearest-
even midpoints, saturation, the quantisation invariants, closed forms for
lossless inputs, the direct (one-pass) definition where the running max never
moves, and a bounded distance to exact attention."""

import math

import numpy as np
import pytest

import oracle
import synth
from oracle.sage import e4m3_decode, e4m3_encode, e4m3_round


def test_e4m3_code_values_from_the_format_definition():
    d = e4m3_decode(np.arange(256, dtype=np.uint8))
    assert d[0x00] == 0.0 and d[0x38] == 1.0 and d[0x40] == 2.0 and d[0x30] == 0.5
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0
    assert d[0x08] == 2.0 ** -6 and d[0x01] == 2.0 ** -9 and d[0x07] == 7 * 2.0 ** -9
    assert d[0x39] == 1.125 and d[0x3F] == 1.875
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    pos = d[:0x7F]
    assert np.all(np.diff(pos) > 0)                  # codes 0..0x7E increase strictly
    assert np.array_equal(d[0x80:0xFF], -pos[:])     # sign bit


def test_e4m3_round_trip_and_midpoints():
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = e4m3_decode(codes)
    assert np.array_equal(e4m3_round(vals), vals)
    assert np.array_equal(e4m3_encode(vals), codes)
    assert np.array_equal(e4m3_encode(-vals[1:]), codes[1:] | 0x80)
    # a midpoint between neighbours goes to the even code (mantissa LSB 0)
    mid = (vals[:-1] + vals[1:]) / 2
    got = e4m3_encode(mid)
    even = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    assert np.array_equal(got, even)
    # just off the midpoint goes to the nearer neighbour
    eps = (vals[1:] - vals[:-1]) * 1e-3
    assert np.array_equal(e4m3_encode(mid - eps), codes[:-1])
    assert np.array_equal(e4m3_encode(mid + eps), codes[1:])


def test_e4m3_saturates():
    assert e4m3_round(np.array([449.0, 464.0, 1e6, -1e9])).tolist() == [448, 448, 448, -448]
    assert e4m3_round(np.array([2.0 ** -11, 2.0 ** -10 * 1.01])).tolist() == [0.0, 2.0 ** -9]


def test_quantisation_invariants():
    q, k, v, pos, cu = synth.draw_random_case([70, 33, 16], 2, 128, seed=301)
    z = oracle.sage_quantize(q, k, v, cu, pos, (32, 48, 48))
    q8, k8, v8 = z["q8"], z["k8"], z["v8"]
    # every scale group reaches +-448 exactly and all codes are e4m3 values
    assert np.all(np.max(np.abs(q8), axis=2) == 448.0)
    for t in (q8, k8, v8):
        assert np.array_equal(e4m3_round(t), t)
    # dequantisation error within half a quantum (relative 2^-4 for normals)
    Qr = oracle.rope_ref(oracle.bf16_bits_to_f64(q), pos, (32, 48, 48), 1e4)
    deq = q8 * z["s_q"].T[:, :, None]
    amax = np.max(np.abs(Qr), axis=2, keepdims=True)
    assert np.all(np.abs(deq - Qr) <= 2.0 ** -4 * np.abs(Qr) + 2.0 ** -10 * amax / 448 * 8)
    # K: one scale per block of 16 from the segment start; a block never straddles
    sk = z["s_k"]
    starts = []
    for s in range(len(cu) - 1):
        starts += list(range(int(cu[s]), int(cu[s + 1]), 16))
    for b0 in starts:
        b1 = min([x for x in list(cu[1:]) + starts if x > b0])
        assert np.all(sk[:, b0:b1] == sk[:, b0:b0 + 1])
        assert np.all(np.max(np.abs(k8[b0:b1]), axis=(0, 2)) == 448.0)
    # V: per (segment, head, channel)
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        assert np.all(np.max(np.abs(v8[a:e]), axis=0) == 448.0)


def test_lossless_inputs_uniform_scores_give_the_segment_mean():
    # entries in {0, +-c} with c = 448 * 2^-n: every quantisation and every
    # dequantisation scale is exact; with scale 0 every P8 is exactly 112, so
    # O is the exact segment mean of V
    rng = np.random.default_rng(302)
    seg = [37, 200, 1]
    N, H, D = sum(seg), 2, 64
    def lossless(c):
        x = rng.choice([-1.0, 0.0, 1.0], size=(N, H, D)) * c
        x[:, :, 0] = c                                   # every group has amax c
        return synth.f32_to_bf16_bits(x.astype(np.float32))
    q, k, v = lossless(0.875), lossless(3.5), lossless(1.75)
    cu = synth.cu_seqlens_of(seg)
    O, LSE = oracle.sage_attention_ref(q, k, v, cu, 0.0)
    V = oracle.bf16_bits_to_f64(v)
    for s in range(len(seg)):
        a, e = int(cu[s]), int(cu[s + 1])
        np.testing.assert_allclose(O[a:e], np.broadcast_to(V[a:e].mean(axis=0), O[a:e].shape),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSE[:, a:e], math.log(e - a), rtol=0, atol=1e-12)


def _direct(qz, a, e, h, scale, tau, m=None):
    """One-pass definition with a fixed reference max m per row (the true row
    max unless given): equal to the online result whenever the reference max
    never moves after the first tile."""
    q8, k8, v8 = qz["q8"][a:e, h], qz["k8"][a:e, h], qz["v8"][a:e, h]
    x = (q8 @ k8.T) * qz["s_q"][h, a:e, None].astype(np.float64) \
        * qz["s_k"][h, None, a:e].astype(np.float64) * scale / math.log(2.0)
    if m is None:
        m = x.max(axis=1)
    p = oracle.sage.p_scale(tau) * np.exp2(x - m[:, None])
    return (e4m3_round(p) @ v8) * qz["s_v"][0, h].astype(np.float64) / p.sum(axis=1, keepdims=True)


def _case(L, seed, big_key=None, big=8.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, 1, 64)).astype(np.float32) * 0.3
    q[:, :, 0] = 3.0
    k = rng.standard_normal((L, 1, 64)).astype(np.float32) * 0.3
    if big_key is not None:
        k[big_key, 0, :] = 0.0
        k[big_key, 0, 0] = big
    v = rng.standard_normal((L, 1, 64)).astype(np.float32)
    return tuple(synth.f32_to_bf16_bits(t) for t in (q, k, v))


@pytest.mark.parametrize("tau", [0.0, 2.0])
def test_online_equals_direct_definition_when_the_max_never_moves(tau):
    # key 0 aligns with every query, so the first tile holds each row's max
    L = 400
    qb, kb, vb = _case(L, 303, big_key=0)
    cu = np.array([0, L], dtype=np.int32)
    qz = oracle.sage_quantize(qb, kb, vb, cu)
    O, _ = oracle.sage_attention_ref(qb, kb, vb, cu, 0.125, quant=qz, tau=tau)
    np.testing.assert_allclose(O[:, 0], _direct(qz, 0, L, 0, 0.125, tau), rtol=0, atol=1e-12)
    # and one tile only: always the direct definition
    qz1 = oracle.sage_quantize(qb[:100], kb[:100], vb[:100], np.array([0, 100]))
    O1, _ = oracle.sage_attention_ref(qb[:100], kb[:100], vb[:100], np.array([0, 100]), 0.2,
                                      quant=qz1, tau=tau)
    np.testing.assert_allclose(O1[:, 0], _direct(qz1, 0, 100, 0, 0.2, tau), rtol=0, atol=1e-12)


def test_a_rise_below_the_threshold_keeps_the_reference_max():
    # the key of tile 2 scores about 1 (log2 units) above tile 0's max for
    # every row: with tau = 2 the reference stays tile 0's max (P up to 224),
    # which is the direct definition with m = tile 0's max
    L = 300
    qb, kb, vb = _case(L, 304, big_key=0, big=8.0)
    k = oracle.bf16_bits_to_f64(kb).astype(np.float32)
    k[290, 0, :] = 0.0
    k[290, 0, 0] = 8.0 + 1.0 / (3.0 * 0.125 / math.log(2.0))   # +1 in log2 units
    kb = synth.f32_to_bf16_bits(k)
    cu = np.array([0, L], dtype=np.int32)
    qz = oracle.sage_quantize(qb, kb, vb, cu)
    x = (qz["q8"][:, 0] @ qz["k8"][:, 0].T) * qz["s_q"][0][:, None] * qz["s_k"][0][None, :] \
        * 0.125 / math.log(2.0)
    m0 = x[:, :128].max(axis=1)
    rise = x.max(axis=1) - m0
    assert np.all((rise > 0.5) & (rise < 1.5))
    O, _ = oracle.sage_attention_ref(qb, kb, vb, cu, 0.125, quant=qz, tau=2.0)
    np.testing.assert_allclose(O[:, 0], _direct(qz, 0, L, 0, 0.125, 2.0, m=m0), rtol=0, atol=1e-12)
    # with the eager update the reference moves and the result differs
    O0, _ = oracle.sage_attention_ref(qb, kb, vb, cu, 0.125, quant=qz, tau=0.0)
    assert not np.allclose(O0[:, 0], O[:, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(O0[:, 0], _direct(qz, 0, L, 0, 0.125, 0.0), rtol=0, atol=0.05)


def test_online_rescaling_matters():
    # a late key scoring about 5 (log2 units) above the earlier tiles: the
    # reference max moves; the result differs from the direct one only by P8
    # rounding on the earlier tiles' grid
    L = 300
    qb, kb, vb = _case(L, 305, big_key=290, big=10.0)
    cu = np.array([0, L], dtype=np.int32)
    qz = oracle.sage_quantize(qb, kb, vb, cu)
    for tau in (0.0, 2.0):
        O, _ = oracle.sage_attention_ref(qb, kb, vb, cu, 0.125, quant=qz, tau=tau)
        Od = _direct(qz, 0, L, 0, 0.125, tau)
        assert not np.allclose(O[:, 0], Od, rtol=0, atol=1e-12)
        assert np.abs(O[:, 0] - Od).max() < 0.05


def test_single_token_segments_return_dequantised_v():
    q, k, v, pos, cu = synth.draw_random_case([1, 1, 1], 2, 64, seed=305)
    O, _ = oracle.sage_attention_ref(q, k, v, cu, 0.125, pos, (16, 24, 24))
    V = oracle.bf16_bits_to_f64(v)
    # one key: P8 = 112 exactly, O = dequantised v (per-channel scale = |v|
    # itself, so v maps to +-448 and back exactly)
    np.testing.assert_allclose(O, V, rtol=1e-6, atol=0)


def test_close_to_exact_attention():
    q, k, v, pos, cu = synth.draw_random_case([300, 129, 40], 2, 128, seed=306)
    O, L = oracle.sage_attention_ref(q, k, v, cu, 1 / math.sqrt(128), pos, (32, 48, 48))
    Oe, Le = oracle.attention_ref(q, k, v, cu, 1 / math.sqrt(128), pos, (32, 48, 48))
    err = np.abs(O - Oe)
    # FP8 P and V carry 3 mantissa bits: errors of a few 1e-3 on average
    assert err.max() < 0.1 and err.mean() < 0.01
    assert np.abs(L - Le).max() < 0.05


def test_rows_ref_matches_full():
    q, k, v, pos, cu = synth.draw_random_case([200, 150], 3, 128, seed=307)
    O, L = oracle.sage_attention_ref(q, k, v, cu, 0.09, pos, (32, 48, 48))
    rows = np.array([0, 5, 199, 200, 263, 349])
    Or, Lr = oracle.sage_attention_rows_ref(q, k, v, cu, 0.09, rows, [0, 2], pos, (32, 48, 48))
    np.testing.assert_allclose(Or, O[rows][:, [0, 2]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lr, L[[0, 2]][:, rows], rtol=0, atol=1e-12)
