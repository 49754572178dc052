"""Pins for the CPU oracle: closed forms, invariants and brute force.

Nothing here compares the oracle with itself through the same code path;
each check fails on a plausible mistake (dropped term, wrong sign, wrong
index or transposed operand) somewhere in ``oracle/``.
"""

import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------- bf16

def test_bf16_decode_closed_forms():
    bits = np.array([0x3F80, 0xC000, 0x3FC0, 0x0000, 0x8000, 0x7F7F, 0x0001, 0x4049],
                    dtype=np.uint16)
    want = [1.0, -2.0, 1.5, 0.0, -0.0, (2 - 2 ** -7) * 2.0 ** 127, 2.0 ** -133,
            3.140625]
    got = oracle.bf16_bits_to_f64(bits)
    assert got.dtype == np.float64
    assert list(got) == want


def test_generator_rounds_ties_to_even():
    # 1 + 2^-8 is a tie between 0x3F80 and 0x3F81 -> even 0x3F80;
    # 1 + 3*2^-8 is a tie between 0x3F81 and 0x3F82 -> even 0x3F82.
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -20],
                 dtype=np.float32)
    assert list(synth.f32_to_bf16_bits(x)) == [0x3F80, 0x3F82, 0xBF80, 0x3F81]


# ---------------------------------------------------------------- positions

def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def test_positions_closed_forms():
    n = 0
    for name, seg, tok, t, h, w in _golden_rows("positions_closed_form.txt"):
        wl = synth.workload(name)
        p = oracle.segment_positions(wl.segments[int(seg)])
        assert p.dtype == np.float32
        got = p[int(tok)]
        assert float(got[0]) == float(t), (name, seg, tok)
        assert float(got[1]) == float(h) and float(got[2]) == float(w), (name, seg, tok)
        n += 1
    assert n >= 20


def test_positions_shapes_and_audio_clock():
    for wl in synth.WORKLOADS:
        p = oracle.packed_positions(wl.segments)
        assert p.shape == (wl.n_tokens, 3)
    # audio tail spans exactly the video grid's T frames: strictly increasing,
    # first at the grid start, last below grid start + T
    lay = synth.workload("max").segments[0]
    p = oracle.segment_positions(lay)
    T = lay.video[0]
    tail = p[-lay.audio_tail:, 0].astype(np.float64)
    assert tail[0] == 0.0 and np.all(np.diff(tail) > 0) and tail[-1] < T
    assert np.all(p[-lay.audio_tail:, 1:] == 0)
    # each audio reference advances the clock by len / rate = 8
    lay = synth.workload("packed").segments[3]
    p = oracle.segment_positions(lay)
    start_video = 9 * 1008 + 3 * 256
    assert p[start_video, 0] == 9 + 3 * 8


# --------------------------------------------------------------------- RoPE

def test_rope_closed_form_rotations():
    n = 0
    for row in _golden_rows("rope_closed_form.txt"):
        st, sh, sw, theta, axis, pair, posv, _angle, c, s = row
        split = (int(st), int(sh), int(sw))
        D = sum(split)
        axis, pair = int(axis), int(pair)
        ch0 = sum(split[:axis]) + 2 * pair
        x = np.zeros((1, 1, D))
        x[0, 0, ch0] = 1.0
        pos = np.zeros((1, 3), dtype=np.float32)
        pos[0, axis] = np.float32(float(posv))
        y = oracle.rope_ref(x, pos, split, float(theta))
        want = np.zeros(D)
        want[ch0] = float(c)
        want[ch0 + 1] = float(s)
        np.testing.assert_allclose(y[0, 0], want, rtol=0, atol=1e-12)
        # the second channel of the pair rotates to (-sin, cos)
        x2 = np.zeros((1, 1, D))
        x2[0, 0, ch0 + 1] = 1.0
        y2 = oracle.rope_ref(x2, pos, split, float(theta))
        want2 = np.zeros(D)
        want2[ch0] = -float(s)
        want2[ch0 + 1] = float(c)
        np.testing.assert_allclose(y2[0, 0], want2, rtol=0, atol=1e-12)
        n += 1
    assert n == 8


def test_rope_half_layout_switch_moves_pairs():
    x = np.zeros((1, 1, 8))
    x[0, 0, 0] = 1.0
    pos = np.array([[1.0, 0, 0]], dtype=np.float32)
    y = oracle.rope_ref(x, pos, (8, 0, 0), 10000.0, pair_layout="half")
    assert abs(y[0, 0, 4] - math.sin(1.0)) < 1e-12 and abs(y[0, 0, 1]) == 0.0


@pytest.mark.parametrize("split", [(16, 24, 24), (32, 48, 48), (2, 4, 2)])
def test_rope_preserves_norm_per_axis_chunk(split):
    rng = _rng(1)
    D = sum(split)
    x = rng.standard_normal((37, 3, D))
    pos = (rng.random((37, 3)) * 100).astype(np.float32)
    y = oracle.rope_ref(x, pos, split, 10000.0)
    c = 0
    for d in split:
        nx = np.linalg.norm(x[:, :, c:c + d], axis=-1)
        ny = np.linalg.norm(y[:, :, c:c + d], axis=-1)
        np.testing.assert_allclose(ny, nx, rtol=1e-12, atol=1e-12)
        c += d
    assert not np.allclose(x, y)


def test_rope_identity_at_zero_and_composition():
    rng = _rng(2)
    split = (16, 24, 24)
    x = rng.standard_normal((11, 2, 64))
    zero = np.zeros((11, 3), dtype=np.float32)
    np.testing.assert_array_equal(oracle.rope_ref(x, zero, split, 10000.0), x)
    a = rng.integers(-40, 40, size=(11, 3)).astype(np.float32)
    b = rng.integers(-40, 40, size=(11, 3)).astype(np.float32)
    lhs = oracle.rope_ref(oracle.rope_ref(x, a, split, 10000.0), b, split, 10000.0)
    rhs = oracle.rope_ref(x, a + b, split, 10000.0)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-11)


def test_rope_dot_depends_only_on_position_difference():
    rng = _rng(3)
    split = (32, 48, 48)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    p = np.array([[3.0, 7.0, 11.0]], dtype=np.float32)
    pp = np.array([[9.0, 2.0, 30.0]], dtype=np.float32)
    base = np.dot(oracle.rope_ref(q, p, split, 1e4)[0, 0], oracle.rope_ref(k, pp, split, 1e4)[0, 0])
    for delta in ([1.0, 0, 0], [0, 5.0, 0], [0, 0, -17.0], [2.5, -3.0, 4.0]):
        d = np.array([delta], dtype=np.float32)
        got = np.dot(oracle.rope_ref(q, p + d, split, 1e4)[0, 0],
                     oracle.rope_ref(k, pp + d, split, 1e4)[0, 0])
        assert abs(got - base) < 1e-11 * max(1.0, abs(base))
    # and it does depend on the difference
    got = np.dot(oracle.rope_ref(q, p + np.float32(1), split, 1e4)[0, 0],
                 oracle.rope_ref(k, pp, split, 1e4)[0, 0])
    assert abs(got - base) > 1e-6


def test_rope_audio_tokens_leave_h_w_chunks_unchanged():
    rng = _rng(4)
    split = (32, 48, 48)
    x = rng.standard_normal((5, 2, 128))
    pos = np.zeros((5, 3), dtype=np.float32)
    pos[:, 0] = [0.25, 1.5, 7.0, 30.0, 59.9]
    y = oracle.rope_ref(x, pos, split, 1e4)
    np.testing.assert_array_equal(y[:, :, 32:], x[:, :, 32:])
    assert not np.allclose(y[1:, :, :32], x[1:, :, :32])


# ---------------------------------------------------------------- attention

def _tiny_case(seg_lens, H=2, D=8, split=(2, 4, 2), seed=5, std=1.0):
    q, k, v, pos, cu = synth.draw_random_case(seg_lens, H, D, seed, pos_range=8.0, std=std)
    return q, k, v, pos, cu, split


@pytest.mark.parametrize("seg_lens", [[5], [3, 4], [1, 6, 2], [0, 4, 0, 3]])
def test_attention_matches_dense_bruteforce(seg_lens):
    q, k, v, pos, cu, split = _tiny_case(seg_lens)
    scale = 1 / math.sqrt(8)
    O, L = oracle.attention_ref(q, k, v, cu, scale, pos, split, 10000.0, block=2)
    Ob, Lb = oracle.attention_dense_bruteforce(q, k, v, cu, scale, pos, split, 10000.0)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


def test_attention_matches_bruteforce_tiny_workload_shape():
    # the first workload's shape (2 segments of 80, 2 heads, D=64), cut to
    # 2 segments of 12 tokens so the scalar brute force stays fast
    wl = synth.workload("tiny")
    q, k, v = synth.draw_qkv(wl)
    pos = oracle.packed_positions(wl.segments)
    idx = np.r_[0:12, 80:92]
    cu = np.array([0, 12, 24], dtype=np.int32)
    O, L = oracle.attention_ref(q[idx], k[idx], v[idx], cu, wl.softmax_scale, pos[idx], wl.split)
    Ob, Lb = oracle.attention_dense_bruteforce(q[idx], k[idx], v[idx], cu, wl.softmax_scale,
                                               pos[idx], wl.split)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


def test_uniform_scores_give_segment_mean_of_v():
    seg = [7, 1, 12]
    q, k, v, pos, cu, split = _tiny_case(seg)
    q0 = np.zeros_like(q)                       # all scores zero
    O, L = oracle.attention_ref(q0, k, v, cu, 0.35, pos, split)
    V = oracle.bf16_bits_to_f64(v)
    for s in range(3):
        a, e = cu[s], cu[s + 1]
        np.testing.assert_allclose(O[a:e], np.broadcast_to(V[a:e].mean(0), O[a:e].shape),
                                   rtol=0, atol=1e-14)
        np.testing.assert_allclose(L[:, a:e], math.log(e - a), rtol=0, atol=1e-14)
    # scale = 0 gives the same closed form with any q
    O2, _ = oracle.attention_ref(q, k, v, cu, 0.0, pos, split)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-14)


def test_single_token_segments_return_v():
    q, k, v, pos, cu, split = _tiny_case([1] * 9)
    O, L = oracle.attention_ref(q, k, v, cu, 0.3, pos, split)
    np.testing.assert_array_equal(O, oracle.bf16_bits_to_f64(v))
    Qr = oracle.rope_ref(oracle.bf16_bits_to_f64(q), pos, split, 1e4)
    Kr = oracle.rope_ref(oracle.bf16_bits_to_f64(k), pos, split, 1e4)
    np.testing.assert_allclose(L.T, 0.3 * np.einsum("nhd,nhd->nh", Qr, Kr), atol=1e-12)


def test_packing_invariance():
    seg = [5, 9, 3]
    q, k, v, pos, cu, split = _tiny_case(seg, seed=9)
    O, L = oracle.attention_dense_bruteforce(q, k, v, cu, 0.4, pos, split)
    for s in range(3):
        a, e = cu[s], cu[s + 1]
        Os, Ls = oracle.attention_dense_bruteforce(q[a:e], k[a:e], v[a:e],
                                                   np.array([0, e - a]), 0.4, pos[a:e], split)
        np.testing.assert_allclose(O[a:e], Os, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L[:, a:e], Ls, rtol=0, atol=1e-13)


def test_key_shift_leaves_output_unchanged():
    # adding one vector w to every key adds q.w to a whole score row
    rng = _rng(7)
    q, k, v, pos, cu, split = _tiny_case([6, 5], seed=11)
    K = oracle.bf16_bits_to_f64(k)
    w = rng.standard_normal((1, 2, 8))
    O, L = oracle.attention_ref(q, K, v, cu, 0.5)
    O2, L2 = oracle.attention_ref(q, K + w, v, cu, 0.5)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    Q = oracle.bf16_bits_to_f64(q)
    np.testing.assert_allclose(L2 - L, 0.5 * np.einsum("nhd,hd->hn", Q, w[0]), atol=1e-12)


def test_large_logits_pick_the_argmax_value():
    # scores 0 and 1000 for the two keys: the softmax is one-hot up to e^-1000
    q = np.zeros((2, 1, 2)); k = np.zeros((2, 1, 2)); v = np.zeros((2, 1, 2))
    q[:, 0, 0] = 1.0
    k[1, 0, 0] = 1000.0
    v[0, 0] = [1.0, 2.0]; v[1, 0] = [-3.0, 5.0]
    O, L = oracle.attention_ref(q, k, v, np.array([0, 2]), 1.0)
    np.testing.assert_array_equal(O[:, 0], [[-3.0, 5.0], [-3.0, 5.0]])
    np.testing.assert_allclose(L[0], [1000.0, 1000.0], rtol=0, atol=1e-12)


def test_head_permutation_permutes_outputs():
    q, k, v, pos, cu, split = _tiny_case([4, 7], H=3, seed=13)
    perm = [2, 0, 1]
    O, L = oracle.attention_ref(q, k, v, cu, 0.3, pos, split)
    Op, Lp = oracle.attention_ref(q[:, perm], k[:, perm], v[:, perm], cu, 0.3, pos, split)
    np.testing.assert_array_equal(Op, O[:, perm])
    np.testing.assert_array_equal(Lp, L[perm])


def test_attention_invariant_to_shifting_a_segments_clock():
    # q.k after RoPE depends on position differences only, so moving every
    # position of a segment by the same delta leaves its attention unchanged
    q, k, v, pos, cu, split = _tiny_case([6, 9], seed=17)
    # positions on a 1/64 grid so that the shifted values stay exact in fp32
    pos = (np.round(pos.astype(np.float64) * 64) / 64).astype(np.float32)
    O, L = oracle.attention_ref(q, k, v, cu, 0.4, pos, split)
    pos2 = pos.copy()
    pos2[6:] += np.array([3.0, -2.0, 5.0], dtype=np.float32)
    O2, L2 = oracle.attention_ref(q, k, v, cu, 0.4, pos2, split)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L, rtol=0, atol=1e-12)
    # but it is not invariant to moving one token only
    pos3 = pos.copy()
    pos3[7] += np.float32(1.0)
    O3, _ = oracle.attention_ref(q, k, v, cu, 0.4, pos3, split)
    assert np.abs(O3[6:] - O[6:]).max() > 1e-6


def test_positions_clock_origin_shifts_t_only():
    # a continuation chunk on the global clock: with an origin that keeps the
    # values exact in float32 (integer video frames, audio steps of 1/32), every
    # t moves by the origin and h, w stay
    lay = synth.SegmentLayout(video=(3, 4, 5), audio_tail=96, image_refs=1,
                              image_grid=(2, 2), audio_refs=1, audio_ref_len=64,
                              audio_rate=32)
    base = oracle.segment_positions(lay)
    shifted = oracle.segment_positions(lay, 1441.0)
    np.testing.assert_array_equal(shifted[:, 1:], base[:, 1:])
    np.testing.assert_array_equal(shifted[:, 0].astype(np.float64),
                                  base[:, 0].astype(np.float64) + 1441.0)
    two = oracle.packed_positions([lay, lay], [0.0, 1441.0])
    np.testing.assert_array_equal(two, np.concatenate([base, shifted]))


def test_rope_inside_attention_equals_prerotated_inputs():
    q, k, v, pos, cu, split = _tiny_case([5, 4], seed=19)
    O, L = oracle.attention_ref(q, k, v, cu, 0.4, pos, split)
    Qr = oracle.rope_ref(oracle.bf16_bits_to_f64(q), pos, split, 1e4)
    Kr = oracle.rope_ref(oracle.bf16_bits_to_f64(k), pos, split, 1e4)
    O2, L2 = oracle.attention_ref(Qr, Kr, v, cu, 0.4)
    np.testing.assert_array_equal(O2, O)


def test_sampled_rows_match_full_oracle():
    wl = synth.workload("tiny")
    q, k, v = synth.draw_qkv(wl)
    pos = oracle.packed_positions(wl.segments)
    cu = synth.cu_seqlens_of(wl.seg_lens)
    O, L = oracle.attention_ref(q, k, v, cu, wl.softmax_scale, pos, wl.split)
    rows = [0, 5, 79, 80, 133, 159]
    Os, Ls = oracle.attention_rows_ref(q, k, v, cu, wl.softmax_scale, rows, [1, 0], pos, wl.split)
    np.testing.assert_allclose(Os, O[rows][:, [1, 0]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Ls, L[[1, 0]][:, rows], rtol=0, atol=1e-13)
