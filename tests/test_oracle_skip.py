"""Pins for the skip-softmax oracle (oracle/skip_softmax.py)."""

import math

import numpy as np

import oracle
import synth


def _two_tile_case(gap, H=1, D=8, L=256):
    # no RoPE; every query row is e0 and the keys of tile 0 score 1.0, those of
    # tile 1 score 1.0 - gap (scale 1), so exp(m_tile1 - m_run) = exp(-gap)
    q = np.zeros((L, H, D)); k = np.zeros((L, H, D))
    q[:, :, 0] = 1.0
    k[:128, :, 0] = 1.0
    k[128:, :, 0] = 1.0 - gap
    rng = np.random.default_rng(3)
    v = rng.standard_normal((L, H, D))
    return q, k, v, np.array([0, L])


def test_threshold_zero_is_dense_attention():
    q, k, v, pos, cu = synth.draw_random_case([300, 129, 77], 2, 16, seed=5, pos_range=16.0)
    O, L, skipped = oracle.attention_skip_ref(q, k, v, cu, 0.25, 0.0, pos, (4, 8, 4))
    Od, Ld = oracle.attention_ref(q, k, v, cu, 0.25, pos, (4, 8, 4))
    assert skipped == 0
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


def test_negligible_tile_is_dropped_closed_form():
    q, k, v, cu = _two_tile_case(gap=11.0)
    O, L, skipped = oracle.attention_skip_ref(q, k, v, cu, 1.0, 0.05)
    assert skipped == 256 // 32                     # every 32-row block skips tile 1
    # uniform scores over tile 0 -> the mean of its V rows; LSE = 1 + log 128
    np.testing.assert_allclose(O[:, 0], np.broadcast_to(v[:128, 0].mean(0), (256, 8)), atol=1e-12)
    np.testing.assert_allclose(L[0], 1.0 + math.log(128), atol=1e-12)


def test_threshold_boundary_at_a_known_gap():
    q, k, v, cu = _two_tile_case(gap=3.0)           # exp(-3) = 0.049787
    _, _, s_hi = oracle.attention_skip_ref(q, k, v, cu, 1.0, 0.05)
    O_lo, _, s_lo = oracle.attention_skip_ref(q, k, v, cu, 1.0, 0.049)
    assert s_hi == 8 and s_lo == 0
    Od, _ = oracle.attention_ref(q, k, v, cu, 1.0)
    np.testing.assert_allclose(O_lo, Od, rtol=0, atol=1e-12)


def test_decision_is_per_32_row_block():
    q, k, v, cu = _two_tile_case(gap=11.0)
    q[40, 0, 0] = -1.0           # row 40 now prefers tile 1 (its score there is 10)
    O, _, skipped = oracle.attention_skip_ref(q, k, v, cu, 1.0, 0.05)
    assert skipped == 7          # rows 32-63 keep tile 1, the other 7 blocks skip it
    Od, _ = oracle.attention_ref(q, k, v, cu, 1.0)
    np.testing.assert_allclose(O[32:64], Od[32:64], rtol=0, atol=1e-12)
    np.testing.assert_allclose(O[:32, 0], np.broadcast_to(v[:128, 0].mean(0), (32, 8)), atol=1e-12)


def test_sampled_rows_match_full_skip_oracle():
    q, k, v, cu = synth.draw_group_case([700, 300], 2, 16, group_len=100, amp=6.0, eps=0.05, seed=3)
    O, L, _ = oracle.attention_skip_ref(q, k, v, cu, 0.25, 0.05)
    rows = [0, 31, 32, 99, 100, 333, 699, 700, 731, 999]
    Os, Ls = oracle.attention_skip_rows_ref(q, k, v, cu, 0.25, 0.05, rows, [1, 0])
    np.testing.assert_allclose(Os, O[rows][:, [1, 0]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ls, L[[1, 0]][:, rows], rtol=0, atol=1e-12)


def test_group_inputs_skip_far_tiles_once_the_own_group_is_seen():
    # with clear locality, tiles past a query's own frame group are skipped
    q, k, v, cu = synth.draw_group_case([1024], 1, 16, group_len=256, amp=6.0, eps=0.05, seed=4)
    _, _, skipped = oracle.attention_skip_ref(q, k, v, cu, 0.25, 0.05)
    assert skipped > 0
