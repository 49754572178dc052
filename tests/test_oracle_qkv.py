"""Pins for oracle/qkv_rope.py."""

import numpy as np

import oracle
import synth


def test_projection_closed_form_and_split():
    # W = identity blocks: q, k, v are slices of X (then q, k rotated)
    N, H, D = 5, 2, 8
    K = 3 * H * D
    rng = np.random.default_rng(1)
    x = rng.standard_normal((N, K))
    w = np.eye(K)
    pos = np.zeros((N, 3), np.float32)
    q, k, v = oracle.qkv_rope_ref(x, w, H, D, pos, (2, 4, 2))
    np.testing.assert_array_equal(q.reshape(N, -1), x[:, :H * D])
    np.testing.assert_array_equal(k.reshape(N, -1), x[:, H * D:2 * H * D])
    np.testing.assert_array_equal(v.reshape(N, -1), x[:, 2 * H * D:])


def test_rotation_applies_to_q_and_k_only_and_matches_rope():
    N, H, D, K = 7, 2, 8, 12
    rng = np.random.default_rng(2)
    x = rng.standard_normal((N, K)); w = rng.standard_normal((3 * H * D, K))
    pos = (rng.random((N, 3)) * 10).astype(np.float32)
    q, k, v = oracle.qkv_rope_ref(x, w, H, D, pos, (2, 4, 2))
    q0, k0, v0 = oracle.qkv_rope_ref(x, w, H, D)
    np.testing.assert_array_equal(v, v0)
    np.testing.assert_allclose(q, oracle.rope_ref(q0, pos, (2, 4, 2), 1e4), atol=1e-12)
    np.testing.assert_allclose(k, oracle.rope_ref(k0, pos, (2, 4, 2), 1e4), atol=1e-12)
    # the projection is the matrix product, checked entry by entry with a scalar sum
    y = x @ w.T
    assert abs(y[3, 5] - sum(x[3, i] * w[5, i] for i in range(K))) < 1e-12
    np.testing.assert_allclose(q0.reshape(N, -1), y[:, :H * D], atol=1e-12)


def test_rows_selection():
    N, H, D, K = 9, 2, 8, 16
    rng = np.random.default_rng(3)
    x = synth.f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32))
    w = synth.f32_to_bf16_bits(rng.standard_normal((3 * H * D, K), dtype=np.float32))
    pos = (rng.random((N, 3)) * 10).astype(np.float32)
    full = oracle.qkv_rope_ref(x, w, H, D, pos, (2, 4, 2))
    part = oracle.qkv_rope_ref(x, w, H, D, pos, (2, 4, 2), rows=[1, 4, 8])
    for a, b in zip(full, part):
        np.testing.assert_array_equal(a[[1, 4, 8]], b)
