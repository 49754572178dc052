"""h3_rope_apply on the GPU against the float64 oracle.

Bound per element: the kernel rounds the rotated value to bf16 once (half an
ulp, at most 2^-8 relative) on top of fp32 angle/sincos error (~1e-6
absolute for |angle| <= 100), so |gpu - oracle| <= 2^-8 |oracle| + 1e-5.
"""

import numpy as np
import pytest

import oracle
import synth
from gpu_util import dev, dev_bf16, host_f64, host_bits

pytestmark = pytest.mark.gpu


def _h3():
    import audio_diffusion_transformer_h3_b200 as h3
    return h3


def _check_rope(x_bits, pos, split, theta=1e4, rows=None):
    import torch
    h3 = _h3()
    x = dev_bf16(x_bits)
    p = dev(pos)
    y = h3.rope_apply_t(x, p, split, theta)
    torch.cuda.synchronize()
    got = host_f64(y)
    if rows is not None:
        got = got[rows]
        x_bits = x_bits[rows]
        pos = pos[rows]
    want = oracle.rope_ref(oracle.bf16_bits_to_f64(x_bits), pos, split, theta)
    err = np.abs(got - want)
    bound = np.abs(want) * 2.0 ** -8 + 1e-5
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), float((err - bound).max())
    return y


@pytest.mark.parametrize("name", ["tiny", "single"])
def test_rope_workloads_full(name):
    wl = synth.workload(name)
    q, k, v = synth.draw_qkv(wl)
    pos = oracle.packed_positions(wl.segments)
    _check_rope(q, pos, wl.split)
    _check_rope(k, pos, wl.split)


def test_rope_max_workload_sampled_rows():
    wl = synth.workload("max")
    rng = np.random.default_rng(0)
    # draw only k of the largest workload (q has the same recipe)
    q, k, v = synth.draw_qkv(wl)
    del q, v
    pos = oracle.packed_positions(wl.segments)
    rows = np.unique(np.r_[0:4, 60475:60485, 62276:62284, wl.n_tokens - 4:wl.n_tokens,
                           rng.integers(0, wl.n_tokens, 200)])
    _check_rope(k, pos, wl.split, rows=rows)


@pytest.mark.parametrize("N,H,D,split", [(1, 1, 64, (16, 24, 24)), (7, 3, 128, (32, 48, 48)),
                                         (9, 5, 64, (0, 32, 32)), (33, 2, 128, (128, 0, 0)),
                                         (1000, 3, 128, (32, 48, 48))])
def test_rope_edge_shapes(N, H, D, split):
    q, k, v, pos, cu = synth.draw_random_case([N], H, D, seed=N + H, pos_range=100.0)
    _check_rope(q, pos, split)


def test_rope_in_place_and_deterministic():
    import torch
    h3 = _h3()
    q, k, v, pos, cu = synth.draw_random_case([513], 4, 128, seed=3)
    x = dev_bf16(q)
    p = dev(pos)
    y = h3.rope_apply_t(x, p, (32, 48, 48))
    y2 = h3.rope_apply_t(x, p, (32, 48, 48))
    h3.rope_apply_t(x, p, (32, 48, 48), out=x)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(y), host_bits(y2))
    assert np.array_equal(host_bits(y), host_bits(x))


def test_rope_zero_positions_is_identity():
    import torch
    h3 = _h3()
    q, k, v, pos, cu = synth.draw_random_case([100], 2, 128, seed=4)
    x = dev_bf16(q)
    y = h3.rope_apply_t(x, dev(np.zeros_like(pos)), (32, 48, 48))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(y), q)
