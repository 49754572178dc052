"""h3_varlen_attn_fwd_skip (Skip-Softmax, lossy) on the GPU against the float64
skip-softmax oracle (oracle/skip_softmax.py).

The decision to skip a (32-row block, key tile) pair compares scores computed
in different precisions on the two sides, so parity is checked on inputs
whose decisions are far from the threshold (frame-group locality from
synth.draw_group_case: a tile is either within ~1 of the row max or ~20
below it); there the skipped counts must agree exactly and the outputs within
the tolerance of the dense path (max |d| <= 2e-2, mean |d| <= 2e-3).
"""

import math

import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close_bf16, dev, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _h3():
    import audio_diffusion_transformer_h3_b200 as h3
    return h3


def _skip(q, k, v, cu, max_seqlen, thr, pos=None, split=None, scale=None):
    import torch
    h3 = _h3()
    N, H, D = q.shape
    ws = h3.workspace_for(N, H, D, len(cu) - 1)
    o, lse = h3.varlen_attn_fwd_skip_t(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu),
                                       max_seqlen, thr, None if pos is None else dev(pos),
                                       split, 1e4, scale, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    assert h3.device_status_t(ws) == h3.H3_OK
    return o, lse, h3.skip_count_t(ws)


def _dense(q, k, v, cu, max_seqlen, pos=None, split=None, scale=None):
    import torch
    h3 = _h3()
    o = h3.varlen_attn_fwd_t(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu), max_seqlen,
                             None if pos is None else dev(pos), split, 1e4, scale)
    torch.cuda.synchronize()
    return o


def test_threshold_zero_equals_dense_bitwise():
    q, k, v, pos, cu = synth.draw_random_case([700, 129, 300], 3, 128, seed=201)
    o, lse, n = _skip(q, k, v, cu, 700, 0.0, pos, (32, 48, 48), 0.09)
    assert n == 0
    assert np.array_equal(host_bits(o), host_bits(_dense(q, k, v, cu, 700, pos, (32, 48, 48), 0.09)))


def test_random_inputs_skip_nothing_at_the_pages_threshold():
    # N(0,1) inputs: tile maxima stay within ~1 of the running max, far above
    # log(0.05); the oracle agrees that nothing is skipped
    q, k, v, pos, cu = synth.draw_random_case([900, 400], 2, 128, seed=202)
    o, _, n = _skip(q, k, v, cu, 900, 0.05, pos, (32, 48, 48), 1 / math.sqrt(128))
    _, _, n_ref = oracle.attention_skip_ref(q, k, v, cu, 1 / math.sqrt(128), 0.05, pos, (32, 48, 48))
    assert n == n_ref == 0
    assert np.array_equal(host_bits(o), host_bits(_dense(q, k, v, cu, 900, pos, (32, 48, 48),
                                                        1 / math.sqrt(128))))


@pytest.mark.parametrize("D", [64, 128])
def test_group_locality_parity_and_count(D):
    seg = [3000, 1200, 77]
    q, k, v, cu = synth.draw_group_case(seg, 2, D, group_len=256, amp=15.0, eps=0.05, seed=203)
    scale = 1.0 / math.sqrt(D)
    o, lse, n = _skip(q, k, v, cu, 3000, 0.05, scale=scale)
    O, L, n_ref = oracle.attention_skip_ref(q, k, v, cu, scale, 0.05)
    assert n_ref > 0 and n == n_ref
    assert_close_bf16(host_f64(o), O, f"skip D={D}")
    np.testing.assert_allclose(host_f64(lse), L, rtol=0, atol=2e-2)
    # the skipped tiles are negligible by construction (weights ~ e^-20 or less),
    # so the sparse result also equals dense attention up to rounding
    Od, _ = oracle.attention_ref(q, k, v, cu, scale)
    assert np.abs(Od - O).max() < 1e-6


def test_group_locality_full_size_sampled():
    # the shape of the largest workload (62,280 + 16,128 tokens, 48 heads)
    import torch
    wl = synth.workload("max")
    q, k, v, cu = synth.draw_group_case(wl.seg_lens, wl.heads, wl.head_dim, group_len=1008,
                                        amp=15.0, eps=0.05, seed=204)
    o, lse, n = _skip(q, k, v, cu, wl.max_seqlen, 0.05, scale=wl.softmax_scale)
    rng = np.random.default_rng(5)
    rows = np.unique(np.r_[0:40, 62240:62320, rng.integers(0, wl.n_tokens, 60)])
    heads = [0, 47]
    O, L = oracle.attention_skip_rows_ref(q, k, v, cu, wl.softmax_scale, 0.05, rows, heads)
    got = host_f64(o[torch.as_tensor(rows).cuda()][:, heads])
    assert_close_bf16(got, O, "skip max-size sampled")
    # a large share of the (block, tile) pairs is skipped on these inputs
    n_pairs = sum(((L_ + 31) // 32) * ((L_ + 127) // 128 - 1) for L_ in wl.seg_lens) * wl.heads
    assert n > 0.3 * n_pairs


def test_skip_threshold_argument_checked_on_host():
    h3 = _h3()
    cfg = h3.rope_cfg((32, 48, 48), 1e4)
    for bad in (-0.1, 1.5, float("nan")):
        st = h3.h3_varlen_attn_fwd_skip(0x10000, 0x20000, 0x30000, 0x40000, 0, 0x50000, 1, 8,
                                        0, cfg, 8, 1, 128, 0.1, bad, 0x70000, 1 << 20, 0)
        assert st == h3.H3_ERR_INVALID_ARG
