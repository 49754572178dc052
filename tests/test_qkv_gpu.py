"""h3_qkv_rope_gemm (QKV projection with RoPE on q and k in the epilogue) on
the GPU against the float64 oracle (oracle/qkv_rope.py).

Tolerance: each output is one bf16 rounding of an fp32 value, so the
elementwise bound is 2^-8 |ref| (a full bf16 ulp, twice the rounding error)
plus 2e-3 for the fp32 accumulation and the fp32 rotation; the outputs are
~N(0, 1) (w is scaled by 1/sqrt(K)), so the path's own bound (max |d| <=
2e-2, mean |d| <= 2e-3) is checked as well.
"""

import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_close_bf16, dev, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8
ABS = 2e-3


def _h3():
    import audio_diffusion_transformer_h3_b200 as h3
    return h3


def _run(x, w, H, D, pos=None, split=None, theta=1e4):
    import torch
    h3 = _h3()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    q, k, v = h3.qkv_rope_gemm_t(dev_bf16(x), dev_bf16(w), H, D,
                                 None if pos is None else dev(pos), split, theta, workspace=ws)
    torch.cuda.synchronize()
    assert h3.device_status_t(ws) == h3.H3_OK
    return q, k, v


def _check(got, want, what):
    g = host_f64(got)
    err = np.abs(g - want)
    bound = REL * np.abs(want) + ABS
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {len(bad)} outside bound, first {bad[:3].tolist()}, " \
                          f"max|d|={err.max():.3g}"
    assert_close_bf16(g, want, what)


def _pos(N, seed, rng_range=64.0):
    rng = np.random.default_rng(seed)
    return (rng.random((N, 3), dtype=np.float32) * np.float32(rng_range)).astype(np.float32)


@pytest.mark.parametrize("N,K,H,D,split", [
    (300, 192, 2, 128, (32, 48, 48)),     # 3 row tiles (ragged), 3 column tiles
    (300, 192, 4, 64, (16, 24, 24)),      # two heads of 64 per column tile
    (129, 64, 4, 128, (32, 48, 48)),      # one k-step, one row past a tile
    (1, 128, 2, 128, (32, 48, 48)),       # a single token
])
def test_small_parity(N, K, H, D, split):
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=N + K + H + D)
    pos = _pos(N, seed=N)
    q, k, v = _run(x, w, H, D, pos, split)
    Q, Kr, V = oracle.qkv_rope_ref(x, w, H, D, pos, split)
    _check(q, Q, "q")
    _check(k, Kr, "k")
    _check(v, V, "v")


def test_many_tiles_per_cta():
    # 40 row tiles (two raster groups, the second partial) x 24 column tiles:
    # every CTA takes several tiles, both accumulators and every barrier phase
    # wrap; 5 k-steps per tile make the 4-stage ring wrap across tiles
    N, K, H, D, split = 5050, 320, 16, 128, (32, 48, 48)
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=71)
    pos = _pos(N, seed=72)
    q, k, v = _run(x, w, H, D, pos, split)
    Q, Kr, V = oracle.qkv_rope_ref(x, w, H, D, pos, split)
    _check(q, Q, "q")
    _check(k, Kr, "k")
    _check(v, V, "v")


def test_without_positions_is_the_plain_projection():
    N, K, H, D = 700, 256, 2, 128
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=73)
    q, k, v = _run(x, w, H, D)
    Q, Kr, V = oracle.qkv_rope_ref(x, w, H, D)
    _check(q, Q, "q")
    _check(k, Kr, "k")
    _check(v, V, "v")


@pytest.mark.parametrize("D,split", [(128, (32, 48, 48)), (64, (16, 24, 24))])
def test_exact_projection_matches_standalone_rope_bitwise(D, split):
    # w = [I; I; I] makes the fp32 accumulator hold x exactly, so the fused
    # rotation must equal h3_rope_apply on x bit for bit (same table, pair
    # layout and rounding sequence), and v must equal x
    import torch
    h3 = _h3()
    H = 256 // D
    N, K = 517, H * D
    x, _ = synth.draw_linear_case(N, K, 1, seed=74)
    one = np.uint16(0x3F80)                                   # bf16 1.0
    eye = np.where(np.eye(K, dtype=bool), one, np.uint16(0))
    w = np.concatenate([eye, eye, eye], axis=0)
    pos = _pos(N, seed=75)
    q, k, v = _run(x, w, H, D, pos, split)
    xr = h3.rope_apply_t(dev_bf16(x.reshape(N, H, D)), dev(pos), split, 1e4)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(q), host_bits(xr))
    assert np.array_equal(host_bits(k), host_bits(xr))
    assert np.array_equal(host_bits(v).reshape(N, K), x)


def test_deterministic():
    N, K, H, D = 1000, 384, 4, 128
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=76)
    pos = _pos(N, seed=77)
    a = _run(x, w, H, D, pos, (32, 48, 48))
    b = _run(x, w, H, D, pos, (32, 48, 48))
    for t, u in zip(a, b):
        assert np.array_equal(host_bits(t), host_bits(u))


def test_projection_feeds_attention():
    # the fused projection's q, k (already rotated) go to the attention with
    # no positions; the result matches the oracle's projection + attention
    import torch
    h3 = _h3()
    seg = [300, 211]
    N, K, H, D = sum(seg), 256, 2, 128
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=78)
    pos = _pos(N, seed=79, rng_range=16.0)
    cu = synth.cu_seqlens_of(seg)
    q, k, v = _run(x, w, H, D, pos, (32, 48, 48))
    o = h3.varlen_attn_fwd_t(q, k, v, dev(cu), max(seg), softmax_scale=D ** -0.5)
    torch.cuda.synchronize()
    Q, Kr, V = oracle.qkv_rope_ref(x, w, H, D, pos, (32, 48, 48))
    # the attention takes bf16 tensors: round the oracle's projections too
    Qb, Kb, Vb = (synth.f32_to_bf16_bits(t.astype(np.float32)) for t in (Q, Kr, V))
    O, _ = oracle.attention_ref(Qb, Kb, Vb, cu, D ** -0.5)
    assert_close_bf16(host_f64(o), O, "projection -> attention")


def test_dit_projection_full_size_sampled():
    # the DiT's qkv projection (hidden 5376 -> 3 x 56 x 128) over the tokens
    # of the largest attention workload, with its positions; sampled rows
    import torch
    p = synth.QKV_PROJECTION
    wl = synth.workload("max")
    N, K, H, D = wl.n_tokens, p.hidden, p.heads, p.head_dim
    x, w = synth.draw_linear_case(N, K, p.out_features, seed=80)
    pos = oracle.packed_positions(wl.segments).astype(np.float32)
    q, k, v = _run(x, w, H, D, pos, p.split, p.theta)
    rng = np.random.default_rng(81)
    rows = np.unique(np.r_[0:8, N - 8:N, 62270:62290, rng.integers(0, N, 24)])
    Q, Kr, V = oracle.qkv_rope_ref(x[rows], w, H, D, pos[rows], p.split, p.theta)
    idx = torch.as_tensor(rows).cuda()
    _check(q[idx], Q, "q")
    _check(k[idx], Kr, "k")
    _check(v[idx], V, "v")


# ------------------------------------------ projection chained into attention

def test_chained_projection_attention_single_workload_in_full():
    # h3_qkv_rope_attn_fwd on the single-clip workload (8,320 tokens, 24 heads,
    # hidden 5,376 as in the DiT): the projection rotates q and k in its
    # epilogue and the attention reads them without positions. Every output
    # element is compared with the float64 oracle chain (projection, rotation,
    # attention, no intermediate rounding) within the path's tolerance.
    import torch
    from oracle_pool import attention_rows_parallel
    h3 = _h3()
    wl = synth.workload("single")
    H, D, K = wl.heads, wl.head_dim, synth.QKV_PROJECTION.hidden
    x, w = synth.draw_linear_case(wl.n_tokens, K, 3 * H * D, seed=141)
    pos, cu = h3.h3_build_positions(wl.segments)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    qkv = tuple(torch.empty((wl.n_tokens, H, D), dtype=torch.bfloat16, device="cuda")
                for _ in range(3))
    o, lse = h3.qkv_rope_attn_fwd_t(dev_bf16(x), dev_bf16(w), H, D, dev(cu), wl.max_seqlen,
                                    dev(pos), wl.split, wl.theta, wl.softmax_scale, qkv=qkv,
                                    return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    assert h3.device_status_t(ws) == h3.H3_OK
    Q, Kr, V = oracle.qkv_rope_ref(x, w, H, D, oracle.packed_positions(wl.segments), wl.split,
                                   wl.theta)
    for got, want, name in ((qkv[0], Q, "q"), (qkv[1], Kr, "k"), (qkv[2], V, "v")):
        _check(got, want, f"chained projection {name}")
    O, L = attention_rows_parallel(Q, Kr, V, cu, wl.softmax_scale, np.arange(wl.n_tokens),
                                   range(H))
    assert_close_bf16(host_f64(o), O, "chained projection + attention (all elements)")
    np.testing.assert_allclose(host_f64(lse), L, rtol=0, atol=1e-2)


def test_chained_projection_attention_equals_the_two_calls_bitwise():
    # the chain is the projection followed by the attention without positions
    import torch
    h3 = _h3()
    seg = [300, 129, 1000]
    N, K, H, D, split = sum(seg), 256, 2, 128, (32, 48, 48)
    x, w = synth.draw_linear_case(N, K, 3 * H * D, seed=142)
    pos = _pos(N, 143)
    cu = synth.cu_seqlens_of(seg)
    o1 = h3.qkv_rope_attn_fwd_t(dev_bf16(x), dev_bf16(w), H, D, dev(cu), 1000, dev(pos), split,
                                1e4, 0.09)
    q, k, v = _run(x, w, H, D, pos, split)
    o2 = h3.varlen_attn_fwd_t(q, k, v, dev(cu), 1000, None, None, 1e4, 0.09)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(o1), host_bits(o2))
