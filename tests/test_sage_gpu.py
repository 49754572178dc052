"""h3_varlen_attn_fwd_sage (SAGE-style FP8 attention, lossy) on the GPU against
the SAGE oracle (oracle/sage.py).

Without positions the quantisation is decided in the same float32 arithmetic
on both sides (max, 448 / max, one product, e4m3 round-to-nearest-even), so
every code and scale must agree bit for bit. With positions the rotation
differs in the last float32 bits (fp32 sincos on the GPU, float64 on the
oracle), so a few codes may sit on the other side of a rounding boundary:
those are compared through their dequantised values. The attention output is
compared with the SAGE oracle within the path's tolerance (max |d| <= 2e-2,
mean |d| <= 2e-3). Its distance to EXACT attention (the float64 oracle of
the dense path) is bounded separately, by a first-order model of e4m3
rounding of Q, K, P and V (tests/fp8_error_model.py) that knows nothing of
the kernel's tiling, lazy maximum or scale choices: every element within 6
of the model's standard deviations (plus the bf16 rounding of the output),
and the mean error below the mean predicted deviation.
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


def _run(q, k, v, cu, max_seqlen, pos=None, split=None, scale=None, ws=None):
    import torch
    h3 = _h3()
    N, H, D = q.shape
    nseg = len(cu) - 1
    ws = h3.sage_workspace_for(N, H, D, nseg) if ws is None else ws
    o, lse = h3.varlen_attn_fwd_sage_t(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu),
                                       max_seqlen, None if pos is None else dev(pos), split,
                                       1e4, scale, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    return o, lse, ws


def test_quantisation_bit_exact_without_rotation():
    h3 = _h3()
    seg = [300, 129, 40, 1, 0, 16]
    q, k, v, _, cu = synth.draw_random_case(seg, 2, 128, seed=401)
    N = sum(seg)
    _, _, ws = _run(q, k, v, cu, 300)
    assert h3.device_status_t(ws) == h3.H3_OK
    got = h3.sage_workspace_views(ws, N, 2, len(seg))
    z = oracle.sage_quantize(q, k, v, cu)
    for name in ("q8", "k8", "v8"):
        assert np.array_equal(got[name].cpu().numpy(), oracle.e4m3_encode(z[name])), name
    for name in ("s_q", "s_k", "s_v"):
        assert np.array_equal(got[name].cpu().numpy().view(np.uint32),
                              z[name].astype(np.float32).view(np.uint32)), name


def test_quantisation_with_rotation_agrees_up_to_boundary_cases():
    h3 = _h3()
    seg = [700, 260]
    q, k, v, pos, cu = synth.draw_random_case(seg, 2, 128, seed=402)
    N = sum(seg)
    _, _, ws = _run(q, k, v, cu, 700, pos, (32, 48, 48))
    got = h3.sage_workspace_views(ws, N, 2, len(seg))
    z = oracle.sage_quantize(q, k, v, cu, pos, (32, 48, 48))
    assert np.array_equal(got["v8"].cpu().numpy(), oracle.e4m3_encode(z["v8"]))
    for name, sname in (("q8", "s_q"), ("k8", "s_k")):
        codes = got[name].cpu().numpy()
        want = oracle.e4m3_encode(z[name])
        assert np.mean(codes != want) < 1e-3, name
        deq_g = oracle.e4m3_decode(codes) * got[sname].cpu().numpy().T[:, :, None]
        deq_o = z[name] * z[sname].T[:, :, None]
        # one e4m3 step (relative 2^-3) at most, where the codes differ
        assert np.all(np.abs(deq_g - deq_o) <= 2.0 ** -3 * np.abs(deq_o) + 1e-6), name


@pytest.mark.parametrize("seg_lens", [[300, 129, 40], [1, 1, 2], [0, 513, 0, 17], [1000]])
def test_attention_parity_with_rotation(seg_lens):
    q, k, v, pos, cu = synth.draw_random_case(seg_lens, 2, 128, seed=sum(seg_lens) + 403)
    ms = max(max(seg_lens), 1)
    scale = 1 / math.sqrt(128)
    o, lse, _ = _run(q, k, v, cu, ms, pos, (32, 48, 48), scale)
    O, L = oracle.sage_attention_ref(q, k, v, cu, scale, pos, (32, 48, 48))
    assert_close_bf16(host_f64(o), O, f"sage {seg_lens}")
    np.testing.assert_allclose(host_f64(lse), L, rtol=0, atol=1e-2)
    # the lossy error against exact attention stays inside the e4m3 model
    from fp8_error_model import sigma_rows
    got = host_f64(o)
    for s in range(len(seg_lens)):
        a, e = int(cu[s]), int(cu[s + 1])
        for h in range(2):
            if e > a:
                Oe, sig = sigma_rows(q, k, v, cu, scale, np.arange(a, e), h, pos, (32, 48, 48))
                _assert_within_fp8_model(got[a:e, h], Oe, sig, f"{seg_lens} seg {s} head {h}")


def _assert_within_fp8_model(got, exact, sigma, what):
    bound = sigma + 2.0 ** -9 * np.abs(exact)
    err = np.abs(got - exact)
    z = err / bound
    assert np.all(np.isfinite(got)), what
    assert z.max() <= 6.0, f"{what}: max error {z.max():.2f} model deviations"
    assert err.mean() <= bound.mean(), f"{what}: mean |d| {err.mean():.3g} > {bound.mean():.3g}"


@pytest.mark.parametrize("name", ["long", "max"])
def test_full_size_against_exact_attention(name):
    # the lossy error of the whole FP8 path against exact float64 attention,
    # at full size: sampled rows of every segment (its edges and random rows)
    # on a strided set of heads, bounded by the e4m3 error model
    import torch
    from oracle_pool import fp8_sigma_rows_parallel
    wl = synth.workload(name)
    q, k, v = synth.draw_qkv(wl)
    pos = oracle.packed_positions(wl.segments).astype(np.float32)
    cu = synth.cu_seqlens_of(wl.seg_lens)
    o, _, ws = _run(q, k, v, cu, wl.max_seqlen, pos, wl.split, wl.softmax_scale)
    assert _h3().device_status_t(ws) == _h3().H3_OK
    rng = np.random.default_rng(wl.index + 200)
    rows = []
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        rows += [r for r in (a, a + 1, a + 127, a + 128, e - 129, e - 2, e - 1) if a <= r < e]
        rows += list(rng.integers(a, e, 32))
    rows = np.unique(np.asarray(rows, dtype=np.int64))
    heads = list(range(0, wl.heads, 8))
    idx = torch.as_tensor(rows).cuda()
    got = host_f64(o[idx][:, heads])
    Oe, sig = fp8_sigma_rows_parallel(q, k, v, cu, wl.softmax_scale, rows, heads, pos,
                                      wl.split, wl.theta)
    _assert_within_fp8_model(got, Oe, sig, f"sage {name} vs exact")


def test_scale_zero_gives_the_mean_of_v_on_lossless_inputs():
    rng = np.random.default_rng(404)
    seg = [37, 300, 1]
    N, H, D = sum(seg), 2, 128

    def lossless(c):
        x = rng.choice([-1.0, 0.0, 1.0], size=(N, H, D)) * c
        x[:, :, 0] = c
        return synth.f32_to_bf16_bits(x.astype(np.float32))
    q, k, v = lossless(0.875), lossless(3.5), lossless(1.75)
    cu = synth.cu_seqlens_of(seg)
    o, lse, _ = _run(q, k, v, cu, 300, scale=0.0)
    V = oracle.bf16_bits_to_f64(v)
    for s in range(len(seg)):
        a, e = int(cu[s]), int(cu[s + 1])
        want = np.broadcast_to(V[a:e].mean(axis=0), (e - a, H, D))
        np.testing.assert_allclose(host_f64(o[a:e]), want, rtol=2.0 ** -8, atol=1e-6)
        # every score is 0, so every exponential is evaluated at the same point
        # and the row sum carries that point's relative error in full: half of
        # the exponentials run on the degree-2 polynomial (relative error below
        # 1.8e-3, tests/test_exp2_fma.py), so |LSE - log n| <= -log(1 - 1.8e-3)
        np.testing.assert_allclose(host_f64(lse[:, a:e]), math.log(e - a), rtol=0,
                                   atol=-math.log1p(-1.8e-3))


def test_deterministic():
    q, k, v, pos, cu = synth.draw_random_case([900, 333], 3, 128, seed=405)
    a, _, _ = _run(q, k, v, cu, 900, pos, (32, 48, 48))
    b, _, _ = _run(q, k, v, cu, 900, pos, (32, 48, 48))
    assert np.array_equal(host_bits(a), host_bits(b))


def test_bad_seqlens_reported_without_access_outside():
    import torch
    h3 = _h3()
    q, k, v, _, _ = synth.draw_random_case([300], 2, 128, seed=406)
    for cu in (np.array([0, 200, 150, 300], dtype=np.int32),
               np.array([0, 100, 400], dtype=np.int32)):
        ws = h3.sage_workspace_for(300, 2, 128, len(cu) - 1)
        h3.varlen_attn_fwd_sage_t(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu), 300,
                                  workspace=ws)
        torch.cuda.synchronize()
        assert h3.device_status_t(ws) == h3.H3_ERR_BAD_SEQLENS


def test_full_size_sampled():
    # the largest workload's shape and positions (62,280 + 16,128 tokens, 48 heads)
    import torch
    wl = synth.workload("max")
    q, k, v = synth.draw_qkv(wl)
    pos = oracle.packed_positions(wl.segments).astype(np.float32)
    cu = synth.cu_seqlens_of(wl.seg_lens)
    o, lse, ws = _run(q, k, v, cu, wl.max_seqlen, pos, wl.split, wl.softmax_scale)
    assert _h3().device_status_t(ws) == _h3().H3_OK
    rng = np.random.default_rng(7)
    rows = np.unique(np.r_[0:24, 62260:62300, wl.n_tokens - 8:wl.n_tokens,
                          rng.integers(0, wl.n_tokens, 40)])
    heads = [0, 47]
    O, L = oracle.sage_attention_rows_ref(q, k, v, cu, wl.softmax_scale, rows, heads, pos,
                                          wl.split)
    idx = torch.as_tensor(rows).cuda()
    assert_close_bf16(host_f64(o[idx][:, heads]), O, "sage max-size sampled")
    np.testing.assert_allclose(host_f64(lse[heads][:, idx]), L, rtol=0, atol=1e-2)
