"""h3_varlen_attn_fwd_static against h3_varlen_attn_fwd, through the C ABI.

The static entry point serves hosts that cannot allocate device memory (they
own all of it, or allocate only at start-up), so it cannot be given a
workspace; it uses scratch compiled into the library instead. Its output must
match the workspace entry point's within the tolerance of the other GPU tests
(max |d| <= 2e-2, mean |d| <= 2e-3; here the two are the same kernels, so
they agree exactly), on two calls in a row, with different inputs, so that
what the first call leaves in the shared scratch cannot leak into the second.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process
(its first call does the per-device set-up).
"""

import math

import numpy as np
import pytest

import synth
from gpu_util import assert_close_bf16, dev, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu


def _inputs(seg_lens, H, D, split, seed):
    q, k, v, pos, cu = synth.draw_random_case(seg_lens, H, D, seed, pos_range=64.0)
    return dict(q=dev_bf16(q), k=dev_bf16(k), v=dev_bf16(v), pos=dev(pos), cu=dev(cu),
                max_seqlen=max(seg_lens), split=split, N=q.shape[0], H=H, D=D, nseg=len(seg_lens))


def _workload_inputs(name):
    import audio_diffusion_transformer_h3_b200 as h3
    wl = synth.workload(name)
    q, k, v = synth.draw_qkv(wl)
    pos, cu = h3.h3_build_positions(wl.segments)
    return dict(q=dev_bf16(q), k=dev_bf16(k), v=dev_bf16(v), pos=dev(pos), cu=dev(cu),
                max_seqlen=wl.max_seqlen, split=wl.split, N=wl.n_tokens, H=wl.heads,
                D=wl.head_dim, nseg=len(wl.seg_lens))


def _reference(x, scale):
    import torch
    import audio_diffusion_transformer_h3_b200 as h3
    o, lse = h3.varlen_attn_fwd_t(x["q"], x["k"], x["v"], x["cu"], x["max_seqlen"], x["pos"],
                                  x["split"], 1e4, scale, return_lse=True)
    torch.cuda.synchronize()
    return o, lse


def _static(x, scale):
    import torch
    import audio_diffusion_transformer_h3_b200 as h3
    o = torch.empty_like(x["q"])
    lse = torch.empty((x["H"], x["N"]), dtype=torch.float32, device="cuda")
    st = h3.h3_varlen_attn_fwd_static(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
        x["cu"].data_ptr(), x["nseg"], x["max_seqlen"], x["pos"].data_ptr(),
        h3.rope_cfg(x["split"], 1e4), x["N"], x["H"], x["D"], scale,
        torch.cuda.current_stream().cuda_stream)
    assert st == h3.H3_OK, h3.h3_status_string(st)
    torch.cuda.synchronize()
    return o, lse


def _compare(got, want):
    o, lse = got
    o_ref, lse_ref = want
    assert_close_bf16(host_f64(o), host_f64(o_ref), "static vs workspace entry point")
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), rtol=0, atol=1e-2)


@pytest.mark.parametrize("first,second", [
    (("tiny", None), ("rand", ([300, 129, 1000], 3, 128, (32, 48, 48), 5))),
    (("rand", ([77, 640], 2, 64, (16, 24, 24), 6)), ("single", None)),
])
def test_static_entry_matches_workspace_entry_on_two_calls(first, second):
    xs = []
    for kind, arg in (first, second):
        xs.append(_workload_inputs(kind) if kind != "rand" else _inputs(*arg))
    refs = [_reference(x, 1.0 / math.sqrt(x["D"])) for x in xs]
    outs = [_static(x, 1.0 / math.sqrt(x["D"])) for x in xs]   # two calls in a row
    for got, want in zip(outs, refs):
        _compare(got, want)
        assert np.array_equal(host_bits(got[0]), host_bits(want[0]))
    # and the first input again after the second one
    _compare(_static(xs[0], 1.0 / math.sqrt(xs[0]["D"])), refs[0])


def test_static_entry_rejects_sizes_beyond_its_scratch():
    import audio_diffusion_transformer_h3_b200 as h3
    # N*H*D = 2^25 + 128 elements does not fit; rejected before anything is
    # enqueued. Every pointer is NULL: if the size check ever moved behind the
    # argument checks, the call would still fail on the host (invalid
    # argument) instead of launching anything.
    N, H, D = (1 << 18) + 1, 1, 128
    st = h3.h3_varlen_attn_fwd_static(0, 0, 0, 0, 0, 0, 1, N, 0,
                                      h3.rope_cfg((32, 48, 48), 1e4), N, H, D, 0.1, 0)
    assert st == h3.H3_ERR_WORKSPACE
    # malformed shapes report what h3_varlen_attn_fwd reports, also when too large
    assert h3.h3_varlen_attn_fwd_static(0, 0, 0, 0, 0, 0, 1, N, 0,
                                        h3.rope_cfg((32, 48, 48), 1e4), N, H, 256, 0.1,
                                        0) == h3.H3_ERR_UNSUPPORTED
    assert h3.h3_varlen_attn_fwd_static(0, 0, 0, 0, 0, 0, 0, N, 0,
                                        h3.rope_cfg((32, 48, 48), 1e4), N, H, D, 0.1,
                                        0) == h3.H3_ERR_INVALID_ARG
    assert h3.h3_workspace_size(1 << 18, 1, 128, 1) <= h3.H3_STATIC_WORKSPACE_BYTES
