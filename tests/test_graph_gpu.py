"""The entry points inside a CUDA graph: each call enqueues only asynchronous
work on the given stream (no allocation, no synchronisation), so it can be
captured once and replayed on new inputs written into the same buffers. A
replay must equal an eager call on those inputs bit for bit."""

import numpy as np
import pytest

import synth
from gpu_util import dev, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


def _h3():
    import audio_diffusion_transformer_h3_b200 as h3
    return h3


def test_attention_graph_replay_equals_eager():
    import torch
    h3 = _h3()
    seg = [700, 129, 300]
    q, k, v, pos, cu = synth.draw_random_case(seg, 3, 128, seed=501)
    tq, tk, tv, tcu, tpos = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu), dev(pos)
    N, H, D = q.shape
    out = torch.empty_like(tq)
    lse = torch.empty((H, N), dtype=torch.float32, device="cuda")
    ws = h3.workspace_for(N, H, D, len(seg))
    scale = D ** -0.5

    def call(o, l, w):
        st = h3.h3_varlen_attn_fwd(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), o.data_ptr(),
                                   l.data_ptr(), tcu.data_ptr(), len(seg), 700, tpos.data_ptr(),
                                   h3.rope_cfg((32, 48, 48), 1e4), N, H, D, scale,
                                   w.data_ptr(), w.numel(),
                                   torch.cuda.current_stream().cuda_stream)
        assert st == h3.H3_OK

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(out, lse, ws)                       # first call sets the kernel attributes
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(out, lse, ws)
    # new inputs in the captured buffers, then replay
    q2, k2, v2, _, _ = synth.draw_random_case(seg, 3, 128, seed=502)
    tq.copy_(dev_bf16(q2)); tk.copy_(dev_bf16(k2)); tv.copy_(dev_bf16(v2))
    g.replay()
    torch.cuda.synchronize()
    assert h3.device_status_t(ws) == h3.H3_OK
    ref_o = torch.empty_like(out)
    ref_l = torch.empty_like(lse)
    ws2 = h3.workspace_for(N, H, D, len(seg))
    call(ref_o, ref_l, ws2)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), host_bits(ref_o))
    assert torch.equal(lse, ref_l)


def test_sage_and_qkv_graph_replay_equal_eager():
    import torch
    h3 = _h3()
    seg = [400, 77]
    q, k, v, pos, cu = synth.draw_random_case(seg, 2, 128, seed=503)
    tq, tk, tv, tcu, tpos = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(cu), dev(pos)
    N, H, D = q.shape
    ws = h3.sage_workspace_for(N, H, D, len(seg))
    o = torch.empty_like(tq)
    x, w = synth.draw_linear_case(N, 256, 3 * H * D, seed=504)
    tx, tw = dev_bf16(x), dev_bf16(w)
    outs = tuple(torch.empty((N, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    ws_g = torch.zeros(256, dtype=torch.uint8, device="cuda")

    def calls():
        h3.varlen_attn_fwd_sage_t(tq, tk, tv, tcu, 400, tpos, (32, 48, 48), 1e4, D ** -0.5,
                                  out=o, workspace=ws)
        h3.qkv_rope_gemm_t(tx, tw, H, D, tpos, (32, 48, 48), out=outs, workspace=ws_g)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    q2, k2, v2, _, _ = synth.draw_random_case(seg, 2, 128, seed=505)
    x2, _ = synth.draw_linear_case(N, 256, 3 * H * D, seed=506)
    tq.copy_(dev_bf16(q2)); tk.copy_(dev_bf16(k2)); tv.copy_(dev_bf16(v2)); tx.copy_(dev_bf16(x2))
    g.replay()
    torch.cuda.synchronize()
    got = [host_bits(o)] + [host_bits(t) for t in outs]
    calls()
    torch.cuda.synchronize()
    want = [host_bits(o)] + [host_bits(t) for t in outs]
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    assert h3.device_status_t(ws) == h3.H3_OK and h3.device_status_t(ws_g) == h3.H3_OK
