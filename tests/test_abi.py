"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, rejects bad arguments on the host before any CUDA call,
and builds positions on the host bit-identically to the oracle."""

import os
import re
import subprocess

import numpy as np
import pytest

import audio_diffusion_transformer_h3_b200 as h3
import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h3attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) == len(h3.EXPORTED)
    assert sorted(h3.EXPORTED) == names
    out = subprocess.run(["nm", "-D", "--defined-only", h3.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    for n in names:
        assert n in exported, n
        assert hasattr(h3._lib, n)


def test_status_strings():
    for s in range(8):
        assert h3.h3_status_string(s)
    assert h3.h3_status_string(99) == "unknown status"
    assert h3.h3_status_string(h3.H3_ERR_BAD_SEQLENS) == "invalid cu_seqlens"


def test_workspace_size():
    assert h3.h3_workspace_size(0, 1, 64, 1) == 256
    assert h3.h3_workspace_size(1, 1, 64, 1) == 256 + 256
    n = 78408 * 48 * 128 * 2
    assert h3.h3_workspace_size(78408, 48, 128, 2) == 256 + (n + 255) // 256 * 256


def _attn(**over):
    a = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0, cu_seqlens=0x50000, nseg=2,
             max_seqlen=80, pos=0x60000, rope=h3.rope_cfg((16, 24, 24), 1e4), N=160, H=2, D=64,
             softmax_scale=0.125, workspace=0x70000, workspace_bytes=1 << 20, stream=0)
    a.update(over)
    return h3.h3_varlen_attn_fwd(**a)


def test_attention_host_argument_errors():
    # each of these is rejected before any CUDA call (no GPU needed)
    assert _attn(D=96) == h3.H3_ERR_UNSUPPORTED
    assert _attn(D=256, rope=h3.rope_cfg((64, 96, 96), 1e4)) == h3.H3_ERR_UNSUPPORTED
    assert _attn(H=0) == h3.H3_ERR_INVALID_ARG
    assert _attn(N=-1) == h3.H3_ERR_INVALID_ARG
    assert _attn(nseg=0) == h3.H3_ERR_INVALID_ARG
    assert _attn(cu_seqlens=0) == h3.H3_ERR_INVALID_ARG
    assert _attn(q=0) == h3.H3_ERR_INVALID_ARG
    assert _attn(max_seqlen=0) == h3.H3_ERR_INVALID_ARG
    assert _attn(max_seqlen=161) == h3.H3_ERR_INVALID_ARG
    assert _attn(softmax_scale=float("nan")) == h3.H3_ERR_INVALID_ARG
    assert _attn(softmax_scale=-0.5) == h3.H3_ERR_INVALID_ARG
    assert _attn(rope=h3.rope_cfg((16, 24, 22), 1e4)) == h3.H3_ERR_INVALID_ARG   # sum != D
    assert _attn(rope=h3.rope_cfg((15, 25, 24), 1e4)) == h3.H3_ERR_INVALID_ARG   # odd width
    assert _attn(rope=h3.rope_cfg((16, 24, 24), 0.0)) == h3.H3_ERR_INVALID_ARG   # theta
    assert _attn(q=0x10008) == h3.H3_ERR_MISALIGNED
    assert _attn(o=0x40001) == h3.H3_ERR_MISALIGNED
    assert _attn(pos=0x60002) == h3.H3_ERR_MISALIGNED
    assert _attn(workspace=0) == h3.H3_ERR_WORKSPACE
    assert _attn(workspace=0x70010) == h3.H3_ERR_WORKSPACE
    assert _attn(workspace_bytes=1000) == h3.H3_ERR_WORKSPACE


def test_rope_host_argument_errors():
    cfg = h3.rope_cfg((32, 48, 48), 1e4)
    assert h3.h3_rope_apply(0x1000, 0x2000, 0x3000, 10, 4, 96, cfg, 0) == h3.H3_ERR_UNSUPPORTED
    assert h3.h3_rope_apply(0x1000, 0x2000, 0x3000, 10, 0, 128, cfg, 0) == h3.H3_ERR_INVALID_ARG
    assert h3.h3_rope_apply(0, 0x2000, 0x3000, 10, 4, 128, cfg, 0) == h3.H3_ERR_INVALID_ARG
    assert h3.h3_rope_apply(0x1004, 0x2000, 0x3000, 10, 4, 128, cfg, 0) == h3.H3_ERR_MISALIGNED
    bad = h3.rope_cfg((32, 48, 46), 1e4)
    assert h3.h3_rope_apply(0x1000, 0x2000, 0x3000, 10, 4, 128, bad, 0) == h3.H3_ERR_INVALID_ARG
    # N = 0 is a no-op that succeeds without touching the device
    assert h3.h3_rope_apply(0, 0, 0, 0, 4, 128, cfg, 0) == h3.H3_OK


@pytest.mark.parametrize("name", [w.name for w in synth.WORKLOADS])
def test_host_positions_match_oracle_bitwise(name):
    wl = synth.workload(name)
    pos, cu = h3.h3_build_positions(wl.segments)
    want = oracle.packed_positions(wl.segments)
    assert pos.dtype == np.float32 and pos.shape == want.shape
    assert np.array_equal(pos.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(cu, synth.cu_seqlens_of(wl.seg_lens))


def test_host_positions_edge_layouts():
    lays = [synth.SegmentLayout(video=(0, 0, 0)),
            synth.SegmentLayout(video=(1, 1, 1)),
            synth.SegmentLayout(video=(3, 2, 5), audio_tail=7, image_refs=2, image_grid=(2, 3),
                                audio_refs=2, audio_ref_len=5, audio_rate=3),
            synth.SegmentLayout(video=(0, 4, 4), audio_tail=0, audio_refs=1, audio_ref_len=9,
                                audio_rate=7)]
    pos, cu = h3.h3_build_positions(lays)
    want = oracle.packed_positions(lays)
    assert np.array_equal(pos.view(np.uint32), want.view(np.uint32))
    assert list(cu) == [0, 0, 1, 1 + 12 + 10 + 30 + 7, 1 + 12 + 10 + 30 + 7 + 9]


@pytest.mark.parametrize("name", ["packed", "max"])
def test_host_positions_with_clock_origins_match_oracle_bitwise(name):
    # long-video continuation: each segment's clock starts at a global origin
    wl = synth.workload(name)
    origins = [37.25 + 1000.0 * s for s in range(len(wl.segments))]
    pos, cu = h3.h3_build_positions(wl.segments, t_origins=origins)
    want = oracle.packed_positions(wl.segments, origins)
    assert np.array_equal(pos.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(cu, synth.cu_seqlens_of(wl.seg_lens))
    zero, _ = h3.h3_build_positions(wl.segments, t_origins=[0.0] * len(wl.segments))
    assert np.array_equal(zero.view(np.uint32),
                          h3.h3_build_positions(wl.segments)[0].view(np.uint32))


def test_host_positions_origin_errors():
    seg = h3.h3_segment_layout(0, 0, 0, 0, 0, 32, 2, 2, 2, 0)
    arr = (h3.h3_segment_layout * 1)(seg)
    buf = np.zeros((8, 3), np.float32)
    for bad in (float("nan"), float("inf")):
        org = np.array([bad])
        assert h3._lib.h3_build_positions_at(arr, 1, org.ctypes.data, buf.ctypes.data, 8,
                                             None) == h3.H3_ERR_INVALID_ARG
    org = np.array([5.0])
    assert h3._lib.h3_build_positions_at(arr, 1, org.ctypes.data, buf.ctypes.data, 8,
                                         None) == h3.H3_OK
    assert buf[0, 0] == 5.0 and buf[4, 0] == 6.0


def test_host_positions_errors():
    seg = h3.h3_segment_layout(0, 0, 0, 1, 4, 0, 1, 1, 1, 0)   # audio refs with rate 0
    arr = (h3.h3_segment_layout * 1)(seg)
    buf = np.zeros((16, 3), np.float32)
    assert h3._lib.h3_build_positions(arr, 1, buf.ctypes.data, 16, None) == h3.H3_ERR_INVALID_ARG
    seg = h3.h3_segment_layout(0, 0, 0, 0, 0, 32, 2, 2, 2, 0)  # 8 tokens, capacity 4
    arr = (h3.h3_segment_layout * 1)(seg)
    assert h3._lib.h3_build_positions(arr, 1, buf.ctypes.data, 4, None) == h3.H3_ERR_INVALID_ARG
    assert h3.h3_segment_tokens(h3.h3_segment_layout(-1, 0, 0, 0, 0, 0, 0, 0, 0, 0)) == -1


def test_selftest_host_argument_errors():
    assert h3.h3_selftest_bounded_wait(0, 256, 1000, 0) == h3.H3_ERR_WORKSPACE
    assert h3.h3_selftest_bounded_wait(0x10010, 256, 1000, 0) == h3.H3_ERR_WORKSPACE
    assert h3.h3_selftest_bounded_wait(0x10000, 128, 1000, 0) == h3.H3_ERR_WORKSPACE
    assert h3.h3_selftest_bounded_wait(0x10000, 256, 0, 0) == h3.H3_ERR_INVALID_ARG


def _qkv(**over):
    a = dict(x=0x10000, w=0x20000, q=0x30000, k=0x40000, v=0x50000, pos=0x60000,
             rope=h3.rope_cfg((32, 48, 48), 1e4), N=300, K=256, H=2, D=128,
             workspace=0x70000, workspace_bytes=256, stream=0)
    a.update(over)
    return h3.h3_qkv_rope_gemm(**a)


def test_qkv_gemm_host_argument_errors():
    # rejected before any CUDA call (no GPU needed)
    assert _qkv(D=96) == h3.H3_ERR_UNSUPPORTED
    assert _qkv(K=200) == h3.H3_ERR_INVALID_ARG          # K % 64 != 0
    assert _qkv(K=0) == h3.H3_ERR_INVALID_ARG
    assert _qkv(H=1, D=64, rope=h3.rope_cfg((16, 24, 24), 1e4)) == h3.H3_ERR_INVALID_ARG  # HD % 256
    assert _qkv(H=3) == h3.H3_ERR_INVALID_ARG            # HD = 384
    assert _qkv(H=0) == h3.H3_ERR_INVALID_ARG
    assert _qkv(N=-1) == h3.H3_ERR_INVALID_ARG
    assert _qkv(x=0) == h3.H3_ERR_INVALID_ARG
    assert _qkv(v=0) == h3.H3_ERR_INVALID_ARG
    assert _qkv(rope=h3.rope_cfg((32, 48, 46), 1e4)) == h3.H3_ERR_INVALID_ARG
    assert _qkv(x=0x10008) == h3.H3_ERR_MISALIGNED
    assert _qkv(k=0x40002) == h3.H3_ERR_MISALIGNED
    assert _qkv(pos=0x60002) == h3.H3_ERR_MISALIGNED
    assert _qkv(workspace=0) == h3.H3_ERR_WORKSPACE
    assert _qkv(workspace=0x70080) == h3.H3_ERR_WORKSPACE
    assert _qkv(workspace_bytes=255) == h3.H3_ERR_WORKSPACE


def _chain(**over):
    a = dict(x=0x10000, w=0x20000, q=0x30000, k=0x40000, v=0x50000, o=0x58000, lse=0x5c000,
             cu_seqlens=0x5e000, nseg=1, max_seqlen=300, pos=0x60000,
             rope=h3.rope_cfg((32, 48, 48), 1e4), N=300, K=256, H=2, D=128,
             softmax_scale=0.1, workspace=0x70000, workspace_bytes=256, stream=0)
    a.update(over)
    return h3.h3_qkv_rope_attn_fwd(**a)


def test_chained_projection_attention_host_argument_errors():
    # the attention's checks first (nothing launched), then the projection's
    assert _chain(D=96) == h3.H3_ERR_UNSUPPORTED
    assert _chain(nseg=0) == h3.H3_ERR_INVALID_ARG
    assert _chain(max_seqlen=0) == h3.H3_ERR_INVALID_ARG
    assert _chain(max_seqlen=301) == h3.H3_ERR_INVALID_ARG
    assert _chain(softmax_scale=-1.0) == h3.H3_ERR_INVALID_ARG
    assert _chain(softmax_scale=float("nan")) == h3.H3_ERR_INVALID_ARG
    assert _chain(cu_seqlens=0) == h3.H3_ERR_INVALID_ARG
    assert _chain(o=0) == h3.H3_ERR_INVALID_ARG
    assert _chain(o=0x58008) == h3.H3_ERR_MISALIGNED
    assert _chain(lse=0x5c002) == h3.H3_ERR_MISALIGNED
    assert _chain(K=200) == h3.H3_ERR_INVALID_ARG            # projection: K % 64 != 0
    assert _chain(H=3) == h3.H3_ERR_INVALID_ARG              # projection: HD % 256 != 0
    assert _chain(x=0x10008) == h3.H3_ERR_MISALIGNED
    assert _chain(workspace=0) == h3.H3_ERR_WORKSPACE
    assert _chain(workspace_bytes=255) == h3.H3_ERR_WORKSPACE


def test_sage_workspace_layout_and_host_errors():
    # status | q8 k8 v8 | s_q s_k | v_amax s_v, every region 256-aligned
    N, H, nseg = 1000, 3, 2
    up = lambda x: (x + 255) // 256 * 256
    assert h3.h3_sage_workspace_size(N, H, 128, nseg) == \
        256 + 3 * up(N * H * 128) + 2 * up(N * H * 4) + 2 * up(nseg * H * 512)
    assert h3.h3_sage_workspace_size(N, H, 64, nseg) == 0
    a = dict(q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0, cu_seqlens=0x50000, nseg=2,
             max_seqlen=80, pos=0, rope=h3.h3_rope_cfg(0, 0, 0, 0.0), N=160, H=2, D=128,
             softmax_scale=0.125, workspace=0x70000, workspace_bytes=1 << 24, stream=0)

    def call(**over):
        b = dict(a)
        b.update(over)
        return h3.h3_varlen_attn_fwd_sage(**b)
    assert call(D=64) == h3.H3_ERR_UNSUPPORTED
    assert call(nseg=0) == h3.H3_ERR_INVALID_ARG
    assert call(softmax_scale=-1.0) == h3.H3_ERR_INVALID_ARG
    assert call(max_seqlen=0) == h3.H3_ERR_INVALID_ARG
    assert call(pos=0x60000, rope=h3.rope_cfg((32, 48, 46), 1e4)) == h3.H3_ERR_INVALID_ARG
    assert call(q=0x10008) == h3.H3_ERR_MISALIGNED
    assert call(workspace_bytes=1000) == h3.H3_ERR_WORKSPACE
    assert call(workspace=0x70010) == h3.H3_ERR_WORKSPACE
