"""Python binding of libh3attn (include/h3attn.h).

Argument marshalling only: every step of the path runs in the CUDA library.
PyTorch supplies device memory and the current stream. The functions keep
the C names; the ``*_t`` helpers take torch tensors and call the same entry
points with their pointers.

The library is loaded from this directory (built in-tree by
``python audio_diffusion_transformer_h3_b200/build.py`` or
``__graft_entry__.build()``). There is no fallback: if it is missing or does
not load, importing this package raises.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libh3attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python audio_diffusion_transformer_h3_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- C types

H3_OK = 0
H3_ERR_INVALID_ARG = 1
H3_ERR_UNSUPPORTED = 2
H3_ERR_MISALIGNED = 3
H3_ERR_WORKSPACE = 4
H3_ERR_CUDA = 5
H3_ERR_DEVICE_TIMEOUT = 6
H3_ERR_BAD_SEQLENS = 7


class h3_rope_cfg(ctypes.Structure):
    _fields_ = [("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_w", ctypes.c_int32),
                ("theta", ctypes.c_float)]


class h3_segment_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "image_refs", "image_h", "image_w", "audio_refs", "audio_ref_len", "audio_rate",
        "video_t", "video_h", "video_w", "audio_tail")]


_c = ctypes
_P = _c.c_void_p
_lib.h3_segment_tokens.argtypes = [_c.POINTER(h3_segment_layout)]
_lib.h3_segment_tokens.restype = _c.c_int64
_lib.h3_build_positions.argtypes = [_c.POINTER(h3_segment_layout), _c.c_int32, _P, _c.c_int64, _P]
_lib.h3_build_positions.restype = _c.c_int
_lib.h3_build_positions_at.argtypes = [_c.POINTER(h3_segment_layout), _c.c_int32, _P, _P,
                                       _c.c_int64, _P]
_lib.h3_build_positions_at.restype = _c.c_int
_lib.h3_rope_apply.argtypes = [_P, _P, _P, _c.c_int64, _c.c_int32, _c.c_int32, h3_rope_cfg, _P]
_lib.h3_rope_apply.restype = _c.c_int
_lib.h3_workspace_size.argtypes = [_c.c_int64, _c.c_int32, _c.c_int32, _c.c_int32]
_lib.h3_workspace_size.restype = _c.c_size_t
_lib.h3_varlen_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _c.c_int32, _c.c_int32, _P,
                                    h3_rope_cfg, _c.c_int64, _c.c_int32, _c.c_int32,
                                    _c.c_float, _P, _c.c_size_t, _P]
_lib.h3_varlen_attn_fwd.restype = _c.c_int
_lib.h3_varlen_attn_fwd_static.argtypes = [_P, _P, _P, _P, _P, _P, _c.c_int32, _c.c_int32, _P,
                                           h3_rope_cfg, _c.c_int64, _c.c_int32, _c.c_int32,
                                           _c.c_float, _P]
_lib.h3_varlen_attn_fwd_static.restype = _c.c_int
_lib.h3_varlen_attn_fwd_skip.argtypes = [_P, _P, _P, _P, _P, _P, _c.c_int32, _c.c_int32, _P,
                                         h3_rope_cfg, _c.c_int64, _c.c_int32, _c.c_int32,
                                         _c.c_float, _c.c_float, _P, _c.c_size_t, _P]
_lib.h3_varlen_attn_fwd_skip.restype = _c.c_int
_lib.h3_sage_workspace_size.argtypes = [_c.c_int64, _c.c_int32, _c.c_int32, _c.c_int32]
_lib.h3_sage_workspace_size.restype = _c.c_size_t
_lib.h3_varlen_attn_fwd_sage.argtypes = [_P, _P, _P, _P, _P, _P, _c.c_int32, _c.c_int32, _P,
                                         h3_rope_cfg, _c.c_int64, _c.c_int32, _c.c_int32,
                                         _c.c_float, _P, _c.c_size_t, _P]
_lib.h3_varlen_attn_fwd_sage.restype = _c.c_int
_lib.h3_qkv_rope_gemm.argtypes = [_P, _P, _P, _P, _P, _P, h3_rope_cfg, _c.c_int64, _c.c_int32,
                                  _c.c_int32, _c.c_int32, _P, _c.c_size_t, _P]
_lib.h3_qkv_rope_gemm.restype = _c.c_int
_lib.h3_qkv_rope_attn_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _c.c_int32, _c.c_int32,
                                      _P, h3_rope_cfg, _c.c_int64, _c.c_int32, _c.c_int32,
                                      _c.c_int32, _c.c_float, _P, _c.c_size_t, _P]
_lib.h3_qkv_rope_attn_fwd.restype = _c.c_int
_lib.h3_read_skip_count.argtypes = [_P, _P, _c.POINTER(_c.c_uint64)]
_lib.h3_read_skip_count.restype = _c.c_int
_lib.h3_selftest_bounded_wait.argtypes = [_P, _c.c_size_t, _c.c_int64, _P]
_lib.h3_selftest_bounded_wait.restype = _c.c_int
_lib.h3_read_device_status.argtypes = [_P, _P]
_lib.h3_read_device_status.restype = _c.c_int
_lib.h3_status_string.argtypes = [_c.c_int]
_lib.h3_status_string.restype = _c.c_char_p
_lib.h3_last_cuda_error.argtypes = []
_lib.h3_last_cuda_error.restype = _c.c_int32

EXPORTED = ("h3_segment_tokens", "h3_build_positions", "h3_build_positions_at", "h3_rope_apply", "h3_workspace_size",
            "h3_varlen_attn_fwd", "h3_varlen_attn_fwd_skip", "h3_read_skip_count",
            "h3_qkv_rope_gemm", "h3_qkv_rope_attn_fwd", "h3_sage_workspace_size",
            "h3_varlen_attn_fwd_sage",
            "h3_varlen_attn_fwd_static", "h3_selftest_bounded_wait",
            "h3_read_device_status", "h3_status_string", "h3_last_cuda_error")

# Scratch bytes compiled into the library for h3_varlen_attn_fwd_static
# (H3_STATIC_WORKSPACE_BYTES in include/h3attn.h).
H3_STATIC_WORKSPACE_BYTES = 256 + (64 << 20)


class H3Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = h3_status_string(status)
        if status == H3_ERR_CUDA:
            msg += f" (cudaError {h3_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str) -> None:
    if status != H3_OK:
        raise H3Error(status, where)


def rope_cfg(split: Sequence[int], theta: float) -> h3_rope_cfg:
    return h3_rope_cfg(int(split[0]), int(split[1]), int(split[2]), float(theta))


# -------------------------------------------------------- raw C entry points

def h3_status_string(status: int) -> str:
    return _lib.h3_status_string(int(status)).decode()


def h3_last_cuda_error() -> int:
    return int(_lib.h3_last_cuda_error())


def h3_segment_tokens(layout: h3_segment_layout) -> int:
    return int(_lib.h3_segment_tokens(ctypes.byref(layout)))


def h3_workspace_size(N: int, H: int, D: int, nseg: int) -> int:
    return int(_lib.h3_workspace_size(N, H, D, nseg))


def h3_rope_apply(x: int, out: int, pos: int, N: int, H: int, D: int,
                  rope: h3_rope_cfg, stream: int) -> int:
    return int(_lib.h3_rope_apply(x, out, pos, N, H, D, rope, stream))


def h3_varlen_attn_fwd(q: int, k: int, v: int, o: int, lse: int, cu_seqlens: int, nseg: int,
                       max_seqlen: int, pos: int, rope: h3_rope_cfg, N: int, H: int, D: int,
                       softmax_scale: float, workspace: int, workspace_bytes: int,
                       stream: int) -> int:
    return int(_lib.h3_varlen_attn_fwd(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos, rope,
                                       N, H, D, softmax_scale, workspace, workspace_bytes,
                                       stream))


def h3_varlen_attn_fwd_skip(q: int, k: int, v: int, o: int, lse: int, cu_seqlens: int,
                            nseg: int, max_seqlen: int, pos: int, rope: h3_rope_cfg, N: int,
                            H: int, D: int, softmax_scale: float, skip_threshold: float,
                            workspace: int, workspace_bytes: int, stream: int) -> int:
    return int(_lib.h3_varlen_attn_fwd_skip(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos,
                                            rope, N, H, D, softmax_scale, skip_threshold,
                                            workspace, workspace_bytes, stream))


def h3_sage_workspace_size(N: int, H: int, D: int, nseg: int) -> int:
    return int(_lib.h3_sage_workspace_size(N, H, D, nseg))


def h3_varlen_attn_fwd_sage(q: int, k: int, v: int, o: int, lse: int, cu_seqlens: int,
                            nseg: int, max_seqlen: int, pos: int, rope: h3_rope_cfg, N: int,
                            H: int, D: int, softmax_scale: float, workspace: int,
                            workspace_bytes: int, stream: int) -> int:
    return int(_lib.h3_varlen_attn_fwd_sage(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen, pos,
                                            rope, N, H, D, softmax_scale, workspace,
                                            workspace_bytes, stream))


def h3_qkv_rope_gemm(x: int, w: int, q: int, k: int, v: int, pos: int, rope: h3_rope_cfg,
                     N: int, K: int, H: int, D: int, workspace: int, workspace_bytes: int,
                     stream: int) -> int:
    return int(_lib.h3_qkv_rope_gemm(x, w, q, k, v, pos, rope, N, K, H, D, workspace,
                                     workspace_bytes, stream))


def h3_qkv_rope_attn_fwd(x: int, w: int, q: int, k: int, v: int, o: int, lse: int,
                         cu_seqlens: int, nseg: int, max_seqlen: int, pos: int,
                         rope: h3_rope_cfg, N: int, K: int, H: int, D: int,
                         softmax_scale: float, workspace: int, workspace_bytes: int,
                         stream: int) -> int:
    return int(_lib.h3_qkv_rope_attn_fwd(x, w, q, k, v, o, lse, cu_seqlens, nseg, max_seqlen,
                                         pos, rope, N, K, H, D, softmax_scale, workspace,
                                         workspace_bytes, stream))


def h3_read_skip_count(workspace: int, stream: int) -> int:
    n = ctypes.c_uint64(0)
    _check(_lib.h3_read_skip_count(workspace, stream, ctypes.byref(n)), "h3_read_skip_count")
    return int(n.value)


def h3_varlen_attn_fwd_static(q: int, k: int, v: int, o: int, lse: int, cu_seqlens: int,
                              nseg: int, max_seqlen: int, pos: int, rope: h3_rope_cfg, N: int,
                              H: int, D: int, softmax_scale: float, stream: int) -> int:
    """h3_varlen_attn_fwd without a caller workspace: for hosts that cannot
    allocate device memory, the library's own compiled-in scratch is used
    (N*H*D <= 2^25; calls on one device must not overlap on the GPU)."""
    return int(_lib.h3_varlen_attn_fwd_static(q, k, v, o, lse, cu_seqlens, nseg, max_seqlen,
                                              pos, rope, N, H, D, softmax_scale, stream))


def h3_selftest_bounded_wait(workspace: int, workspace_bytes: int, limit_cycles: int,
                             stream: int) -> int:
    return int(_lib.h3_selftest_bounded_wait(workspace, workspace_bytes, limit_cycles, stream))


def h3_read_device_status(workspace: int, stream: int) -> int:
    return int(_lib.h3_read_device_status(workspace, stream))


def h3_build_positions(layouts, t_origins=None):
    """Host position build. ``layouts``: objects with the attributes of
    ``h3_segment_layout`` (or of a segment description with ``video``,
    ``audio_tail``, ``image_refs``, ``image_grid``, ``audio_refs``,
    ``audio_ref_len``, ``audio_rate``); ``t_origins``: optional clock origin
    per segment (h3_build_positions_at). Returns (pos float32 [N, 3],
    cu_seqlens int32 [nseg + 1]) as NumPy arrays."""
    import numpy as np
    segs = (h3_segment_layout * max(1, len(layouts)))()
    for i, l in enumerate(layouts):
        segs[i] = to_c_layout(l)
    total = sum(max(0, h3_segment_tokens(segs[i])) for i in range(len(layouts)))
    pos = np.zeros((max(total, 1), 3), dtype=np.float32)
    cu = np.zeros(len(layouts) + 1, dtype=np.int32)
    if t_origins is None:
        st = _lib.h3_build_positions(segs, len(layouts), pos.ctypes.data, total,
                                     cu.ctypes.data)
    else:
        org = np.ascontiguousarray(t_origins, dtype=np.float64)
        if org.shape != (len(layouts),):
            raise ValueError("one clock origin per segment")
        st = _lib.h3_build_positions_at(segs, len(layouts), org.ctypes.data,
                                        pos.ctypes.data, total, cu.ctypes.data)
    _check(st, "h3_build_positions")
    return pos[:total], cu


def to_c_layout(l) -> h3_segment_layout:
    if isinstance(l, h3_segment_layout):
        return l
    T, Hg, Wg = l.video
    ih, iw = l.image_grid
    return h3_segment_layout(l.image_refs, ih, iw, l.audio_refs, l.audio_ref_len, l.audio_rate,
                             T, Hg, Wg, l.audio_tail)


# ------------------------------------------------------ torch tensor helpers

def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _thd(x, name):
    import torch
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 3 and x.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA bfloat16 tensor [N, H, D]")
    return x


def rope_apply_t(x, pos, split, theta: float = 10000.0, out=None, stream=None):
    """out = RoPE(x, pos) through h3_rope_apply. x bf16 [N, H, D], pos fp32 [N, 3]."""
    import torch
    _thd(x, "x")
    if out is None:
        out = torch.empty_like(x)
    N, H, D = x.shape
    _check(h3_rope_apply(x.data_ptr(), out.data_ptr(), pos.data_ptr(), N, H, D,
                         rope_cfg(split, theta), _stream(stream)), "h3_rope_apply")
    return out


def workspace_for(N: int, H: int, D: int, nseg: int, device=None):
    import torch
    n = h3_workspace_size(N, H, D, nseg)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def varlen_attn_fwd_t(q, k, v, cu_seqlens, max_seqlen: int, pos=None, split=None,
                      theta: float = 10000.0, softmax_scale: Optional[float] = None,
                      out=None, return_lse: bool = False, workspace=None, stream=None):
    """O (and LSE [H, N] if asked) through h3_varlen_attn_fwd."""
    import torch
    _thd(q, "q"); _thd(k, "k"); _thd(v, "v")
    N, H, D = q.shape
    nseg = int(cu_seqlens.numel()) - 1
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device=q.device) if return_lse else None
    if workspace is None:
        workspace = workspace_for(N, H, D, nseg, q.device)
    scale = (1.0 / math.sqrt(D)) if softmax_scale is None else float(softmax_scale)
    rope = rope_cfg(split, theta) if pos is not None else h3_rope_cfg(0, 0, 0, 0.0)
    st = h3_varlen_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr() if lse is not None else 0,
                            cu_seqlens.data_ptr(), nseg, int(max_seqlen),
                            pos.data_ptr() if pos is not None else 0, rope, N, H, D, scale,
                            workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(st, "h3_varlen_attn_fwd")
    return (out, lse) if return_lse else out


def varlen_attn_fwd_skip_t(q, k, v, cu_seqlens, max_seqlen: int, skip_threshold: float,
                           pos=None, split=None, theta: float = 10000.0,
                           softmax_scale: Optional[float] = None, out=None,
                           return_lse: bool = False, workspace=None, stream=None):
    """Skip-softmax variant through h3_varlen_attn_fwd_skip; the number of
    skipped (32-row block, key tile) pairs is read with skip_count_t(workspace)."""
    import torch
    _thd(q, "q"); _thd(k, "k"); _thd(v, "v")
    N, H, D = q.shape
    nseg = int(cu_seqlens.numel()) - 1
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device=q.device) if return_lse else None
    if workspace is None:
        workspace = workspace_for(N, H, D, nseg, q.device)
    scale = (1.0 / math.sqrt(D)) if softmax_scale is None else float(softmax_scale)
    rope = rope_cfg(split, theta) if pos is not None else h3_rope_cfg(0, 0, 0, 0.0)
    st = h3_varlen_attn_fwd_skip(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr() if lse is not None else 0,
                                 cu_seqlens.data_ptr(), nseg, int(max_seqlen),
                                 pos.data_ptr() if pos is not None else 0, rope, N, H, D, scale,
                                 float(skip_threshold), workspace.data_ptr(), workspace.numel(),
                                 _stream(stream))
    _check(st, "h3_varlen_attn_fwd_skip")
    return (out, lse) if return_lse else out


def qkv_rope_gemm_t(x, w, heads: int, head_dim: int, pos=None, split=None,
                    theta: float = 10000.0, out=None, workspace=None, stream=None):
    """(q, k, v) [N, H, D] bf16 through h3_qkv_rope_gemm: the projection
    x [N, K] @ w[3*H*D, K]^T with RoPE applied to q and k in its epilogue."""
    import torch
    for t, name in ((x, "x"), (w, "w")):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 2 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 matrix")
    N, K = x.shape
    if tuple(w.shape) != (3 * heads * head_dim, K):
        raise ValueError(f"w must be [3*H*D, K] = [{3 * heads * head_dim}, {K}]")
    if out is None:
        out = tuple(torch.empty((N, heads, head_dim), dtype=torch.bfloat16, device=x.device)
                    for _ in range(3))
    q, k, v = out
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=x.device)
    rope = rope_cfg(split, theta) if pos is not None else h3_rope_cfg(0, 0, 0, 0.0)
    st = h3_qkv_rope_gemm(x.data_ptr(), w.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                          pos.data_ptr() if pos is not None else 0, rope, N, K, heads,
                          head_dim, workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(st, "h3_qkv_rope_gemm")
    return q, k, v


def qkv_rope_attn_fwd_t(x, w, heads: int, head_dim: int, cu_seqlens, max_seqlen: int,
                        pos=None, split=None, theta: float = 10000.0,
                        softmax_scale: Optional[float] = None, qkv=None, out=None,
                        return_lse: bool = False, workspace=None, stream=None):
    """O (and LSE [H, N] if asked) of attention over the projection x w^T,
    through h3_qkv_rope_attn_fwd: q and k are rotated in the projection's
    epilogue and the attention reads them as they are. ``qkv`` receives the
    projection ([N, H, D] bf16 each; allocated if None)."""
    import torch
    for t, name in ((x, "x"), (w, "w")):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 2 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 matrix")
    N, K = x.shape
    if tuple(w.shape) != (3 * heads * head_dim, K):
        raise ValueError(f"w must be [3*H*D, K] = [{3 * heads * head_dim}, {K}]")
    if qkv is None:
        qkv = tuple(torch.empty((N, heads, head_dim), dtype=torch.bfloat16, device=x.device)
                    for _ in range(3))
    q, k, v = qkv
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _thd(t, name)
    if out is None:
        out = torch.empty_like(q)
    lse = (torch.empty((heads, N), dtype=torch.float32, device=x.device) if return_lse
           else None)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=x.device)
    nseg = int(cu_seqlens.numel()) - 1
    scale = (1.0 / math.sqrt(head_dim)) if softmax_scale is None else float(softmax_scale)
    rope = rope_cfg(split, theta) if pos is not None else h3_rope_cfg(0, 0, 0, 0.0)
    st = h3_qkv_rope_attn_fwd(x.data_ptr(), w.data_ptr(), q.data_ptr(), k.data_ptr(),
                              v.data_ptr(), out.data_ptr(),
                              lse.data_ptr() if lse is not None else 0, cu_seqlens.data_ptr(),
                              nseg, int(max_seqlen), pos.data_ptr() if pos is not None else 0,
                              rope, N, K, heads, head_dim, scale, workspace.data_ptr(),
                              workspace.numel(), _stream(stream))
    _check(st, "h3_qkv_rope_attn_fwd")
    return (out, lse) if return_lse else out


def sage_workspace_for(N: int, H: int, D: int, nseg: int, device=None):
    import torch
    n = h3_sage_workspace_size(N, H, D, nseg)
    if n == 0:
        raise ValueError("the SAGE variant supports head dim 128 only")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sage_workspace_views(workspace, N: int, H: int, nseg: int) -> dict:
    """Views of the regions h3_varlen_attn_fwd_sage leaves in its workspace
    (layout of h3_sage_workspace_size in include/h3attn.h): q8, k8, v8 uint8
    [N, H, 128]; s_q, s_k float32 [H, N]; v_amax, s_v float32 [nseg, H, 128]."""
    import torch

    def up(x):
        return (x + 255) // 256 * 256
    codes, scales, vsc = up(N * H * 128), up(N * H * 4), up(nseg * H * 128 * 4)
    off = {"q8": 256}
    off["k8"] = off["q8"] + codes
    off["v8"] = off["k8"] + codes
    off["s_q"] = off["v8"] + codes
    off["s_k"] = off["s_q"] + scales
    off["v_amax"] = off["s_k"] + scales
    off["s_v"] = off["v_amax"] + vsc
    out = {}
    for name in ("q8", "k8", "v8"):
        out[name] = workspace[off[name]:off[name] + N * H * 128].view(N, H, 128)
    for name in ("s_q", "s_k"):
        out[name] = workspace[off[name]:off[name] + N * H * 4].view(torch.float32).view(H, N)
    for name in ("v_amax", "s_v"):
        out[name] = workspace[off[name]:off[name] + nseg * H * 512].view(torch.float32) \
            .view(nseg, H, 128)
    return out


def varlen_attn_fwd_sage_t(q, k, v, cu_seqlens, max_seqlen: int, pos=None, split=None,
                           theta: float = 10000.0, softmax_scale: Optional[float] = None,
                           out=None, return_lse: bool = False, workspace=None, stream=None):
    """SAGE-style FP8 variant through h3_varlen_attn_fwd_sage (head dim 128)."""
    import torch
    _thd(q, "q"); _thd(k, "k"); _thd(v, "v")
    N, H, D = q.shape
    nseg = int(cu_seqlens.numel()) - 1
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device=q.device) if return_lse else None
    if workspace is None:
        workspace = sage_workspace_for(N, H, D, nseg, q.device)
    scale = (1.0 / math.sqrt(D)) if softmax_scale is None else float(softmax_scale)
    rope = rope_cfg(split, theta) if pos is not None else h3_rope_cfg(0, 0, 0, 0.0)
    st = h3_varlen_attn_fwd_sage(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr() if lse is not None else 0,
                                 cu_seqlens.data_ptr(), nseg, int(max_seqlen),
                                 pos.data_ptr() if pos is not None else 0, rope, N, H, D, scale,
                                 workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(st, "h3_varlen_attn_fwd_sage")
    return (out, lse) if return_lse else out


def skip_count_t(workspace, stream=None) -> int:
    """Skipped (32-row block, key tile) pairs of the last skip call on ``workspace`` (syncs)."""
    return h3_read_skip_count(workspace.data_ptr(), _stream(stream))


def device_status_t(workspace, stream=None) -> int:
    """Device status word of the last call that used ``workspace`` (syncs)."""
    return h3_read_device_status(workspace.data_ptr(), _stream(stream))
