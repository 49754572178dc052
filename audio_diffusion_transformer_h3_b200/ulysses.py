"""Ulysses (head-sharded) sequence parallelism around the single-GPU kernel.

"MiniMax H3" vLLM-Omni recipe, section "Four GPUs: throughput-oriented
combined service" (``--usp 4 --ring 1``), and "Day 0 Support for MiniMax-H3
on AMD Instinct GPUs" (Ulysses parallelism splits the joint spatiotemporal
sequence across GPUs): each of P ranks holds a contiguous N/P-token shard of
the packed sequence with all H heads. One all-to-all turns that into all N
tokens for H/P heads, the unchanged fused RoPE + varlen attention runs on
those heads (cu_seqlens and positions are global, so packed documents and
the shared clock are untouched), and a second all-to-all returns each rank's
tokens with all heads. Ring attention (splitting K/V) is not used: the pages
report that it does not preserve packed padding boundaries.

Communication per rank: 3 N H D (P-1)/P^2 elements in, N H D (P-1)/P^2 out.
The collectives are torch.distributed all_to_all_single (NCCL over NVLink on
B200 ranks; gloo on CPU in the tests).
"""

from __future__ import annotations

from typing import Callable, Optional


def _seq_to_heads(x, world: int, group):
    """[N/P, H, D] on every rank -> [N, H/P, D] (this rank's head group)."""
    import torch
    import torch.distributed as dist
    n_local, H, D = x.shape
    hp = H // world
    send = x.reshape(n_local, world, hp, D).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[s] = tokens of rank s, heads of this rank's group
    return recv.reshape(world * n_local, hp, D)


def _heads_to_seq(y, world: int, group):
    """[N, H/P, D] (this rank's head group) -> [N/P, H, D] (this rank's tokens)."""
    import torch
    import torch.distributed as dist
    N, hp, D = y.shape
    n_local = N // world
    send = y.reshape(world, n_local, hp, D).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[r] = this rank's tokens, heads of group r
    return recv.permute(1, 0, 2, 3).reshape(n_local, world * hp, D)


def _lse_heads_to_seq(lse, world: int, group):
    """[H/P, N] -> [H, N/P] for this rank's tokens."""
    import torch
    import torch.distributed as dist
    hp, N = lse.shape
    n_local = N // world
    send = lse.reshape(hp, world, n_local).permute(1, 0, 2).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.reshape(world * hp, n_local)


def ulysses_attention(q, k, v, cu_seqlens, max_seqlen: int, pos=None, split=None,
                      theta: float = 10000.0, softmax_scale: Optional[float] = None,
                      group=None, attn: Optional[Callable] = None, return_lse: bool = False):
    """Head-sharded fused RoPE + varlen attention over P ranks.

    q, k, v: this rank's [N/P, H, D] token shard (rank r holds tokens
    [r N/P, (r+1) N/P) of the packed sequence). cu_seqlens [nseg+1] and pos
    [N, 3] are global (the same on every rank). Requires N and H divisible by
    the group size (one rank when no process group is initialised). ``attn``
    defaults to the CUDA kernel
    (``varlen_attn_fwd_t``); it is called as
    ``attn(q, k, v, cu_seqlens, max_seqlen, pos, split, theta, softmax_scale,
    return_lse=...)`` on [N, H/P, D] tensors. Returns O [N/P, H, D] (and LSE
    [H, N/P] if asked).
    """
    import torch.distributed as dist
    # without an initialised process group the caller is a single rank
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    n_local, H, D = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    if attn is None:
        from . import varlen_attn_fwd_t as attn
    if world == 1:
        return attn(q, k, v, cu_seqlens, max_seqlen, pos, split, theta, softmax_scale,
                    return_lse=return_lse)
    qh = _seq_to_heads(q, world, group)
    kh = _seq_to_heads(k, world, group)
    vh = _seq_to_heads(v, world, group)
    out = attn(qh, kh, vh, cu_seqlens, max_seqlen, pos, split, theta, softmax_scale,
               return_lse=return_lse)
    if return_lse:
        oh, lse = out
        return _heads_to_seq(oh, world, group), _lse_heads_to_seq(lse, world, group)
    return _heads_to_seq(out, world, group)
