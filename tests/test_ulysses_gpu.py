"""The Ulysses head-sharded wrapper around the CUDA kernel, with two ranks.

Two processes (spawned, gloo process group) share cuda:0. Each holds a
contiguous token shard of a packed sequence of two documents; the shard
boundary falls inside the second document. ``ulysses_attention`` exchanges
the shards on the host (gloo all-to-all of bf16 tensors), each rank
runs ``varlen_attn_fwd_t`` on the GPU for its head group, and the second
all-to-all returns its tokens (gloo all-to-all carries bf16 tensors). The kernels of the two ranks do not wait on
each other (each launch is independent; the exchange is on the host). Each
rank's O and LSE must match the whole-sequence float64 oracle within the
path's tolerance (max |d| <= 2e-2, mean |d| <= 2e-3; LSE within 1e-2); with
the SAGE-style FP8 kernel as the attention step, each rank matches the
whole-sequence SAGE oracle within the same tolerance.
"""

import math
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _gpu_attn(q, k, v, cu, max_seqlen, pos, split, theta, scale, return_lse=False):
    """The attention step of the wrapper on the GPU: the host bf16 head group
    in, host tensors out."""
    import torch
    import audio_diffusion_transformer_h3_b200 as h3
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    o, lse = h3.varlen_attn_fwd_t(dq, dk, dv, cu.cuda(), max_seqlen,
                                  None if pos is None else pos.cuda(), split, theta, scale,
                                  return_lse=True)
    torch.cuda.synchronize()
    o = o.cpu()
    return (o, lse.cpu()) if return_lse else o


def _gpu_sage_attn(q, k, v, cu, max_seqlen, pos, split, theta, scale, return_lse=False):
    """The SAGE-style FP8 attention step of the wrapper on the GPU."""
    import torch
    import audio_diffusion_transformer_h3_b200 as h3
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    o, lse = h3.varlen_attn_fwd_sage_t(dq, dk, dv, cu.cuda(), max_seqlen,
                                       None if pos is None else pos.cuda(), split, theta, scale,
                                       return_lse=True)
    torch.cuda.synchronize()
    o = o.cpu()
    return (o, lse.cpu()) if return_lse else o


def _worker(rank, world, port, root, errors):
    import sys
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        torch.cuda.set_device(0)
        import oracle
        import synth
        from audio_diffusion_transformer_h3_b200.ulysses import ulysses_attention
        from gpu_util import assert_close_bf16

        seg = [700, 1350]                   # N = 2050; shard boundary 1025 inside document 1
        H, D, split = 4, 128, (32, 48, 48)
        q, k, v, pos, cu = synth.draw_random_case(seg, H, D, seed=131, pos_range=64.0)
        N = q.shape[0]
        lo, hi = rank * N // world, (rank + 1) * N // world
        scale = 1.0 / math.sqrt(D)

        def shard(bits):
            return torch.from_numpy(np.ascontiguousarray(bits[lo:hi]).view(np.int16)).view(
                torch.bfloat16)

        out, lse = ulysses_attention(shard(q), shard(k), shard(v), torch.from_numpy(cu),
                                     max(seg), torch.from_numpy(pos), split, 1e4, scale,
                                     attn=_gpu_attn, return_lse=True)
        got = out.float().numpy().astype(np.float64)
        O, L = oracle.attention_ref(q, k, v, cu, scale, pos, split, 1e4)
        assert got.shape == (hi - lo, H, D) and lse.shape == (H, hi - lo)
        assert_close_bf16(got, O[lo:hi], f"ulysses rank {rank}")
        np.testing.assert_allclose(lse.numpy(), L[:, lo:hi], rtol=0, atol=1e-2)
        # the SAGE-style FP8 kernel quantises per head (Q per token, K per 16-key
        # block from the segment start, V per segment and channel), so the head
        # split reproduces the whole-sequence SAGE reading
        out, lse = ulysses_attention(shard(q), shard(k), shard(v), torch.from_numpy(cu),
                                     max(seg), torch.from_numpy(pos), split, 1e4, scale,
                                     attn=_gpu_sage_attn, return_lse=True)
        Os, Ls = oracle.sage_attention_ref(q, k, v, cu, scale, pos, split, 1e4)
        assert_close_bf16(out.float().numpy().astype(np.float64), Os[lo:hi],
                          f"ulysses sage rank {rank}")
        np.testing.assert_allclose(lse.numpy(), Ls[:, lo:hi], rtol=0, atol=1e-2)
        dist.barrier()
    except Exception as e:  # reported to the parent
        import traceback
        errors.put(f"rank {rank}: {e!r}\n{traceback.format_exc()}")
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_ranks_on_one_gpu_match_the_whole_sequence_oracle():
    import torch.multiprocessing as mp
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    ctx = mp.get_context("spawn")
    errors = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, root, errors)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not alive, "a rank did not finish"
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)
