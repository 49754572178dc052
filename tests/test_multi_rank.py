"""Multi-rank paths on CPU with the gloo backend (world size 2).

* bench.py's weak-scaling plumbing: per-rank seeds give independent batches,
  the timed region is the maximum over ranks, and the job value counts every
  rank's FLOPs.
* The Ulysses head-sharded wrapper: each rank holds a contiguous token shard
  of a packed sequence (the shard boundary falls inside a document); the two
  all-to-alls around the attention must reproduce, on each rank's tokens,
  the attention of the whole packed sequence. The attention step is the
  float64 oracle here (dense, then the SAGE-style FP8 reading), so this
  checks the data movement exactly.
"""

import math
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_attn(q, k, v, cu, max_seqlen, pos, split, theta, scale, return_lse=False):
    import torch
    import oracle
    O, L = oracle.attention_ref(q.numpy(), k.numpy(), v.numpy(), cu.numpy(), scale,
                                None if pos is None else pos.numpy(), split, theta)
    O, L = torch.from_numpy(O), torch.from_numpy(L)
    return (O, L) if return_lse else O


def _sage_oracle_attn(q, k, v, cu, max_seqlen, pos, split, theta, scale, return_lse=False):
    import torch
    import oracle
    O, L = oracle.sage_attention_ref(q.numpy(), k.numpy(), v.numpy(), cu.numpy(), scale,
                                     None if pos is None else pos.numpy(), split, theta)
    O, L = torch.from_numpy(O), torch.from_numpy(L)
    return (O, L) if return_lse else O


def _worker(rank, world, port, root, errors):
    import sys
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bench
        import oracle
        import synth
        from audio_diffusion_transformer_h3_b200.ulysses import ulysses_attention

        # --- bench plumbing
        got = bench.max_over_ranks(1.5 + 3.0 * rank, world)
        assert got == 1.5 + 3.0 * (world - 1), got
        seeds = [bench.rank_seed(1004, r) for r in range(world)]
        assert len(set(seeds)) == world
        wl = synth.workload("tiny")
        mine = synth.draw_qkv(wl, seed=bench.rank_seed(wl.the_seed, rank))[0]
        other = synth.draw_qkv(wl, seed=bench.rank_seed(wl.the_seed, 1 - rank))[0]
        assert not np.array_equal(mine, other)
        assert bench.job_tflops(world, 1e12, 10, 1000.0) == world * 10.0

        # --- Ulysses wrapper against the whole-sequence oracle
        seg = [20, 44]                      # N = 64, shard boundary at 32 inside segment 1
        H, D, split = 4, 8, (2, 4, 2)
        q, k, v, pos, cu = synth.draw_random_case(seg, H, D, seed=77, pos_range=16.0)
        Q, K, V = (torch.from_numpy(oracle.bf16_bits_to_f64(x)) for x in (q, k, v))
        N = Q.shape[0]
        lo, hi = rank * N // world, (rank + 1) * N // world
        scale = 1.0 / math.sqrt(D)
        out, lse = ulysses_attention(Q[lo:hi].contiguous(), K[lo:hi].contiguous(),
                                     V[lo:hi].contiguous(), torch.from_numpy(cu), max(seg),
                                     torch.from_numpy(pos), split, 1e4, scale,
                                     attn=_oracle_attn, return_lse=True)
        O, L = oracle.attention_ref(Q.numpy(), K.numpy(), V.numpy(), cu, scale, pos, split, 1e4)
        assert out.shape == (hi - lo, H, D) and lse.shape == (H, hi - lo)
        np.testing.assert_allclose(out.numpy(), O[lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse.numpy(), L[:, lo:hi], rtol=0, atol=1e-12)
        # the SAGE-style FP8 attention quantises per head (Q per token, K per 16-key
        # block, V per segment and channel), so head sharding reproduces it exactly
        out, lse = ulysses_attention(Q[lo:hi].contiguous(), K[lo:hi].contiguous(),
                                     V[lo:hi].contiguous(), torch.from_numpy(cu), max(seg),
                                     torch.from_numpy(pos), split, 1e4, scale,
                                     attn=_sage_oracle_attn, return_lse=True)
        Os, Ls = oracle.sage_attention_ref(Q.numpy(), K.numpy(), V.numpy(), cu, scale, pos,
                                           split, 1e4)
        np.testing.assert_allclose(out.numpy(), Os[lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse.numpy(), Ls[:, lo:hi], rtol=0, atol=1e-12)
        # heads that do not split over the ranks are refused
        with pytest.raises(ValueError):
            ulysses_attention(Q[lo:hi, :3].contiguous(), K[lo:hi, :3].contiguous(),
                              V[lo:hi, :3].contiguous(), torch.from_numpy(cu), max(seg),
                              torch.from_numpy(pos), split, 1e4, scale, attn=_oracle_attn)
        dist.barrier()
    except Exception as e:  # reported to the parent
        import traceback
        errors.put(f"rank {rank}: {e!r}\n{traceback.format_exc()}")
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_bench_plumbing_and_ulysses_wrapper():
    import torch.multiprocessing as mp
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    ctx = mp.get_context("spawn")
    errors = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, root, errors)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    msgs = []
    while not errors.empty():
        msgs.append(errors.get())
    assert not alive, "a rank did not finish"
    assert not msgs, "\n".join(msgs)
    assert all(p.exitcode == 0 for p in procs)


def test_ulysses_without_a_process_group_is_one_rank():
    # no torch.distributed group: the wrapper is the attention call itself
    import torch
    import oracle
    import synth
    from audio_diffusion_transformer_h3_b200.ulysses import ulysses_attention
    q, k, v, pos, cu = synth.draw_random_case([30, 34], 2, 8, seed=78, pos_range=16.0)
    Q, K, V = (torch.from_numpy(oracle.bf16_bits_to_f64(x)) for x in (q, k, v))
    out = ulysses_attention(Q, K, V, torch.from_numpy(cu), 34, torch.from_numpy(pos), (2, 4, 2),
                            1e4, 0.3, attn=_oracle_attn)
    O, _ = oracle.attention_ref(Q.numpy(), K.numpy(), V.numpy(), cu, 0.3, pos, (2, 4, 2), 1e4)
    np.testing.assert_allclose(out.numpy(), O, rtol=0, atol=0)
