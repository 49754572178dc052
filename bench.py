"""Benchmark: fused RoPE + packed varlen joint attention forward, TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload max] [--impl ours|reference]

One step = one h3_varlen_attn_fwd call over the whole packed workload
(rotary pass over k, then the attention kernel, which rotates each query tile
as it loads it). FLOPs = sum over segments of 4 L^2 H D (QK^T and PV,
non-causal). Inputs are seeded synthetic bf16 tensors shaped like the
workload (each larger than L2, so no flush is needed between steps).

Multi-GPU (torchrun, one process per GPU): every rank runs its own packed
workload (different seed) with no data-path collective: weak scaling. The
only collectives are the barrier and the max over ranks of the timed region.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload (the reference arm); under torchrun only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "fused RoPE+varlen joint attention fwd TFLOP/s and % of B200 BF16 peak"
UNIT = "TFLOP/s"
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = ["audio_diffusion_transformer_h3_b200/csrc/attn_fwd.cuh",
                  "audio_diffusion_transformer_h3_b200/csrc/sm100.cuh",
                  "audio_diffusion_transformer_h3_b200/csrc/rope.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16": float(d["bf16_tflops"]), "bf16_sustained": float(d["bf16_tflops_sustained"]),
                "hbm": float(d["hbm_gbs"]), "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary
    ``profiles/attn_fwd_<workload>_traffic.txt`` (``key: value`` lines), or
    None if it is missing or was taken on a different kernel source."""
    p = os.path.join(PROFILE_DIR, f"attn_fwd_{workload}_traffic.txt")
    if not os.path.exists(p):
        return None
    rec = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.lstrip().startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return int(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self) -> dict:
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                maxs.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


def workload_config(wl) -> dict:
    return {"workload": wl.name, "description": wl.description, "tokens": wl.n_tokens,
            "segments": wl.seg_lens, "heads": wl.heads, "head_dim": wl.head_dim,
            "rope_split": list(wl.split), "theta": wl.theta, "causal": False,
            "l2": "each input tensor exceeds the 126 MB L2; no flush between steps"
            if wl.n_tokens * wl.heads * wl.head_dim * 2 > 126e6 else
            "L2 flushed (256 MB write) before every timed step"}


# ---------------------------------------------------------- multi-rank helpers

def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s own packed workload (weak scaling: every rank
    draws an independent batch of the same shape)."""
    return base_seed + 7919 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of ``x`` over all ranks (the timed region is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU oracle

def host_cpu() -> dict:
    """The machine the CPU baseline ran on: logical CPUs (os.cpu_count()) and
    the model name that lscpu reports."""
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        model = None
    return {"host_cpu_count": os.cpu_count(), "cpu_model": model}


def cpu_oracle_sample(wl, q, k, v, pos, cu, budget_s: float):
    """Time the float64 oracle on (head, 128-row block) units of the workload
    until ``budget_s`` seconds are spent. Returns (TFLOP/s, description, threads)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    rng = np.random.default_rng(7)
    flops = 0.0
    units = 0
    t0 = time.perf_counter()
    while True:
        s = int(rng.integers(0, len(cu) - 1))
        a, e = int(cu[s]), int(cu[s + 1])
        h = int(rng.integers(0, wl.heads))
        r0 = int(rng.integers(a, max(a + 1, e - 128)))
        rows = np.arange(r0, min(e, r0 + 128))
        oracle.attention_rows_ref(q, k, v, cu, wl.softmax_scale, rows, [h], pos, wl.split, wl.theta)
        flops += 4.0 * len(rows) * (e - a) * wl.head_dim
        units += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"{units} units of (1 head, up to 128 query rows) against their full segment, "
            f"random over the workload's segments and heads; {flops:.3g} FLOP in {dt:.1f} s")
    return flops / dt / 1e12, desc, threads


# -------------------------------------------------------------------- arms

def run_reference(args, wl, rank, world):
    if rank != 0:
        return 0
    q, k, v = synth.draw_qkv(wl)
    import oracle
    pos = oracle.packed_positions(wl.segments)
    cu = synth.cu_seqlens_of(wl.seg_lens)
    budget = min(args.ref_step_seconds, max(1.0, 90.0 / (args.steps + args.warmup / 4.0)))
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, q, k, v, pos, cu, budget / 4)
    vals = []
    desc, threads = "", 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        val, desc, threads = cpu_oracle_sample(wl, q, k, v, pos, cu, budget)
        vals.append(val)
    total = time.perf_counter() - t0
    value = float(np.mean(vals))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, bf16 inputs widened to float64)",
            "config": workload_config(wl), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": desc, "blas_threads": threads, **host_cpu(),
                             "ms_per_step_covers": "the sampled units of one step only "
                                                   "(a bounded sample, not the whole workload)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import audio_diffusion_transformer_h3_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    seed = rank_seed(wl.the_seed, rank)
    q, k, v = synth.draw_qkv(wl, seed=seed)
    pos, cu = h3.h3_build_positions(wl.segments)
    N, H, D = wl.n_tokens, wl.heads, wl.head_dim
    nseg = len(wl.seg_lens)
    flops_step = wl.flops()

    def pinned_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

    hq, hk, hv = pinned_bf16(q), pinned_bf16(k), pinned_bf16(v)
    hpos = torch.from_numpy(pos).pin_memory()
    hcu = torch.from_numpy(cu).pin_memory()
    ho = torch.empty((N, H, D), dtype=torch.bfloat16).pin_memory()
    del q, k, v

    dq, dk, dv = hq.to(dev), hk.to(dev), hv.to(dev)
    dpos, dcu = hpos.to(dev), hcu.to(dev)
    do = torch.empty_like(dq)
    ws = h3.workspace_for(N, H, D, nseg, dev)
    stream = torch.cuda.current_stream(dev)
    flush = None
    if N * H * D * 2 <= 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        if flush is not None:
            flush.zero_()
        h3.varlen_attn_fwd_t(dq, dk, dv, dcu, wl.max_seqlen, dpos, wl.split, wl.theta,
                             wl.softmax_scale, out=do, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = h3.device_status_t(ws)
    if st != h3.H3_OK:
        raise RuntimeError(f"device status {h3.h3_status_string(st)}")

    # ---- device-timed region: inputs resident in HBM ----
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier()
    torch.cuda.synchronize()
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    smi_id = visible[local_rank] if local_rank < len(visible) else str(local_rank)
    with ClockSampler(smi_id) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev)
    if h3.device_status_t(ws) != h3.H3_OK:
        raise RuntimeError("device status not ok after timed region")
    value = job_tflops(world, flops_step, args.steps, total_ms)
    mean_step_ms = float(np.mean(step_ms))

    # ---- end-to-end through the public API with host buffers ----
    # (skipped with --no-e2e, which profiling runs use to keep device memory low)
    def run_e2e():
        # Every step copies its inputs from pinned host memory and reads its
        # result back. Serial: copy in, compute, copy out on one stream. Pipelined
        # (the reported e2e): two device slots; step i+1's inputs go up on an H2D
        # stream and step i-1's output comes down on a D2H stream while step i's
        # kernels run, with events ordering slot reuse.
        h2d = hq.numel() * 2 * 3 + hpos.numel() * 4 + hcu.numel() * 4
        d2h = ho.numel() * 2

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            dpos.copy_(hpos, non_blocking=True)
            dcu.copy_(hcu, non_blocking=True)
            h3.varlen_attn_fwd_t(dq, dk, dv, dcu, wl.max_seqlen, dpos, wl.split, wl.theta,
                                 wl.softmax_scale, out=do, workspace=ws, stream=stream)
            ho.copy_(do, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

        slots = [dict(q=dq, k=dk, v=dv, pos=dpos, cu=dcu, o=do, ws=ws, ho=ho),
                 dict(q=torch.empty_like(dq), k=torch.empty_like(dk), v=torch.empty_like(dv),
                      pos=torch.empty_like(dpos), cu=torch.empty_like(dcu), o=torch.empty_like(do),
                      ws=h3.workspace_for(N, H, D, nseg, dev), ho=torch.empty_like(ho).pin_memory())]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def pipelined(n_steps, start_event):
            ev_in = [torch.cuda.Event() for _ in range(2)]
            ev_done = [None, None]      # step's kernels done (inputs and o free to reuse)
            ev_out = [None, None]       # step's output read back
            up.wait_event(start_event)

            def upload(i):
                sl = slots[i & 1]
                with torch.cuda.stream(up):
                    if ev_done[i & 1] is not None:
                        up.wait_event(ev_done[i & 1])
                    sl["q"].copy_(hq, non_blocking=True)
                    sl["k"].copy_(hk, non_blocking=True)
                    sl["v"].copy_(hv, non_blocking=True)
                    sl["pos"].copy_(hpos, non_blocking=True)
                    sl["cu"].copy_(hcu, non_blocking=True)
                    ev_in[i & 1].record(up)

            upload(0)
            for i in range(n_steps):
                sl = slots[i & 1]
                stream.wait_event(ev_in[i & 1])
                if ev_out[i & 1] is not None:
                    stream.wait_event(ev_out[i & 1])
                h3.varlen_attn_fwd_t(sl["q"], sl["k"], sl["v"], sl["cu"], wl.max_seqlen, sl["pos"],
                                     wl.split, wl.theta, wl.softmax_scale, out=sl["o"],
                                     workspace=sl["ws"], stream=stream)
                done = torch.cuda.Event()
                done.record(stream)
                ev_done[i & 1] = done
                if i + 1 < n_steps:
                    upload(i + 1)
                with torch.cuda.stream(down):
                    down.wait_event(done)
                    sl["ho"].copy_(sl["o"], non_blocking=True)
                    out = torch.cuda.Event()
                    out.record(down)
                    ev_out[i & 1] = out
            stream.wait_stream(down)
            stream.wait_stream(up)

        start = torch.cuda.Event()
        start.record(stream)
        pipelined(2, start)                 # warm-up of the pipeline
        torch.cuda.synchronize()
        barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        pipelined(args.steps, p0)
        p1.record(stream)
        torch.cuda.synchronize()
        barrier()
        for sl in slots:
            if h3.device_status_t(sl["ws"]) != h3.H3_OK:
                raise RuntimeError("device status not ok after the end-to-end steps")
        e2e_ms = max_over_ranks(p0.elapsed_time(p1), world, dev)
        e2e_value = job_tflops(world, flops_step, args.steps, e2e_ms)
        e2e_serial_value = job_tflops(world, flops_step, args.steps, e2e_serial_ms)
        return e2e_value, e2e_serial_value, e2e_ms, e2e_serial_ms, h2d, d2h

    e2e_res = None if args.no_e2e else run_e2e()

    peaks = measured_peaks()
    achieved = flops_step / (mean_step_ms * 1e-3) / 1e12
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded bf16 ~N(0,1) q/k/v, fp32 positions on the shared clock)",
        "config": workload_config(wl),
        "pct_of_bf16_peak": {"burst_measured": 100 * achieved / peaks["bf16"],
                             "sustained_measured": 100 * achieved / peaks["bf16_sustained"],
                             "datasheet_2250": 100 * achieved / 2250.0},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16"],
                     "peak_kind": f"bf16 dense, burst ({peaks['source']})",
                     "traffic": recorded_traffic(wl.name),
                     "kernel": "attn_fwd_kernel<128> (step = k rotary pass + attention kernel)"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if e2e_res is not None:
        e2e_value, e2e_serial_value, e2e_ms, e2e_serial_ms, h2d, d2h = e2e_res
        line["e2e"] = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                       "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms / args.steps,
                       "mode": "pipelined: step i+1's host->device copy and step i-1's "
                               "device->host copy overlap step i's kernels (two device slots)",
                       "serial_value": e2e_serial_value,
                       "serial_ms_per_step": e2e_serial_ms / args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle  # CPU baseline leg only
        def host_bits(t):
            return t.view(torch.int16).numpy().view(np.uint16)
        opos = oracle.packed_positions(wl.segments)
        val, desc, threads = cpu_oracle_sample(wl, host_bits(hq), host_bits(hk), host_bits(hv),
                                               opos, cu, args.cpu_seconds)
        line["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc, "blas_threads": threads, **host_cpu()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_skip(args, wl, rank, world, local_rank):
    """Skip-softmax variant on inputs with frame-group locality (one group per
    1008-token frame, synth.draw_group_case): dense-equivalent TFLOP/s (the
    dense FLOPs over the time of the skip call), the skipped share of
    (32-row block, key tile) pairs, and the dense kernel's time on the same
    inputs for comparison. Single process only."""
    import torch

    import audio_diffusion_transformer_h3_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    q, k, v, cu = synth.draw_group_case(wl.seg_lens, wl.heads, wl.head_dim, group_len=1008,
                                        amp=15.0, eps=0.05, seed=rank_seed(wl.the_seed, rank))
    pos, _ = h3.h3_build_positions(wl.segments)
    N, H, D = wl.n_tokens, wl.heads, wl.head_dim

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    dq, dk, dv, dcu = bf(q), bf(k), bf(v), torch.from_numpy(cu).to(dev)
    do = torch.empty_like(dq)
    ws = h3.workspace_for(N, H, D, len(wl.seg_lens), dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    # no RoPE here: the group codes are the locality structure
    ms_skip = timed(lambda: h3.varlen_attn_fwd_skip_t(dq, dk, dv, dcu, wl.max_seqlen,
                                                      args.skip_threshold, None, None, wl.theta,
                                                      wl.softmax_scale, out=do, workspace=ws,
                                                      stream=stream))
    skipped = h3.skip_count_t(ws)
    ms_dense = timed(lambda: h3.varlen_attn_fwd_t(dq, dk, dv, dcu, wl.max_seqlen, None, None,
                                                  wl.theta, wl.softmax_scale, out=do,
                                                  workspace=ws, stream=stream))
    pairs = sum(((L + 31) // 32) * ((L + 127) // 128 - 1) for L in wl.seg_lens) * H
    line = {"metric": "skip-softmax fused varlen joint attention fwd, dense-equivalent TFLOP/s",
            "value": wl.flops() / (ms_skip * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_skip,
            "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic frame-group locality (synth.draw_group_case, 1008-token groups)",
            "config": workload_config(wl), "skip_threshold": args.skip_threshold,
            "skipped_fraction": skipped / pairs, "dense_ms_same_inputs": ms_dense,
            "speedup_vs_dense": ms_dense / ms_skip, "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)
    return 0


def run_sage(args, wl, rank, world, local_rank):
    """SAGE-style FP8 variant (h3_varlen_attn_fwd_sage) on the workload's
    seeded N(0,1) inputs and positions: dense-equivalent TFLOP/s (the dense
    FLOPs over the time of the FP8 call, its two quantisation passes
    included), the dense kernel on the same inputs, the distance between the
    two outputs, and two rooflines: the FP8 tensor peak (twice the measured
    bf16 one, the nominal ratio) and the exponential unit (16 ex2 per clock
    per SM at the sampled SM clock; one exponential per score, half of
    them on that unit and half on the FMA pipe; the last, partly masked key
    tile of a segment runs all of its exponentials on that unit, which the
    count ignores). Single process only."""
    import torch

    import audio_diffusion_transformer_h3_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    q, k, v = synth.draw_qkv(wl, seed=rank_seed(wl.the_seed, rank))
    pos, cu = h3.h3_build_positions(wl.segments)
    N, H, D = wl.n_tokens, wl.heads, wl.head_dim

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    dq, dk, dv = bf(q), bf(k), bf(v)
    dpos, dcu = torch.from_numpy(pos).to(dev), torch.from_numpy(cu).to(dev)
    o_s, o_d = torch.empty_like(dq), torch.empty_like(dq)
    ws_s = h3.sage_workspace_for(N, H, D, len(wl.seg_lens), dev)
    ws_d = h3.workspace_for(N, H, D, len(wl.seg_lens), dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    with ClockSampler(str(local_rank)) as clocks:
        ms = timed(lambda: h3.varlen_attn_fwd_sage_t(dq, dk, dv, dcu, wl.max_seqlen, dpos,
                                                     wl.split, wl.theta, wl.softmax_scale,
                                                     out=o_s, workspace=ws_s, stream=stream))
    assert h3.device_status_t(ws_s) == h3.H3_OK
    ms_dense = timed(lambda: h3.varlen_attn_fwd_t(dq, dk, dv, dcu, wl.max_seqlen, dpos,
                                                  wl.split, wl.theta, wl.softmax_scale,
                                                  out=o_d, workspace=ws_d, stream=stream))
    diff = (o_s.float() - o_d.float()).abs()
    achieved = wl.flops() / (ms * 1e-3) / 1e12
    peaks = measured_peaks()
    ck = clocks.summary()
    exps = float(sum(L * L for L in wl.seg_lens)) * H
    xu_peak = 16 * 148 * (ck["sm_mhz"] or 1965.0) * 1e6
    line = {"metric": "SAGE-style FP8 fused varlen joint attention fwd, dense-equivalent TFLOP/s",
            "value": achieved, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "e4m3 (Q, K, P, V), fp32 accumulate", "data": "synthetic (synth.draw_qkv)",
            "config": workload_config(wl),
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": 2 * peaks["bf16_sustained"], "unit": "TFLOP/s",
                         "frac": achieved / (2 * peaks["bf16_sustained"]),
                         "peak_kind": "fp8 dense = 2 x measured bf16 sustained"},
            "roofline_xu": {"achieved_ex2_per_s": 0.5 * exps / (ms * 1e-3),
                            "peak_ex2_per_s": xu_peak,
                            "frac": 0.5 * exps / (ms * 1e-3) / xu_peak,
                            "note": "16 ex2/clk/SM x 148 SMs at the sampled SM clock"},
            "dense_ms_same_inputs": ms_dense, "speedup_vs_dense": ms_dense / ms,
            "vs_dense_kernel": {"max_abs": float(diff.max()), "mean_abs": float(diff.mean())},
            "gpu_launches": 3 * args.steps, "clocks": ck}
    print(json.dumps(line), flush=True)
    return 0


def run_qkv(args, wl, rank, world, local_rank):
    """The QKV projection with RoPE fused into its epilogue (h3_qkv_rope_gemm)
    on the DiT's shape (hidden 5376 -> 3 x 56 heads x 128) over the tokens and
    positions of workload ``wl``. Reports TFLOP/s (2 N K 3HD per call) against
    the measured bf16 peaks, and the unfused alternative with the same
    kernels: the projection without rotation followed by the standalone
    rotary pass over q and k. Inputs (X alone is N*5376*2 bytes) exceed L2.
    Single process only."""
    import torch

    import audio_diffusion_transformer_h3_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    p = synth.QKV_PROJECTION
    N, K, H, D = wl.n_tokens, p.hidden, p.heads, p.head_dim
    x_bits, w_bits = synth.draw_linear_case(N, K, p.out_features, seed=rank_seed(90, rank))
    pos, _ = h3.h3_build_positions(wl.segments)

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    x, w = bf(x_bits), bf(w_bits)
    del x_bits, w_bits
    dpos = torch.from_numpy(pos).to(dev)
    out = tuple(torch.empty((N, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    def fused():
        h3.qkv_rope_gemm_t(x, w, H, D, dpos, p.split, p.theta, out=out, workspace=ws,
                           stream=stream)

    def unfused():
        h3.qkv_rope_gemm_t(x, w, H, D, None, None, out=out, workspace=ws, stream=stream)
        h3.rope_apply_t(out[0], dpos, p.split, p.theta, out=out[0], stream=stream)
        h3.rope_apply_t(out[1], dpos, p.split, p.theta, out=out[1], stream=stream)

    with ClockSampler(str(local_rank)) as clocks:
        ms = timed(fused)
    assert h3.device_status_t(ws) == h3.H3_OK
    ms_unfused = timed(unfused)
    flops = 2.0 * N * K * p.out_features
    achieved = flops / (ms * 1e-3) / 1e12
    peaks = measured_peaks()
    line = {"metric": "QKV projection with fused RoPE epilogue, TFLOP/s",
            "value": achieved, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (synth.draw_linear_case, x ~ N(0,1), "
                                     "w ~ N(0,1/K); positions of the workload)",
            "config": {"workload": f"qkv projection {N}x{K} -> 3x{H}x{D} "
                                   f"({wl.name} workload tokens)",
                       "tokens": N, "hidden": K, "heads": H, "head_dim": D,
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_sustained"],
                         "peak_kind": f"bf16 dense, sustained ({peaks['source']})",
                         "frac_of_burst": achieved / peaks["bf16"]},
            "unfused_ms": ms_unfused, "fusion_speedup": ms_unfused / ms,
            "gpu_launches": args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_qkv_attend(args, wl, rank, world, local_rank):
    """The chained product path (h3_qkv_rope_attn_fwd) on workload ``wl``:
    the QKV projection x [N, 5376] @ w^T (the DiT's hidden size, the
    workload's heads) with q and k rotated in its epilogue, then the
    attention on the rotated q and k with no key pass. Reports the chain's
    TFLOP/s (projection 2 N K 3HD plus attention 4 L^2 H D per segment) and,
    on the same data, the projection alone, the attention alone without
    positions, and the dense line (key rotation pass + attention with fused
    query rotation) on unrotated q, k, v. Single process only."""
    import torch

    import audio_diffusion_transformer_h3_b200 as h3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    K = synth.QKV_PROJECTION.hidden
    N, H, D = wl.n_tokens, wl.heads, wl.head_dim
    x_bits, w_bits = synth.draw_linear_case(N, K, 3 * H * D, seed=rank_seed(91, rank))
    pos, cu = h3.h3_build_positions(wl.segments)

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    x, w = bf(x_bits), bf(w_bits)
    del x_bits, w_bits
    dpos, dcu = torch.from_numpy(pos).to(dev), torch.from_numpy(cu).to(dev)
    qkv = tuple(torch.empty((N, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    raw = tuple(torch.empty((N, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    o = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    ws_dense = h3.workspace_for(N, H, D, len(wl.seg_lens), dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    def chain():
        h3.qkv_rope_attn_fwd_t(x, w, H, D, dcu, wl.max_seqlen, dpos, wl.split, wl.theta,
                               wl.softmax_scale, qkv=qkv, out=o, workspace=ws, stream=stream)

    with ClockSampler(str(local_rank)) as clocks:
        ms = timed(chain)
    assert h3.device_status_t(ws) == h3.H3_OK
    ms_proj = timed(lambda: h3.qkv_rope_gemm_t(x, w, H, D, dpos, wl.split, wl.theta, out=qkv,
                                               workspace=ws, stream=stream))
    ms_attn = timed(lambda: h3.varlen_attn_fwd_t(*qkv, dcu, wl.max_seqlen, None, None,
                                                 wl.theta, wl.softmax_scale, out=o,
                                                 workspace=ws, stream=stream))
    h3.qkv_rope_gemm_t(x, w, H, D, None, None, out=raw, workspace=ws, stream=stream)
    ms_dense = timed(lambda: h3.varlen_attn_fwd_t(*raw, dcu, wl.max_seqlen, dpos, wl.split,
                                                  wl.theta, wl.softmax_scale, out=o,
                                                  workspace=ws_dense, stream=stream))
    assert h3.device_status_t(ws_dense) == h3.H3_OK
    f_proj = 2.0 * N * K * 3 * H * D
    f_attn = wl.flops()
    peaks = measured_peaks()
    achieved = (f_proj + f_attn) / (ms * 1e-3) / 1e12
    line = {"metric": "QKV projection with fused RoPE epilogue chained into varlen joint "
                      "attention fwd, TFLOP/s",
            "value": achieved, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (synth.draw_linear_case: x ~ N(0,1), "
                                     "w ~ N(0,1/K); positions of the workload)",
            "config": {**workload_config(wl), "hidden": K,
                       "workload": f"{wl.name}: qkv projection {N}x{K} -> 3x{H}x{D}, then "
                                   "attention"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                         "unit": "TFLOP/s", "frac": achieved / peaks["bf16"],
                         "peak_kind": f"bf16 dense, burst ({peaks['source']})"},
            "projection_ms": ms_proj,
            "attention_no_key_pass_ms": ms_attn,
            "attention_no_key_pass_tflops": f_attn / (ms_attn * 1e-3) / 1e12,
            "dense_line_ms_same_data": ms_dense,
            "dense_line_tflops_same_data": f_attn / (ms_dense * 1e-3) / 1e12,
            "gpu_launches": 2 * args.steps, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_ulysses(args, wl, rank, world, local_rank):
    """The Ulysses head-sharded path ("MiniMax H3" vLLM-Omni recipe, section
    "Four GPUs: throughput-oriented combined service": --usp 4): one packed
    workload is split into contiguous token shards, one per rank; each step
    runs ulysses_attention (all-to-all sequence -> heads over NCCL, the fused
    RoPE + varlen attention on H/P heads of the whole sequence, all-to-all
    back). Strong scaling: the job processes one workload per step whatever
    the number of ranks. With one rank the wrapper is the kernel call."""
    import torch
    import torch.distributed as dist

    import audio_diffusion_transformer_h3_b200 as h3
    from audio_diffusion_transformer_h3_b200.ulysses import ulysses_attention

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    N, H, D = wl.n_tokens, wl.heads, wl.head_dim
    if N % world or H % world:
        raise ValueError(f"{N} tokens and {H} heads must split over {world} ranks")
    q, k, v = synth.draw_qkv(wl)
    pos, cu = h3.h3_build_positions(wl.segments)
    lo, hi = rank * N // world, (rank + 1) * N // world

    def shard(bits):
        return torch.from_numpy(np.ascontiguousarray(bits[lo:hi]).view(np.int16)).view(
            torch.bfloat16).to(dev)

    dq, dk, dv = shard(q), shard(k), shard(v)
    del q, k, v
    dpos, dcu = torch.from_numpy(pos).to(dev), torch.from_numpy(cu).to(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ulysses_attention(dq, dk, dv, dcu, wl.max_seqlen, dpos, wl.split, wl.theta,
                                 wl.softmax_scale)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    smi_id = visible[local_rank] if local_rank < len(visible) else str(local_rank)
    with ClockSampler(smi_id) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    value = wl.flops() * args.steps / (total_ms * 1e-3) / 1e12
    peaks = measured_peaks()
    per_gpu = value / world
    exchanged = 4 * N * H * D * 2 * (world - 1) / world ** 2 if world > 1 else 0
    line = {"metric": METRIC + " (Ulysses head-sharded, one workload across the ranks)",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded bf16 ~N(0,1) q/k/v, fp32 positions)",
            "config": {**workload_config(wl), "parallelism": f"ulysses{world}"},
            "roofline": {"bound": "tensor", "achieved": per_gpu, "peak": peaks["bf16"],
                         "unit": "TFLOP/s per GPU", "frac": per_gpu / peaks["bf16"],
                         "peak_kind": f"bf16 dense, burst ({peaks['source']})"},
            "all_to_all_bytes_per_rank_per_step": exchanged,
            "gpu_launches": 2 * args.steps, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="max")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (profiling runs: less device memory)")
    ap.add_argument("--skip-threshold", type=float, default=None,
                    help="time the skip-softmax variant on frame-group inputs instead")
    ap.add_argument("--sage", action="store_true",
                    help="time the SAGE-style FP8 variant instead")
    ap.add_argument("--qkv-proj", action="store_true",
                    help="time the QKV projection with the fused RoPE epilogue instead")
    ap.add_argument("--ulysses", action="store_true",
                    help="time the Ulysses head-sharded path (one workload over the ranks)")
    ap.add_argument("--attend", action="store_true",
                    help="with --qkv-proj: time the projection chained into the attention")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.workload(args.workload)

    if args.impl == "reference":
        return run_reference(args, wl, rank, world)
    if args.skip_threshold is not None:
        return run_skip(args, wl, rank, world, local_rank)
    if args.qkv_proj and args.attend:
        return run_qkv_attend(args, wl, rank, world, local_rank)
    if args.qkv_proj:
        return run_qkv(args, wl, rank, world, local_rank)
    if args.sage:
        return run_sage(args, wl, rank, world, local_rank)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.ulysses:
            return run_ulysses(args, wl, rank, world, local_rank)
        return run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
