"""Benchmark of the lightning-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_n131k|prefill_n16k] [--no-extras]

A step is one la_prefill call over the long-context workload (B=1, H=64,
N=131072, D=128, beta=128, bf16 inputs, fp32 accumulation, no output norm),
with Q/K/V/O (8.6 GB) resident in HBM.  The inputs are far larger than the
126 MB L2, so no flush is needed between steps.  ``value`` is prefill
tokens/s over all ranks; the JSON line also carries the tensor-core view
(TFLOP/s, % of bf16 peak), the decode step (B=256, H=64, D=128, fp32 state of a
seeded N=4096 prefill; tokens/s and % of HBM bandwidth), the roofline of the
prefill kernel, the end-to-end number through the C ABI with host buffers, a
sweep of the sequence length at a fixed token count, and the fp64 oracle timed on
the host cores as a CPU baseline.

Multi-GPU (torchrun): the heads are independent units, so N ranks run a layer of
64 N heads, 64 heads per rank, with no data-path collective (weak scaling); the
timed region is bracketed by barriers and the slowest rank's time is reported.
The ``lasp`` key adds LASP+ sequence parallelism (strong scaling): one sequence
of N=131072 tokens split into N contiguous chunks, with one all-gather of the
chunk states between the chunk-state and the prefill kernels.

``--impl reference`` times the fp64 CPU oracle on the same metric and unit,
each step a bounded sample of the workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s & TFLOP/s (% bf16 peak); decode tokens/s (% HBM BW)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # name: (B, N, H, D, beta)
    "prefill_n131k": (1, 131072, 64, 128, 128),
    "prefill_n16k": (1, 16384, 64, 128, 128),
    "prefill_n16k_b64": (1, 16384, 64, 128, 64),
}
DECODE = dict(B=256, H=64, D=128, N=4096, steps=64, chunk=32)
KERNEL_SOURCES = [os.path.join(ROOT, "long_context_04_b200", "csrc", f)
                  for f in ("prefill_pair.cuh", "prefill_tc.cuh", "la_device.cuh")]
PREFILL_KERNEL = "la::prefill_pair_kernel (beta=128, D=128)"


# ----------------------------------------------------------------------------- helpers
def tiled_flops_per_token_head(D: int, beta: int) -> int:
    """Tiled-form flops per token and head: 2*beta*D (QK^T) + 2*beta*D (PV) + 2*D*D (Q.KV)
    + 2*D*D (K^T V), with beta x beta score blocks counted in full."""
    return 4 * beta * D + 4 * D * D


def useful_flops_per_token_head(D: int, beta: int) -> float:
    """Causally useful flops: on average (beta+1)/2 keys per query inside a block."""
    return 2 * D * (beta + 1) + 4 * D * D


def prefill_bytes(T: int, H: int, D: int) -> int:
    """Algorithmic HBM bytes of one prefill: read Q, K, V and write O, bf16."""
    return 8 * T * H * D


def decode_bytes(B: int, H: int, D: int) -> int:
    """Per step: fp32 state read + write (8 D^2) and bf16 q, k, v, o (8 D) per (b, h)."""
    return B * H * (8 * D * D + 8 * D)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_digest(paths) -> str:
    """sha256 over the kernel's source files (the record is void once any of them changes)."""
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_record(kernel_srcs):
    """DRAM bytes per token-head from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "prefill_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("source_sha256") == kernel_digest(kernel_srcs):
            return rec
    except (OSError, ValueError):
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than guess
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    _NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
              0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
              0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
              0x100: "display_clock_setting"}

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self._NAMES.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- distributed
def dist_init():
    """(rank, world, local_rank) from the torchrun environment; single process otherwise."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_setup(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_max(x: float, world: int, device=None) -> float:
    """Maximum of a float over all ranks (every rank calls this in the same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(D: int, heads: int, tokens: int, seed: int = 0):
    """A bounded sample of the workload for the fp64 oracle: `heads` heads x `tokens` tokens
    (the first tokens of the sequence), drawn with the same recipe as the GPU inputs."""
    import torch

    from long_context_04_b200 import synth
    q, k, v = synth.qkv(tokens, heads, D, seed=seed, dtype=torch.bfloat16, device="cpu")
    return q, k, v


def time_oracle_prefill(q, k, v, nthreads: int) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v, want_o=True, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_baseline(B, N, H, D, beta, budget_s=12.0):
    """fp64 oracle (recurrent form, the cheapest exact form) on the host cores.

    Calibrates on a small sample, then times `cores` heads x L tokens sized for about
    `budget_s` of wall time.  The value is in the metric's unit: tokens of the H-head
    layer per second = (sampled tokens x sampled heads / H) / time."""
    cores = max(1, os.cpu_count() or 1)
    heads = min(H, cores)
    q, k, v = oracle_sample(D, heads, 1024)
    t = time_oracle_prefill(q, k, v, heads)
    per_token = max(t / 1024.0, 1e-7)
    L = int(max(1024, min(N, budget_s / per_token)))
    L = (L // 1024) * 1024
    q, k, v = oracle_sample(D, heads, L, seed=1)
    t = time_oracle_prefill(q, k, v, heads)
    value = L * heads / H / t
    return {"value": value, "unit": "tokens/s", "cores": heads, "kind": "oracle",
            "sample": f"fp64 recurrent form, {heads} heads x {L} tokens of the N={N} "
                      f"sequence ({heads}/{H} of the heads), {t:.1f} s on {heads} threads; "
                      f"value = sampled token-heads / {H} / time",
            "seconds": t}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_init()
    if rank != 0:
        return 0
    B, N, H, D, beta = WORKLOADS[args.workload]
    cores = max(1, os.cpu_count() or 1)
    heads = min(H, cores)
    q, k, v = oracle_sample(D, heads, 1024)
    per_token = max(time_oracle_prefill(q, k, v, heads) / 1024.0, 1e-7)
    budget = 150.0 / max(1, args.steps + args.warmup)
    L = int(max(256, min(N, budget / per_token)))
    q, k, v = oracle_sample(D, heads, L, seed=1)
    for _ in range(args.warmup):
        time_oracle_prefill(q, k, v, heads)
    times = [time_oracle_prefill(q, k, v, heads) for _ in range(args.steps)]
    total = sum(times)
    value = args.steps * L * heads / H / total
    sample = (f"per step: fp64 recurrent oracle on {heads} heads x {L} tokens of the {args.workload} "
              f"workload, {heads} threads; value = sampled token-heads / {H} / time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.workload), "global_batch": B, "seq_len": N,
                   "heads": H, "head_dim": D, "beta": beta, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": heads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_name(w: str) -> str:
    B, N, H, D, beta = WORKLOADS[w]
    return (f"lightning-attention causal prefill, B={B}, N={N}, H={H}, D={D}, beta={beta}, "
            f"bf16 in / fp32 accumulate, no output norm")


# ----------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch

    from long_context_04_b200 import api, build as lib_build, synth

    rank, world, local = dist_init()
    if world > 1:
        torch.cuda.set_device(local)
        dist_setup(world, "nccl")
    dev = torch.device("cuda", torch.cuda.current_device())
    lib_build.build()
    api.lib()

    B, N, H, D, beta = WORKLOADS[args.workload]
    T = B * N
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.Stream(device=dev)

    with torch.cuda.stream(stream):
        q, k, v = synth.qkv(T, H, D, seed=rank, dtype=torch.bfloat16, device=dev)
        q, k, v = (x.view(B, N, H, D) for x in (q, k, v))
        o = torch.empty_like(q)
    stream.synchronize()

    def step():
        api.prefill(q, k, v, beta=beta, out=o, stream=stream)

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    status = api.device_status(stream)
    if status != api.LA_OK:
        raise RuntimeError(f"device status after warm-up: {api.status_string(status)}")

    # ---- timed region: K prefill launches, per-launch events on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    dist_barrier(world)
    local_ms = t_begin.elapsed_time(t_end)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = dist_max(local_ms, world, dev)
    status = api.device_status(stream)
    if status != api.LA_OK:
        raise RuntimeError(f"device status after timing: {api.status_string(status)}")

    tokens_total = T * world * args.steps
    value = tokens_total / (ms / 1e3)
    ms_per_step = ms / args.steps
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    flops = tiled_flops_per_token_head(D, beta) * T * H
    useful = useful_flops_per_token_head(D, beta) * T * H
    alg_bytes = prefill_bytes(T, H, D)
    tflops = flops / avg_launch_s / 1e12
    hbm_gbs = alg_bytes / avg_launch_s / 1e9
    peak_bw = float(peaks["hbm_gbs"])
    peak_tf = float(peaks["bf16_tflops"])
    trec = traffic_record(KERNEL_SOURCES)
    traffic = None
    if trec is not None:
        traffic = float(trec["bytes_per_launch_per_token_head"]) * T * H
    roofline = {"bound": "hbm", "achieved": hbm_gbs, "peak": peak_bw, "unit": "GB/s",
                "frac": hbm_gbs / peak_bw, "traffic": traffic,
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": alg_bytes,
                "kernel": PREFILL_KERNEL}
    prefill_view = {"tflops_tiled": tflops, "pct_bf16_peak": 100.0 * tflops / peak_tf,
                    "tflops_causal_useful": useful / avg_launch_s / 1e12,
                    "bf16_peak_tflops": peak_tf,
                    "roofline_ceiling_tflops": min(peak_tf, flops / alg_bytes * peak_bw / 1e3),
                    "avg_launch_ms": avg_launch_s * 1e3,
                    "launch_ms_min_median_max": [min(launch_ms), statistics.median(launch_ms),
                                                 max(launch_ms)],
                    "flops_per_token_head": tiled_flops_per_token_head(D, beta)}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: Q, K, V iid N(0,1)/sqrt(D), seeded per head shard (rank)",
        "config": {"workload": workload_name(args.workload), "global_batch": B,
                   "seq_len": N, "heads": H, "head_dim": D, "beta": beta,
                   "heads_total": H * world,
                   "parallelism": (f"heads sharded x{world}: a layer of {H * world} heads, "
                                   f"{H} per rank, no collective" if world > 1 else
                                   "one GPU, no collective"),
                   "l2": "inputs (8.6 GB) larger than the 126 MB L2; no flush"},
        "prefill": prefill_view, "roofline": roofline, "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }

    if not args.no_extras:
        line["e2e"] = e2e_prefill(args, api, torch, q, k, v, B, N, H, D, beta, world, dev)
        line["decode"], dctx = bench_decode(api, synth, torch, dev, stream, peak_bw, rank, world)
        line["concurrent"] = bench_concurrent(api, torch, stream, dctx, q, k, v, o, beta, world)
        if rank == 0 and world == 1:  # the host baseline is a 1-GPU figure
            try:
                line["decode"]["cpu_baseline"] = decode_cpu_baseline(torch, dctx)
            except Exception as e:  # an extra that fails must not cost the main line
                line["decode"]["cpu_baseline"] = {"error": repr(e)}
        del dctx
        line["lasp_chunk_state"] = bench_chunk_state(api, torch, stream, k, v, peak_bw, world)
        if world > 1:   # every rank must reach the same collectives: no local recovery
            line["lasp"] = lasp_leg(api, torch, stream, q, k, v, o, rank, world, peak_bw, dev)
        else:
            try:
                line["lasp"] = lasp_leg(api, torch, stream, q, k, v, o, rank, world, peak_bw, dev)
            except Exception as e:  # an extra that fails must not cost the main line
                line["lasp"] = {"error": repr(e)}
        if world == 1:  # rank-local extra: no collective, so a failure cannot strand other ranks
            try:
                line["length_sweep"] = bench_length_sweep(api, torch, stream, q, k, v, o, beta, peak_bw)
            except Exception as e:  # an extra that fails must not cost the main line
                line["length_sweep"] = {"error": repr(e)}
            try:
                line["prefill_options"] = bench_prefill_options(api, torch, stream, q, k, v, o, peak_bw)
            except Exception as e:
                line["prefill_options"] = {"error": repr(e)}
            try:
                line["headline_repeat"] = bench_headline_repeat(api, torch, stream, q, k, v, o, beta,
                                                                peak_bw, torch.cuda.current_device())
            except Exception as e:
                line["headline_repeat"] = {"error": repr(e)}
            try:
                line["configs"] = bench_configs(api, synth, torch, stream, dev, peaks, cpu=(rank == 0))
            except Exception as e:
                line["configs"] = {"error": repr(e)}
    if rank == 0 and world == 1 and not args.no_extras:  # the host baseline is a 1-GPU figure
        line["cpu_baseline"] = cpu_baseline(B, N, H, D, beta)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def e2e_prefill(args, api, torch, q, k, v, B, N, H, D, beta, world, dev):
    """Same metric through the C ABI with host buffers: each step copies Q, K, V from pinned
    host memory, runs la_prefill and copies O back to pinned host memory."""
    steps = 3
    hq, hk, hv = (x.to("cpu").pin_memory() for x in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    s = torch.cuda.Stream(device=dev)
    dq, dk, dv, do = (torch.empty_like(q) for _ in range(4))

    def one():
        with torch.cuda.stream(s):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            api.prefill(dq, dk, dv, beta=beta, out=do, stream=s)
            ho.copy_(do, non_blocking=True)

    one()
    s.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    e0.record(s)
    for _ in range(steps):
        one()
    e1.record(s)
    s.synchronize()
    dist_barrier(world)
    ms = dist_max(e0.elapsed_time(e1), world, dev)
    nbytes = q.numel() * q.element_size()
    del dq, dk, dv, do
    return {"value": B * N * world * steps / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes, "steps": steps,
            "note": "pinned host Q/K/V -> device, la_prefill, device O -> pinned host; one stream"}


def bench_decode(api, synth, torch, dev, pstream, peak_bw, rank, world):
    """Decode step B=256, H=64, D=128 on its own stream; state from seeded N=4096 prefills
    (8 chunks of 32 sequences, handed over with la_state_out)."""
    B, H, D, N, steps, chunk = (DECODE[x] for x in ("B", "H", "D", "N", "steps", "chunk"))
    state = torch.empty(B, H, D, D, device=dev)
    with torch.cuda.stream(pstream):
        for c in range(B // chunk):
            q, k, v = synth.qkv(chunk * N, H, D, seed=100 + c + 1000 * rank, dtype=torch.bfloat16,
                                device=dev)
            q, k, v = (x.view(chunk, N, H, D) for x in (q, k, v))
            _, ws = api.prefill(q, k, v, beta=128, return_state=True, stream=pstream)
            slots = torch.arange(c * chunk, (c + 1) * chunk, dtype=torch.int32, device=dev)
            api.state_out(ws, state, slots, stream=pstream)
            del q, k, v, ws
    pstream.synchronize()
    dstream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(dstream):
        toks = [synth.decode_tokens(B, H, D, step=t, seed=rank, device=dev) for t in range(steps)]
        outs = [torch.empty(B, H, D, dtype=torch.bfloat16, device=dev) for _ in range(steps)]
    dstream.synchronize()
    for t in range(3):  # warm-up on a copy of the state
        scratch = state.clone()
        api.decode_step(*toks[t], scratch, out=outs[t], stream=dstream)
    dstream.synchronize()
    del scratch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    dist_barrier(world)
    torch.cuda.synchronize()
    ev[0].record(dstream)
    for t in range(steps):
        api.decode_step(*toks[t], state, out=outs[t], stream=dstream)
        ev[t + 1].record(dstream)
    dstream.synchronize()
    dist_barrier(world)
    per = [ev[t].elapsed_time(ev[t + 1]) for t in range(steps)]
    med_ms = statistics.median(per)
    total_ms = dist_max(ev[0].elapsed_time(ev[steps]), world, dev)
    gbs = decode_bytes(B, H, D) / (med_ms / 1e3) / 1e9
    status = api.device_status(dstream)
    res = {"workload": f"decode step, B={B}, H={H}, D={D}, bf16 q/k/v/o, fp32 state from a "
                       f"seeded N={N} prefill, {steps} consecutive steps",
           "tokens_per_s": B * world * steps / (total_ms / 1e3),
           "ms_per_step_median": med_ms, "gbs_median_step": gbs, "pct_hbm": 100.0 * gbs / peak_bw,
           "bytes_per_step": decode_bytes(B, H, D), "gpu_launches": steps,
           "status": api.status_string(status), "stream": "own stream (not the prefill stream)"}
    return res, (dstream, state, toks, outs)


SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072)


def sweep_row(N, T, H, D, beta, ms, peak_bw, status):
    """One point of the length sweep: B = T / N sequences of N tokens in one launch."""
    s = ms / 1e3
    return {"N": N, "B": T // N, "ms_per_launch": ms, "tokens_per_s": T / s,
            "tflops_tiled": tiled_flops_per_token_head(D, beta) * T * H / s / 1e12,
            "hbm_frac": prefill_bytes(T, H, D) / s / 1e9 / peak_bw, "status": status}


def bench_length_sweep(api, torch, stream, q, k, v, o, beta, peak_bw, reps=20, warm=3):
    """Prefill speed against sequence length at a fixed token count per launch.

    The main workload's Q/K/V/O (T tokens x H heads) are viewed as B = T / N sequences of N
    tokens, N = 1K .. 128K, so every launch reads and writes the same bytes.  Attention that
    is linear in N keeps the time per launch independent of N; the pages claim a constant
    speed over 1K-64K tokens (measured against FlashAttention-2 on other GPUs)."""
    H, D = q.shape[-2], q.shape[-1]
    T = q.numel() // (H * D)
    rows = []
    for N in SWEEP_N:
        if N > T or T % N:
            continue
        B = T // N
        qv, kv_, vv, ov = (x.reshape(B, N, H, D) for x in (q, k, v, o))
        for _ in range(warm):
            api.prefill(qv, kv_, vv, beta=beta, out=ov, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            api.prefill(qv, kv_, vv, beta=beta, out=ov, stream=stream)
        e1.record(stream)
        stream.synchronize()
        status = api.status_string(api.device_status(stream))
        rows.append(sweep_row(N, T, H, D, beta, e0.elapsed_time(e1) / reps, peak_bw, status))
    return {"what": "prefill at a fixed T x H per launch, as B = T / N sequences of N tokens",
            "tokens_per_launch": T, "heads": H, "head_dim": D, "beta": beta,
            "launches_per_point": reps, "rows": rows}


def bench_prefill_options(api, torch, stream, q, k, v, o, peak_bw, reps=10, warm=3):
    """The main workload through the other options of la_prefill: the fused output RMSNorm,
    beta = 64 (the unpaired tcgen05 kernel) and a start from an initial state (read only;
    the inter-block term of block 0 is then computed too).  The options and the plain call
    take turns launch by launch, so that each option meets the same clocks and power state
    as the plain launches it is compared with (``vs_plain`` = median over median)."""
    H, D = q.shape[-2], q.shape[-1]
    T = q.numel() // (H * D)
    S = q.shape[0] if q.dim() == 4 else 1
    X = torch.zeros((S, H, D, D), dtype=torch.float32, device=q.device)
    cases = {"plain": dict(beta=128),
             "rmsnorm": dict(beta=128, rmsnorm=True),
             "beta64": dict(beta=64),
             "initial_state": dict(beta=128, initial_state=X)}
    for _ in range(warm):
        for kw in cases.values():
            api.prefill(q, k, v, out=o, stream=stream, **kw)
    ev = {name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(reps)] for name in cases}
    torch.cuda.synchronize()
    for i in range(reps):
        for name, kw in cases.items():
            ev[name][i][0].record(stream)
            api.prefill(q, k, v, out=o, stream=stream, **kw)
            ev[name][i][1].record(stream)
    stream.synchronize()
    med = {name: statistics.median(a.elapsed_time(b) for a, b in ev[name]) for name in cases}
    res = {}
    for name in cases:
        ms = med[name]
        res[name] = {"ms_per_launch": ms, "tokens_per_s": T / (ms / 1e3),
                     "hbm_frac": prefill_bytes(T, H, D) / (ms / 1e3) / 1e9 / peak_bw,
                     "vs_plain": ms / med["plain"]}
    res["status"] = api.status_string(api.device_status(stream))
    res["launches_per_option"] = reps
    res["order"] = "interleaved: " + ", ".join(cases) + " in turn, medians"
    return res


def timed_launches(torch, stream, fn, reps, warm, device_index):
    """Per-launch CUDA-event times (ms) of ``fn`` on ``stream`` after ``warm`` untimed calls,
    with the SM clock sampled while they run."""
    for _ in range(warm):
        fn()
    stream.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    with ClockSampler(device_index, period_s=0.005) as clk:
        ev[0].record(stream)
        for i in range(reps):
            fn()
            ev[i + 1].record(stream)
        stream.synchronize()
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)], clk.summary()


def spread(ms):
    """Median and range of per-launch times."""
    return {"median": statistics.median(ms), "min": min(ms), "max": max(ms), "launches": len(ms)}


def tiled_flops_packed(lengths, H: int, D: int, beta: int) -> int:
    """Tiled-form flops of a packed batch: every block of beta tokens counted in full
    (a partial last block costs a whole block): per block 4 beta^2 D + 4 beta D^2 per head."""
    blocks = sum((n + beta - 1) // beta for n in lengths)
    return blocks * H * (4 * beta * beta * D + 4 * beta * D * D)


def prefill_leg(name, ms, clocks, T, H, D, flops, peaks):
    """Metric view of one timed prefill configuration."""
    s = statistics.median(ms) / 1e3
    bw = prefill_bytes(T, H, D) / s / 1e9
    tf = flops / s / 1e12
    return {"workload": name, "ms_per_launch": spread(ms), "tokens_per_s": T / s,
            "tflops_tiled": tf, "pct_bf16_peak": 100.0 * tf / float(peaks["bf16_tflops"]),
            "hbm_gbs": bw, "hbm_frac": bw / float(peaks["hbm_gbs"]),
            "algorithmic_bytes": prefill_bytes(T, H, D), "clocks": clocks}


def cpu_oracle_quadratic(q, k, v, reps=20):
    """The fp64 quadratic-form oracle on a whole (tiny) workload, mean of ``reps`` runs."""
    import oracle
    cores = max(1, os.cpu_count() or 1)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.quadratic(q, k, v, nthreads=cores)
    t = (time.perf_counter() - t0) / reps
    T, H = q.shape[0], q.shape[1]
    return {"value": T / t, "unit": "tokens/s", "cores": min(cores, H), "kind": "oracle", "seconds": t,
            "sample": f"fp64 quadratic form, the whole workload ({H} heads x {T} tokens), mean of {reps} runs"}


def cpu_oracle_prefill(q, k, v, cu, rmsnorm, heads, what):
    """The fp64 recurrent oracle on the first ``heads`` heads of a workload, all its tokens,
    on the host cores; value in tokens/s of the H-head layer."""
    import oracle
    H = q.shape[1]
    cores = max(1, os.cpu_count() or 1)
    t0 = time.perf_counter()
    oracle.recurrent(q[:, :heads], k[:, :heads], v[:, :heads], cu, rmsnorm=rmsnorm,
                     want_o=True, nthreads=cores)
    t = time.perf_counter() - t0
    T = q.shape[0]
    S = 1 if cu is None else len(cu) - 1
    return {"value": T * heads / H / t, "unit": "tokens/s", "cores": min(cores, heads * S),
            "kind": "oracle", "seconds": t,
            "sample": f"fp64 recurrent form, {what}: {heads}/{H} heads x all {T} tokens, "
                      f"value = token-heads / {H} / time"}


def bench_configs(api, synth, torch, stream, dev, peaks, cpu: bool):
    """The other configurations of the method's workload list, each timed on its own:
    the tiny fp32 case, the MiniMax-layer prefill (64 heads x 128, N = 8192, RMSNorm,
    beta = 128 and 64), the packed varlen batch (262144 tokens, 8 seeded sequences) and a
    mixed batch of one-token (decode) rows and prefill chunks from per-sequence states."""
    di = dev.index if dev.index is not None else torch.cuda.current_device()
    res = {}
    # config 1: B=1, H=2, N=256, D=64, beta=64, fp32, no norm
    q, k, v = synth.qkv(256, 2, 64, seed=0, dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    ms, clk = timed_launches(torch, stream, lambda: api.prefill(q, k, v, beta=64, out=o, stream=stream),
                             200, 5, di)
    res["c1_tiny_fp32"] = {"workload": "B=1, H=2, N=256, D=64, beta=64, fp32, no norm",
                           "ms_per_launch": spread(ms), "tokens_per_s": 256 / (statistics.median(ms) / 1e3),
                           "clocks": clk}
    if cpu:
        res["c1_tiny_fp32"]["cpu_baseline"] = cpu_oracle_quadratic(q, k, v)
    # config 2: MiniMax layer, RMSNorm, beta 128 and 64
    N, H, D = 8192, 64, 128
    q, k, v = synth.qkv(N, H, D, seed=2, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    c2 = {}
    for beta in (128, 64):
        ms, clk = timed_launches(torch, stream, lambda: api.prefill(q, k, v, beta=beta, rmsnorm=True, out=o,
                                                                    stream=stream), 50, 5, di)
        c2[f"beta{beta}"] = prefill_leg(f"B=1, N={N}, H={H}, D={D}, beta={beta}, bf16, RMSNorm", ms, clk,
                                        N, H, D, tiled_flops_packed([N], H, D, beta), peaks)
    if cpu:
        c2["cpu_baseline"] = cpu_oracle_prefill(q, k, v, None, True, H, "config 2 with RMSNorm")
    res["c2_layer_rmsnorm"] = c2
    del q, k, v, o
    # config 4: packed varlen, 262144 tokens, 8 seeded sequences, beta = 128
    T, S = 262144, 8
    cu = synth.cu_seqlens_uniform(T, S, seed=0)
    lens = [int(cu[i + 1] - cu[i]) for i in range(S)]
    q, k, v = synth.qkv(T, H, D, seed=4, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    ms, clk = timed_launches(torch, stream, lambda: api.prefill(q, k, v, beta=128, cu_seqlens=cu, out=o,
                                                                stream=stream), 20, 3, di)
    c4 = prefill_leg(f"packed varlen, T={T}, S={S} seeded uniform lengths {lens}, H={H}, D={D}, "
                     f"beta=128, bf16", ms, clk, T, H, D, tiled_flops_packed(lens, H, D, 128), peaks)
    if cpu:
        c4["cpu_baseline"] = cpu_oracle_prefill(q, k, v, cu, False, min(H, 4), "config 4")
    res["c4_packed_varlen"] = c4
    del q, k, v, o
    # mixed batch: 256 one-token rows and 8 chunks of 4096 tokens, each from its own state,
    # in one la_prefill; against the one-token rows through la_decode_step plus the chunks
    # through la_prefill
    n1, nc, L = 256, 8, 4096
    lens = [1] * n1 + [L] * nc
    cu_m = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tm = int(cu_m[-1])
    q, k, v = synth.qkv(Tm, H, D, seed=6, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    X = synth.initial_state(n1 + nc, H, D, tokens=4096, seed=6, device=dev)
    st = X.clone()
    ms_mix, clk = timed_launches(torch, stream, lambda: api.prefill(
        q, k, v, beta=128, cu_seqlens=cu_m, initial_state=st, state_out=st, out=o, stream=stream), 20, 3, di)
    qd, kd, vd = (x[:n1].contiguous() for x in (q, k, v))
    od = torch.empty_like(qd)
    st1 = X[:n1].clone()
    qc, kc, vc = (x[n1:].contiguous() for x in (q, k, v))
    oc = torch.empty_like(qc)
    stc = X[n1:].clone()
    cu_c = [0] + [L * (i + 1) for i in range(nc)]

    def split():
        api.decode_step(qd, kd, vd, st1, out=od, stream=stream)
        api.prefill(qc, kc, vc, beta=128, cu_seqlens=cu_c, initial_state=stc, state_out=stc, out=oc,
                    stream=stream)
    ms_split, _ = timed_launches(torch, stream, split, 20, 3, di)
    res["f4_mixed_batch"] = {
        "workload": f"{n1} one-token sequences + {nc} chunks of {L} tokens, H={H}, D={D}, bf16, "
                    f"each from its own state (read and written in place)",
        "one_prefill_call_ms": spread(ms_mix),
        "decode_step_plus_prefill_ms": spread(ms_split),
        "clocks": clk,
        "note": "the same work as one la_prefill call (which runs the one-token sequences through "
                "the decode kernel, in place, and the chunks through the prefill kernel), and as "
                "la_decode_step on gathered one-token rows followed by la_prefill for the chunks"}
    res["status"] = api.status_string(api.device_status(stream))
    return res


def bench_headline_repeat(api, torch, stream, q, k, v, o, beta, peak_bw, device_index, reps=100):
    """The main step repeated: the spread of the per-launch time over ``reps`` launches and
    the SM clock while they ran."""
    ms, clk = timed_launches(torch, stream, lambda: api.prefill(q, k, v, beta=beta, out=o, stream=stream),
                             reps, 3, device_index)
    H, D = q.shape[-2], q.shape[-1]
    T = q.numel() // (H * D)
    med = statistics.median(ms)
    return {"ms_per_launch": spread(ms), "hbm_frac_median": prefill_bytes(T, H, D) / (med / 1e3) / 1e9 / peak_bw,
            "clocks": clk, "status": api.status_string(api.device_status(stream))}


def decode_cpu_baseline(torch, dctx, Bs=16):
    """The fp64 decode oracle over the 64 decode steps on the first ``Bs`` sequences of the
    decode batch (all heads), from the GPU state before the steps; tokens/s of the batch."""
    import oracle
    dstream, state0, toks, _ = dctx
    st = state0[:Bs].detach().to("cpu").double().numpy()
    cores = max(1, os.cpu_count() or 1)
    t0 = time.perf_counter()
    for t in range(len(toks)):
        q, k, v = (x[:Bs] for x in toks[t])
        _, st = oracle.decode_step(q, k, v, st, nthreads=cores)
    sec = time.perf_counter() - t0
    B = state0.shape[0]
    return {"value": Bs * len(toks) / sec, "unit": "decode tokens/s", "cores": cores, "kind": "oracle",
            "seconds": sec, "sample": f"fp64 decode oracle, {len(toks)} steps on {Bs}/{B} sequences x all "
                                      f"heads, from a copy of the GPU decode state"}


def bench_chunk_state(api, torch, stream, k, v, peak_bw, world, reps=5):
    """Step 1 of LASP+ on the main workload's K and V: each sequence's K^T V alone.  It
    reads 4 D bytes per token-head (K and V) and writes the fp32 states."""
    H, D = k.shape[-2], k.shape[-1]
    T = k.numel() // (H * D)
    st = api.chunk_state(k, v, stream=stream)  # warm-up and allocation
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    dist_barrier(world)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(reps):
        api.chunk_state(k, v, state_out=st, stream=stream)
        ev[i + 1].record(stream)
    stream.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
    ms = statistics.median(per)
    nbytes = 4 * D * T * H + st.numel() * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"kernel": "la::chunk_state_tc_kernel (the local state of a chunk in LASP+)",
            "ms_median": ms, "bytes": nbytes, "gbs": gbs, "pct_hbm": 100.0 * gbs / peak_bw,
            "launches": reps, "status": api.status_string(api.device_status(stream))}


def dist_gather(values, world: int, device=None):
    """Every rank's list of floats (same length on every rank), in rank order."""
    if world == 1:
        return [list(values)]
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    out = t.new_empty((world * t.numel(),))
    dist.all_gather_into_tensor(out, t)
    return out.view(world, -1).tolist()


LASP_PARTS = ("chunk_state", "all_gather", "state_prefix", "prefill", "step")


def lasp_leg(api, torch, stream, q, k, v, o, rank, world, peak_bw, dev):
    """bench_lasp on the first N / world rows of this rank's inputs ([1, N, H, D] views), as
    chunk r of one sequence.  On one GPU the leg runs in a one-rank NCCL group of its own,
    so that the same all-gather on the kernels' stream is exercised."""
    import datetime

    import torch.distributed as dist

    from long_context_04_b200 import lasp
    L = q.shape[1] // world
    views = [x[:, :L] for x in (q, k, v, o)]
    own = False
    if world == 1 and not dist.is_initialized():
        dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
        own = True
    try:
        return bench_lasp(api, lasp, torch, stream, *views, rank, world, peak_bw, device=dev)
    finally:
        if own:
            dist.destroy_process_group()


def bench_lasp(api, lasp, torch, stream, q, k, v, o, rank, world, peak_bw, device=None,
               beta=128, reps=10, warm=3):
    """LASP+ sequence parallelism over the ranks: one sequence of world * L tokens in
    contiguous chunks, chunk r (q, k, v, o: [1, L, H, D]) on rank r.  One step, in order on
    the kernels' stream:
        la_chunk_state   S_r = K_r^T V_r
        all-gather       the fp32 chunk states of every rank (NCCL, H D^2 4 bytes per rank)
        la_state_prefix  X_r = sum of S_r' over r' < r
        la_prefill       O_r from X_r (LA_READ_STATE)
    Every rank takes the same collectives in the same order.  Reported: each rank's median
    time of every part, and the whole sequence's tokens/s over the slowest rank's time."""
    H, D = q.shape[-2], q.shape[-1]
    L = q.shape[1]
    local = api.chunk_state(k, v, stream=stream)          # warm-up and allocation
    init = local.new_zeros(local.shape)

    def step(marks=None):
        api.chunk_state(k, v, state_out=local, stream=stream)
        if marks:
            marks[1].record(stream)
        gathered = lasp.all_gather_states(local)
        if marks:
            marks[2].record(stream)
        api.state_prefix(gathered, rank, out=init, stream=stream)
        if marks:
            marks[3].record(stream)
        api.prefill(q, k, v, beta=beta, out=o, initial_state=init, stream=stream)
        if marks:
            marks[4].record(stream)

    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):     # the collective is ordered with the kernels
        for _ in range(warm):
            step()
        dist_barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(reps):
            marks[i][0].record(stream)
            step(marks[i])
        t1.record(stream)
        torch.cuda.synchronize()
    dist_barrier(world)
    total_ms = dist_max(t0.elapsed_time(t1), world, device)
    parts = [statistics.median(m[j].elapsed_time(m[j + 1]) for m in marks) for j in range(4)]
    parts.append(statistics.median(m[0].elapsed_time(m[4]) for m in marks))
    per_rank = dist_gather(parts, world, device)
    status = api.status_string(api.device_status(stream))
    tokens = world * L
    return {"workload": f"one sequence of N={tokens} tokens, H={H}, D={D}, beta={beta}, bf16, "
                        f"in {world} contiguous chunks of {L} tokens, chunk r on rank r",
            "steps": reps, "warmup": warm,
            "slowest_rank_ms_per_step": total_ms / reps,
            "tokens_per_s": tokens * reps / (total_ms / 1e3),
            "per_rank_ms_median": [dict(zip(LASP_PARTS, r)) for r in per_rank],
            "gathered_bytes_per_rank": world * H * D * D * 4,
            "prefill_hbm_frac": prefill_bytes(L, H, D) / (parts[3] / 1e3) / 1e9 / peak_bw,
            "scaling": "strong (the sequence is fixed; each rank takes 1/N of it)",
            "status": status}


def bench_concurrent(api, torch, pstream, dctx, q, k, v, o, beta, world, n_prefill=2):
    """The two paths together, as the pages arrange them (length-1 and length>1 requests on
    two streams): the main prefill workload on its stream while the decode steps run on
    theirs.  Each was also measured alone above."""
    dstream, state, toks, outs = dctx
    steps = len(toks)
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    eb = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    dist_barrier(world)
    torch.cuda.synchronize()
    ea[0].record(pstream)
    for _ in range(n_prefill):
        api.prefill(q, k, v, beta=beta, out=o, stream=pstream)
    ea[1].record(pstream)
    eb[0].record(dstream)
    for t in range(steps):
        api.decode_step(*toks[t], state, out=outs[t], stream=dstream)
        eb[t + 1].record(dstream)
    torch.cuda.synchronize()
    dist_barrier(world)
    status = api.device_status(pstream)
    per = [eb[t].elapsed_time(eb[t + 1]) for t in range(steps)]
    first = ea[0] if ea[0].elapsed_time(eb[0]) >= 0 else eb[0]
    last = ea[1] if eb[steps].elapsed_time(ea[1]) >= 0 else eb[steps]
    overlapped = sum(1 for t in range(steps) if eb[t].elapsed_time(ea[1]) > 0)
    return {"prefill_ms_per_launch": ea[0].elapsed_time(ea[1]) / n_prefill,
            "prefill_launches": n_prefill, "decode_steps": steps,
            "decode_steps_started_during_prefill": overlapped,
            "decode_ms_per_step_median": statistics.median(per),
            "decode_ms_per_step_max": max(per),
            "span_ms": first.elapsed_time(last),
            "status": api.status_string(status),
            "note": "prefill on one stream and the decode steps on another, enqueued together; "
                    "the prefill's persistent CTA pairs hold 128 of the 148 SMs while it runs"}


def run_decode_small(args):
    """Decode-only run on one GPU (B=64, H=64, D=128), for profiling the decode kernel."""
    import torch

    from long_context_04_b200 import api, build as lib_build, synth
    lib_build.build()
    B, H, D = 64, 64, 128
    dev = torch.device("cuda", 0)
    g = synth.generator(7, dev)
    state = torch.randn(B, H, D, D, generator=g, device=dev, dtype=torch.float32)
    toks = [synth.decode_tokens(B, H, D, step=t, seed=0, device=dev)
            for t in range(args.steps + args.warmup)]
    out = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    for t in range(args.warmup):
        api.decode_step(*toks[t], state, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(args.steps):
        api.decode_step(*toks[args.warmup + t], state, out=out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peaks, _ = load_peaks()
    gbs = decode_bytes(B, H, D) / (ms / 1e3) / 1e9
    print(json.dumps({"workload": f"decode step B={B} H={H} D={D} (profiling case)",
                      "ms_per_step": ms, "gbs": gbs, "pct_hbm": 100 * gbs / peaks["hbm_gbs"],
                      "status": api.status_string(api.device_status())}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["decode_b64"],
                    default="prefill_n131k",
                    help="decode_b64: decode steps only, B=64 H=64 D=128 with a seeded random "
                         "fp32 state (256 MB, larger than L2); a small case for profiling")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the prefill only (no e2e, decode or CPU baseline)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload == "decode_b64":
        return run_decode_small(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
