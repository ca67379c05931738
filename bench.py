"""Throughput of the future-attention-target hot path on B200.

One step = row logsumexp + transposed future-target pass + keep mask over one
synthetic Qwen3-8B-shaped layer at 16,384 tokens (32 query / 8 KV heads,
head_dim 128, W = 256, 4 sinks, budget 4,032 per KV head), inputs resident
in HBM.  The metric is algorithmic tensor TFLOP/s: 2 * head_dim flops per
unmasked (query, key) pair per query head, for both passes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (under torchrun) every rank runs its own independent layer (its
own seed): weak scaling, no data-path collective.  `--impl reference` times
the CPU float64 oracle on a bounded sample of the same workload.
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
sys.path.insert(0, ROOT)

from future_attention_targets_b200.workloads import WORKLOADS, algorithmic_flops, make_inputs  # noqa: E402

METRIC = "future-attn target TFLOP/s & % BF16 tensor peak, Qwen3-8B shape, 16k ctx"
UNIT = "TFLOP/s"
WORKLOAD = "qwen3_8b_16k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["attn_kernels.cu", "kvpop_device.cuh", "kvpop_sched.h", "kvpop_debug.cuh"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def strip_comments(src: str) -> str:
    """C/C++ source without // and /* */ comments, trailing blanks and empty lines (string and character
    literals kept intact), so that editing a comment leaves the code's fingerprint unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_hash(read=None) -> str:
    """First 16 hex digits of the sha256 of the attention kernels' sources, comments stripped.
    read(name) -> text overrides how a source file is read (to fingerprint another revision)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        if read is None:
            with open(os.path.join(ROOT, "future_attention_targets_b200", "csrc", name)) as f:
                text = f.read()
        else:
            text = read(name)
        h.update(strip_comments(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{WORKLOAD}.traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, cuda_index: int):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle_for(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.nvml, self.error = None, str(e)

    def _handle_for(self, idx):
        import torch
        pynvml = self.nvml
        try:
            props = torch.cuda.get_device_properties(idx)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        pynvml = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def threads_in_use() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(d, kv_head: int = 0):
    """Runs the oracle on one KV-head group: its G query heads over all positions, both passes (1/H_kv of a
    step's work).  Returns (seconds, algorithmic flops of the sample, description)."""
    import oracle
    w = d["workload"]
    G, L, W = w.group, w.seqlen, w.window
    qh = d["q_bits"][:, kv_head * G:(kv_head + 1) * G]
    kh = d["k_bits"][:, kv_head:kv_head + 1]
    cu = d["cu_seqlens"]
    t0 = time.perf_counter()
    oracle.future_target(qh, kh, cu, W, d["scale"], return_lse=True)
    fl = algorithmic_flops([L], G, w.head_dim, W)["total"]
    desc = f"KV head {kv_head} with its {G} query heads, all {L} positions, both passes (1/{w.n_kv_heads} of a step)"
    return time.perf_counter() - t0, fl, desc


# ------------------------------------------------------------------ multi-rank helpers

def rank_seed(rank: int) -> int:
    """Each rank runs its own independent layer: the workload seed is the rank."""
    return int(rank)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank number over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_throughput(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ reference arm (CPU oracle)

def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line, identical in both arms."""
    return {"workload": WORKLOAD, "seq_len": w.seqlen, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "window": w.window,
            "sinks": w.sinks, "budget": w.budget, "input": "1% heavy-hitter keys, seed = rank",
            "l2": "inputs larger than L2 (160 MiB of Q and K vs 126 MB L2); no flush",
            "parallelism": f"independent layer per rank x{world}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = make_inputs(WORKLOAD)
    w = d["workload"]
    # The same bounded sample as the GPU arm's cpu_baseline: one whole KV-head
    # group (both passes over all positions), 1/H_kv of a step's work.
    for _ in range(args.warmup):
        oracle_sample(d)
    total_t, total_f = 0.0, 0
    desc = ""
    for _ in range(args.steps):
        t, f, desc = oracle_sample(d)
        total_t += t
        total_f += f
    value = total_f / total_t / 1e12
    step_flops = algorithmic_flops([w.seqlen], w.n_q_heads, w.head_dim, w.window)["total"]
    cores = threads_in_use()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup,
        # a whole step's time at the sample's rate (the sample is 1/H_kv of the step's flops)
        "ms_per_step": 1e3 * step_flops / (value * 1e12),
        "sample_ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {desc}; ms_per_step scales the sample time by the step's flops"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def run_head_sharded(args, w, cu, W, S, budgets, scale, world, rank, dev, stream, fl, ms_per_step):
    """One problem (rank 0's layer) with its KV heads split over the ranks: two passes on H_kv / P heads
    (the split transposed pass), one NCCL all-gather of the targets, the keep mask on all heads."""
    import torch
    import torch.distributed as dist

    from future_attention_targets_b200 import check_status
    from future_attention_targets_b200.sharded import HeadShardedTargets, shard_heads
    d0 = make_inputs(WORKLOAD, seed=rank_seed(0))
    q0 = torch.from_numpy(d0["q_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
    k0 = torch.from_numpy(d0["k_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
    q_loc, k_loc = shard_heads(q0, k0, w.n_kv_heads, world, rank)
    del q0, k0, d0
    sharded = HeadShardedTargets(cu, w.n_q_heads, w.n_kv_heads, w.head_dim, W, S, budgets, scale, device=dev)
    for _ in range(max(3, args.warmup)):
        sharded(q_loc, k_loc, stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    torch.cuda.synchronize(dev)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        sharded(q_loc, k_loc, stream)
    z.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    ms_sh = max_over_ranks(a.elapsed_time(z), dev) / args.steps
    check_status(sharded.status, stream)
    result = {
        "ms": ms_sh, "scaling": "strong", "value": fl["total"] / (ms_sh * 1e-3) / 1e12, "unit": UNIT,
        "speedup_vs_one_gpu_step": ms_per_step / ms_sh, "kv_heads_per_rank": w.n_kv_heads // world,
        "collective": "one all_gather_into_tensor (NCCL) of target [H_kv / P, T] fp32 per step",
        "gathered_bytes": int(sharded.target.numel() * 4)}
    del sharded, q_loc, k_loc
    return result


def run_ours(args):
    import torch
    import torch.distributed as dist

    from future_attention_targets_b200 import (HostPipeline, check_status, future_target, future_targets, keep_mask,
                                               lib, row_lse, target_workspace_bytes)
    from future_attention_targets_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    lib()

    d = make_inputs(WORKLOAD, seed=rank_seed(rank))   # an independent layer per rank
    w = d["workload"]
    cu, W, S, budgets, scale = d["cu_seqlens"], d["window"], d["sinks"], d["budgets"], d["scale"]
    q = torch.from_numpy(d["q_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(d["k_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
    T = q.shape[0]
    lse = torch.empty((w.n_q_heads, T), dtype=torch.float32, device=dev)
    tgt = torch.empty((w.n_kv_heads, T), dtype=torch.float32, device=dev)
    keep = torch.empty((w.n_kv_heads, T), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # The transposed pass's normaliser rows (16 bytes per query head and token).
    tws = torch.empty(target_workspace_bytes(T, w.n_q_heads, w.n_kv_heads, w.head_dim), dtype=torch.uint8,
                      device=dev)

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        row_lse(q, k, cu, scale, out=lse, status=status, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        # two launches: lse -> normaliser rows, then the transposed pass
        future_target(q, k, cu, W, lse, scale, out=tgt, workspace=tws, status=status, stream=stream)
        if evs is not None:
            evs[2].record(stream)
        keep_mask(tgt, cu, W, S, budgets, out=keep, stream=stream)
        if evs is not None:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check_status(status, stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    check_status(status, stream)
    elapsed_ms = t_start.elapsed_time(t_end)
    per_kernel = {name: [e[j].elapsed_time(e[j + 1]) for e in evs]
                  for j, name in enumerate(["row_lse", "future_target", "keep_mask"])}
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    fl = algorithmic_flops([w.seqlen], w.n_q_heads, w.head_dim, w.window)
    ms_per_step = elapsed_ms / args.steps
    value = weak_throughput(fl["total"], world, ms_per_step)
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak))

    avg = {n: statistics.mean(v) for n, v in per_kernel.items()}
    dom = max(("row_lse", "future_target"), key=lambda n: avg[n])
    dom_flops = fl["lse"] if dom == "row_lse" else fl["target"]
    achieved = dom_flops / (avg[dom] * 1e-3) / 1e12

    # End to end through the host-buffer C entry point: H2D of q and k, the
    # three kernels, D2H of target and keep, every step.
    e2e = None
    if not args.no_e2e:
        # Two pipelines (workspaces and pinned outputs) on two streams, alternating: each step copies its
        # q and k in and its target and keep out, and one step's copies in overlap the other's compute.
        pipes = [HostPipeline(cu, w.n_q_heads, w.n_kv_heads, w.head_dim, W, S, budgets, scale, device=dev)
                 for _ in range(2)]
        streams = [stream, torch.cuda.Stream(dev)]
        qh = torch.from_numpy(d["q_bits"].view(np.int16)).view(torch.bfloat16).pin_memory()
        kh = torch.from_numpy(d["k_bits"].view(np.int16)).view(torch.bfloat16).pin_memory()
        for i in range(4):
            pipes[i % 2](qh, kh, streams[i % 2])
        # One step on its own, synchronised (the latency a single call sees).
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        l0.record(stream)
        pipes[0](qh, kh, stream)
        l1.record(stream)
        torch.cuda.synchronize(dev)
        lat_ms = max_over_ranks(l0.elapsed_time(l1), dev)
        n_e2e = max(4, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(n_e2e):
            pipes[i % 2].submit(qh, kh, streams[i % 2])
        streams[0].wait_stream(streams[1])
        e1.record(streams[0])
        torch.cuda.synchronize(dev)
        for p_ in pipes:
            check_status(p_.status, stream)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": weak_throughput(fl["total"], world, e_ms / n_e2e), "unit": UNIT,
               "h2d_bytes_per_step": pipes[0].h2d_bytes, "d2h_bytes_per_step": pipes[0].d2h_bytes,
               "ms_per_step": e_ms / n_e2e, "steps": n_e2e,
               "pipelining": "two workspaces on two streams: a step's copies in overlap the previous step's "
                             "compute; every step copies its own q, k in and target, keep out",
               "single_step_latency_ms": lat_ms}
        del pipes

    # Rows beyond the hot path, timed on this step's own targets (outside the timed region above).
    extras = {}
    if not args.no_extras:
        # The same step with both attention passes in one cooperative launch.
        from future_attention_targets_b200 import fused_workspace, future_targets_fused
        ws_f = fused_workspace(cu, w.n_q_heads, w.n_kv_heads, w.head_dim, device=dev)
        lse_f, tgt_f, keep_f = torch.empty_like(lse), torch.empty_like(tgt), torch.empty_like(keep)

        def fused_step():
            future_targets_fused(q, k, cu, W, S, budgets, scale, lse=lse_f, target=tgt_f, keep=keep_f,
                                 workspace=ws_f, status=status, stream=stream)

        for _ in range(max(3, args.warmup)):
            fused_step()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            fused_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        check_status(status, stream)
        ms_f = f0.elapsed_time(f1) / args.steps
        extras["fused_single_launch"] = {
            "ms_per_step": ms_f, "value": fl["total"] / (ms_f * 1e-3) / 1e12, "unit": UNIT,
            "vs_two_launch_step": ms_per_step / ms_f,
            # one CTA per item here, CTA pairs in the two-launch step: the same lse bits, the targets
            # equal up to fp32 rounding (a different grouping of each key's query tiles)
            "lse_identical_to_two_launch": bool(torch.equal(lse_f, lse)),
            "target_max_rel_diff_vs_two_launch": float(((tgt_f.double() - tgt.double()).abs()
                                                        / tgt.double().abs().clamp_min(1e-3)).max()),
            "launches_per_step": 2}
        del ws_f, lse_f, tgt_f, keep_f

        from future_attention_targets_b200 import prefix_topk_thresholds
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # twice the 126 MB L2

        def timed(fn, reps=20):
            """Median device time of fn, with L2 flushed before every repetition: a 256 MiB buffer is
            written and then read back, so the L2 holds none of fn's data and no dirty lines whose
            write-back fn would pay for.  A ~0.1 ms device-side wait after the flush keeps the GPU busy
            while the host enqueues the start event and fn, so the interval holds fn's device work and
            not the host's enqueue time."""
            for _ in range(3):
                fn()
            evs_x = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(reps)]
            for a, z in evs_x:
                flush.zero_()
                torch.amax(flush.view(torch.int32))
                torch.cuda._sleep(200_000)
                a.record(stream)
                fn()
                z.record(stream)
            torch.cuda.synchronize(dev)
            return statistics.median(a.elapsed_time(z) for a, z in evs_x)

        def timed_rotating(fns, reps=40):
            """Mean device time per launch of back-to-back launches cycling over fns, each on its own copy
            of the inputs, the copies together larger than the L2 (so every launch reads from HBM).  The
            launches are captured in one CUDA graph and replayed, so that the host's enqueue rate (slower
            than these kernels) does not set the pace: the fixed cost of a lone event-timed launch is
            left out, the gaps between launches are not."""
            for f in fns:
                f(stream)
            torch.cuda.synchronize(dev)
            graph, side = torch.cuda.CUDAGraph(), torch.cuda.Stream(dev)   # captured on a side stream
            with torch.cuda.graph(graph, stream=side):
                for i in range(reps):
                    fns[i % len(fns)](side)
            graph.replay()
            times = []
            for _ in range(3):
                a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                graph.replay()
                z.record(stream)
                torch.cuda.synchronize(dev)
                times.append(a.elapsed_time(z) / reps)
            del graph
            return statistics.median(times)

        # What a lone launch costs here with nothing in it: the floor under every flushed figure below.
        floor_ms = timed(lambda: torch.cuda._sleep(0))
        thr = (torch.empty_like(tgt), torch.empty(tgt.shape, dtype=torch.int32, device=dev))
        ms = timed(lambda: prefix_topk_thresholds(tgt, cu, W, S, budgets, out=thr, stream=stream))
        steps_total = sum(int(L) for L in np.diff(cu)) * w.n_kv_heads
        moved = tgt.numel() * 4 + thr[0].numel() * 4 + thr[1].numel() * 4   # score in, threshold score + position out
        peaks_x, _ = load_peaks()
        extras["prefix_topk_thresholds"] = {
            "ms": ms, "steps_per_s": steps_total / (ms * 1e-3),
            "bound": "latency", "hbm_gbs": moved / (ms * 1e-3) / 1e9,
            "frac_of_hbm": moved / (ms * 1e-3) / 1e9 / float(peaks_x["hbm_gbs"]),
            "launch": (f"{len(cu) - 1} x {w.n_kv_heads} x {-(-(int(max(np.diff(cu))) - S - W) // 1024)} CTAs of 1024 "
                       "threads, one per (sequence, KV head, block of 1024 steps)")}

        # The hot path on the other four workloads (the same kernels, other shapes).  The two large ones
        # hold more Q and K than the L2 and run back to back; the 4k and tiny ones fit in the L2, so each
        # of their repetitions is timed on its own after an L2 flush.
        for other in ("long_64k", "varlen_8x", "qwen3_4b_4k", "tiny"):
            do = make_inputs(other, seed=rank_seed(rank))
            wo = do["workload"]
            qo = torch.from_numpy(do["q_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
            ko = torch.from_numpy(do["k_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
            To = qo.shape[0]
            lo_ = torch.empty((wo.n_q_heads, To), dtype=torch.float32, device=dev)
            to_ = torch.empty((wo.n_kv_heads, To), dtype=torch.float32, device=dev)
            ko_ = torch.empty((wo.n_kv_heads, To), dtype=torch.uint8, device=dev)
            wso = torch.empty(target_workspace_bytes(To, wo.n_q_heads, wo.n_kv_heads, wo.head_dim), dtype=torch.uint8,
                              device=dev)
            run_o = lambda: future_targets(qo, ko, do["cu_seqlens"], do["window"], do["sinks"], do["budgets"],
                                           do["scale"], lse=lo_, target=to_, keep=ko_, workspace=wso, status=status,
                                           stream=stream)
            small = 2 * (qo.numel() + ko.numel()) < (126 << 20)
            if small:
                ms_o = timed(run_o, reps=20)
                how = "median of 20, L2 flushed before each"
            else:
                for _ in range(2):
                    run_o()
                o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n_o = 3
                o0.record(stream)
                for _ in range(n_o):
                    run_o()
                o1.record(stream)
                torch.cuda.synchronize(dev)
                ms_o = o0.elapsed_time(o1) / n_o
                how = "mean of 3 back-to-back steps (inputs larger than L2)"
            check_status(status, stream)
            seqs_o = [int(x) for x in np.diff(do["cu_seqlens"])]
            flo = algorithmic_flops(seqs_o, wo.n_q_heads, wo.head_dim, wo.window)
            extras[f"step_{other}"] = {"ms": ms_o, "value": flo["total"] / (ms_o * 1e-3) / 1e12, "unit": UNIT,
                                       "pct_of_bf16_peak": 100.0 * flo["total"] / (ms_o * 1e-3) / 1e12 / peak,
                                       "keys_per_s": sum(seqs_o) * wo.n_kv_heads / (ms_o * 1e-3),
                                       "tokens": int(To), "sequences": int(len(do["cu_seqlens"]) - 1),
                                       "algorithmic_flops": flo["total"], "launches": 4, "timing": how}
            del qo, ko, lo_, to_, ko_

        # Static cache: compact this step's keep set, then one decode step over it.
        from future_attention_targets_b200 import compact_kv, decode_attention
        from future_attention_targets_b200.workloads import make_decode_inputs
        dd = make_decode_inputs(WORKLOAD, seed=rank_seed(rank))
        v = torch.from_numpy(dd["v_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
        q_dec = torch.from_numpy(dd["q_dec_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
        C = int(max(budgets))
        cache = compact_kv(k, v, keep, cu, C, stream=stream)
        dec_out = decode_attention(q_dec, cache[0], cache[1], cache[3], scale, stream=stream)
        kept_rows = int(cache[3].sum().item())

        row_bytes = w.head_dim * 2
        ms_c_flushed = timed(lambda: compact_kv(k, v, keep, cu, C, out=cache, stream=stream))
        # Eight copies of K, V and the keep mask (537 MB), compacted in turn.
        n_cp = 8
        cps = [(k.clone(), v.clone(), keep.clone(), tuple(torch.empty_like(x) for x in cache)) for _ in range(n_cp)]
        ms_c = timed_rotating([lambda st, c=c: compact_kv(c[0], c[1], c[2], cu, C, out=c[3], stream=st) for c in cps])
        for c in cps:
            assert all(torch.equal(x, y) for x, y in zip(c[3], cache)), "compaction copies disagree"
        del cps
        moved_c = keep.numel() + 2 * 2 * kept_rows * row_bytes + 4 * cache[2].numel()   # mask, K+V in and out, slots
        from future_attention_targets_b200 import decode_workspace_bytes
        ws1 = torch.empty(decode_workspace_bytes(1, w.n_q_heads, w.n_kv_heads, w.head_dim, C), dtype=torch.uint8,
                          device=dev)
        ms_d = timed(lambda: decode_attention(q_dec, cache[0], cache[1], cache[3], scale, out=dec_out[0],
                                              lse=dec_out[1], workspace=ws1, stream=stream))
        moved_d = 2 * kept_rows * row_bytes + q_dec.numel() * 2 + dec_out[0].numel() * 4
        hbm = float(peaks_x["hbm_gbs"])
        extras["compact_kv"] = {"ms": ms_c, "bound": "hbm", "achieved_gbs": moved_c / (ms_c * 1e-3) / 1e9,
                                "peak_gbs": hbm, "frac": moved_c / (ms_c * 1e-3) / 1e9 / hbm,
                                "bytes": moved_c, "rows": kept_rows,
                                "timing": f"mean of 40 back-to-back launches (one CUDA graph) over {n_cp} copies "
                                          "of the inputs (537 MB of K and V, four times the L2)",
                                "ms_l2_flushed_each": ms_c_flushed, "empty_launch_ms_flushed": floor_ms}
        extras["decode_attention"] = {"ms": ms_d, "bound": "hbm", "achieved_gbs": moved_d / (ms_d * 1e-3) / 1e9,
                                      "peak_gbs": hbm, "frac": moved_d / (ms_d * 1e-3) / 1e9 / hbm,
                                      "bytes": moved_d, "cache_slots": C}
        # The same decode step for 16 sequences at once (each a copy of this
        # cache at its own address): 264 MB of K and V, past the L2.
        nb = 16
        kc16, vc16 = cache[0].repeat(nb, 1, 1, 1), cache[1].repeat(nb, 1, 1, 1)
        cnt16, q16 = cache[3].repeat(nb, 1), q_dec.repeat(nb, 1, 1)
        out16 = decode_attention(q16, kc16, vc16, cnt16, scale, stream=stream)
        ws16 = torch.empty(decode_workspace_bytes(nb, w.n_q_heads, w.n_kv_heads, w.head_dim, C), dtype=torch.uint8,
                           device=dev)
        run_d16 = lambda: decode_attention(q16, kc16, vc16, cnt16, scale, out=out16[0], lse=out16[1],
                                           workspace=ws16, stream=stream)
        ms_d16_flushed = timed(run_d16)
        # 264.6 MB of K and V, twice the L2: back-to-back steps read them from HBM as a decode loop would
        # (the flushed figure above also pays for switching from the flush kernel to this kernel's shared
        # memory size before every step).
        for _ in range(3):
            run_d16()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(20):
            run_d16()
        d1.record(stream)
        torch.cuda.synchronize(dev)
        ms_d16 = d0.elapsed_time(d1) / 20
        moved_d16 = nb * moved_d
        # The one-sequence step back to back over the 16 copies in turn (each launch's cache is read from
        # HBM); the flushed single launch stays beside it.
        ms_d_rot = timed_rotating([lambda st, i=i: decode_attention(q16[i:i + 1], kc16[i:i + 1], vc16[i:i + 1],
                                                                    cnt16[i:i + 1], scale, out=dec_out[0],
                                                                    lse=dec_out[1], workspace=ws1, stream=st)
                                   for i in range(nb)], reps=48)
        extras["decode_attention"].update({
            "ms": ms_d_rot, "achieved_gbs": moved_d / (ms_d_rot * 1e-3) / 1e9,
            "frac": moved_d / (ms_d_rot * 1e-3) / 1e9 / hbm,
            "timing": f"mean of 48 back-to-back launches (one CUDA graph) over {nb} copies of the cache "
                      "(264.6 MB, twice the L2)",
            "ms_l2_flushed_each": ms_d, "empty_launch_ms_flushed": floor_ms})
        extras["decode_attention_batch16"] = {
            "ms": ms_d16, "bound": "hbm", "achieved_gbs": moved_d16 / (ms_d16 * 1e-3) / 1e9, "peak_gbs": hbm,
            "frac": moved_d16 / (ms_d16 * 1e-3) / 1e9 / hbm, "bytes": moved_d16, "cache_slots": C, "batch": nb,
            "timing": "mean of 20 back-to-back steps (K and V larger than L2)",
            "ms_l2_flushed_each": ms_d16_flushed}
        extras["timing"] = ("median of 20 repetitions, L2 flushed before each (a 256 MiB buffer written, then "
                            "read back so that no dirty lines remain), then a 0.1 ms device-side wait so that the "
                            "host enqueue time stays outside the interval")
        del kc16, vc16, flush

    # One problem (rank 0's layer) with its KV heads split over the ranks:
    # two passes on H_kv / P heads, one NCCL all-gather of the targets, the
    # keep mask on all heads.  Every rank takes the same collective steps.
    if world > 1 and not args.no_extras and w.n_kv_heads % world == 0:
        try:
            extras["head_sharded"] = run_head_sharded(args, w, cu, W, S, budgets, scale, world, rank, dev, stream,
                                                      fl, ms_per_step)
        except Exception as exc:   # keep the main line; every rank takes this path together or times out
            extras["head_sharded"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t, f, desc = oracle_sample(d)
        cpu = {"value": f / t / 1e12, "unit": UNIT, "cores": threads_in_use(), "kind": "oracle",
               "sample": desc, "seconds": t}

    if rank == 0:
        keys = sum(int(L) for L in np.diff(cu)) * w.n_kv_heads * world
        attn_ms = avg["row_lse"] + avg["future_target"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, world),
            "pct_of_bf16_peak": 100.0 * value / world / peak,
            "pct_of_bf16_peak_sustained": 100.0 * value / world / peak_sus,
            "keys_per_s": keys / (attn_ms * 1e-3),
            "keys_per_s_with_keep_mask": keys / ((attn_ms + avg["keep_mask"]) * 1e-3),
            # The transposed pass on its own, per GPU (its call also runs the normaliser-row kernel).
            "target_pass_only": {"value": fl["target"] / (avg["future_target"] * 1e-3) / 1e12, "unit": UNIT,
                                 "pct_of_bf16_peak": 100.0 * fl["target"] / (avg["future_target"] * 1e-3) / 1e12
                                 / peak},
            "kernel_ms": {n: round(v, 4) for n, v in avg.items()},
            "kernel_ms_median": {n: round(statistics.median(v), 4) for n, v in per_kernel.items()},
            "kernel_ms_best": {n: round(min(v), 4) for n, v in per_kernel.items()},
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": f"{peak_kind} bf16 burst",
                         "traffic": recorded_traffic(dom),
                         "algorithmic_flops_per_launch": dom_flops},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 4 * args.steps,
            "next_rows": extras,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: at least 3 warm-up steps are used", file=sys.stderr)
        args.warmup = 3
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
