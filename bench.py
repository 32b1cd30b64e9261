#!/usr/bin/env python
"""Benchmark of the W8A8 linear layer on B200.

One step = one pass of the Prefill hot path over one batch at 7B shapes:
per-token dynamic quantization of X [2048, 4096] (bf16) and the tcgen05 INT8
GEMM against the shared per-channel INT8 weight [11008, 4096] with the
dequant + bias epilogue fused in, bf16 output [2048, 11008]. The weight is
quantized once before timing (load time, not part of the step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch
(no collective on the data path: replicas, weak scaling); the timed region
is bracketed by a barrier and the slowest rank's time is reported.
--impl reference times the CPU oracle (a plain C implementation, OpenMP over
rows) on a bounded sample of the same workload.

The JSON line also carries the other rows of the path, each measured on its
own workload: "decode" (fused static-quant Decode linear, 1-32 tokens x 4096
-> 11008 / 4096, HBM-bound, CUDA-graph timed), "llm_int8" (outlier split and
mixed-decomposition GEMM at 4096 x 8192 x 8192) and "pdmix_block" (four
Llama-7B-like linears: a 4096-token Prefill pass and 64 Decode steps).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N = 2048, 4096, 11008
DEC_M, DEC_K, DEC_N = 32, 4096, 11008
N_SETS = 4          # rotating input/weight/output sets: 4 x ~115 MB > 126 MB L2
METRIC = "W8A8 linear: prefill INT8 TOPS, decode HBM GB/s (fraction of B200 peak)"
WORKLOAD = ("prefill W8A8 linear at 7B shapes: X bf16 [2048 x 4096] (row-scaled N(0,1), 6 channels x60) "
            "-> per-token symmetric INT8 quant -> INT8 GEMM vs per-channel INT8 W [4096 x 11008] "
            "-> fused dequant + bias -> bf16 [2048 x 11008]")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# INT8 dense tensor throughput is twice bf16 on B200 (4.5 vs 2.25 PFLOP/s nominal)
INT8_OVER_BF16 = 2.0

# DRAM traffic of one launch of the prefill GEMM kernel at this workload, from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum; the summary
# with its command is profiles/gemm_i8_tc2_prefill_7b_2048x4096x11008.txt).
# It describes the kernel built from these sources only: once they change, the
# bench reports no traffic until the kernel is profiled again.
TC2_TRAFFIC = {
    "bytes": 53_671_936 + 10_608_128,
    "sources": ["int8_gemm_token_b200/csrc/gemm_tc.cu", "int8_gemm_token_b200/csrc/gemm_pair.cuh",
                "int8_gemm_token_b200/csrc/device.cuh", "int8_gemm_token_b200/csrc/kernels.h"],
    "sources_sha256": "b6304937c5337acf7e6bf29ee48564866f15b528e674eaa606ab5f82a3099f29",
    "profile": "profiles/gemm_i8_tc2_prefill_7b_2048x4096x11008.txt",
}


def profiled_traffic(entry):
    """The recorded per-launch DRAM bytes if the kernel's sources are unchanged, else None."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    h = hashlib.sha256()
    try:
        for f in entry["sources"]:
            with open(os.path.join(root, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return entry["bytes"] if h.hexdigest() == entry["sources_sha256"] else None


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(backend: str):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (x itself without a process group).
    The tensor lives on `device` (a CUDA device for NCCL, the CPU for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling),
    timed by the slowest rank."""
    return world * ops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def workload_config(world: int) -> dict:
    """The `config` of the JSON line; both arms report the same one."""
    return {"workload": WORKLOAD, "M": M, "K": K, "N": N, "parallelism": f"replicas x{world}",
            "l2": f"{N_SETS} rotating X/Wq/out sets, {N_SETS * 115} MB > 126 MB L2"}


def cpu_baseline_sample(rows: int, seed: int = 0):
    """Time the oracle on `rows` tokens of the workload: per-token quant,
    int64 GEMM and the fixed-order epilogue. Returns (seconds, ops)."""
    import oracle
    from int8_gemm_token_b200 import synth
    case = synth.prefill_7b(seed)
    Wq, s_w, _ = oracle.quant_weight_per_channel(case.W)  # load time, not timed
    X = np.ascontiguousarray(case.X[:rows])
    t0 = time.perf_counter()
    Xq, S = oracle.quant_per_token(X)
    acc = oracle.gemm_i64(Xq, Wq)
    y = oracle.epilogue(acc, S, s_w, bias=case.bias)
    oracle.f32_to_bf16(y)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * N * K


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, as it stands, on a bounded sample per step."""
    if rank != 0:
        return 0
    import oracle
    rows = args.ref_rows
    times = []
    for i in range(args.warmup + args.steps):
        dt, ops = cpu_baseline_sample(rows, seed=0)
        if i >= args.warmup:
            times.append(dt)
    per = statistics.mean(times)
    value = 2.0 * rows * N * K / per / 1e12
    sample = f"{rows} of {M} tokens per step (full K={K}, N={N}); value scaled to TOPS of that sample"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic", "config": workload_config(world),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, world, rank, local):
    import torch

    from int8_gemm_token_b200 import synth
    from int8_gemm_token_b200 import w8a8 as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    int8_sustained = (peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]) * INT8_OVER_BF16

    def bf16_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    # ---------------------------------------------------------------- data
    sets = []
    for i in range(N_SETS):
        case = synth.prefill_7b(seed=1000 * rank + i)
        X = bf16_dev(case.X)
        Wq, s_w, cs = W.w8a8_quant_weight_per_channel(torch.from_numpy(case.W).to(dev))
        sets.append(dict(X=X, Wq=Wq, s_w=s_w, bias=torch.from_numpy(case.bias).to(dev),
                         Xq=torch.empty((M, K), dtype=torch.int8, device=dev),
                         S=torch.empty((M,), dtype=torch.float32, device=dev),
                         out=torch.empty((M, N), dtype=torch.bfloat16, device=dev)))
        del case
    stream = torch.cuda.current_stream()

    def step(s):
        W.w8a8_quant_per_token(s["X"], Xq=s["Xq"], S_x=s["S"], stream=stream)
        W.w8a8_gemm_dequant(s["Xq"], s["S"], s["Wq"], s["s_w"], bias=s["bias"], out=s["out"], stream=stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, dev)

    for i in range(args.warmup):
        step(sets[i % N_SETS])
    torch.cuda.synchronize()

    # ---------------------------------------------------------------- timed
    # The steps run back to back with events only at both ends: the kernels
    # use programmatic dependent launch, so each one starts under the tail of
    # the one before, and an event recorded between two kernels would stop that.
    # The clock sampler runs over this region and the per-kernel passes below.
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.__enter__()
    t0.record(stream)
    for i in range(args.steps):
        step(sets[i % N_SETS])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    total_ms = t0.elapsed_time(t1)
    ms_per_step = max_ranks(total_ms / args.steps)
    # Per-kernel durations (burst roofline, quant row): a second pass of 200
    # steps with events around each kernel, which serialises them.
    n_bd = 200
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_bd)]
    torch.cuda.synchronize()
    for i in range(n_bd):
        s = sets[i % N_SETS]
        ev[i][0].record(stream)
        W.w8a8_quant_per_token(s["X"], Xq=s["Xq"], S_x=s["S"], stream=stream)
        ev[i][1].record(stream)
        W.w8a8_gemm_dequant(s["Xq"], s["S"], s["Wq"], s["s_w"], bias=s["bias"], out=s["out"], stream=stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    quant_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    gemm_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    # Sustained: the GEMM alone, back to back for >= 1 s (the power cap sets
    # the clock there), events only at both ends.
    gemm = lambda s: W.w8a8_gemm_dequant(s["Xq"], s["S"], s["Wq"], s["s_w"], bias=s["bias"], out=s["out"],
                                         stream=stream)
    n_sus, sus_ms = 0, 0.0
    while sus_ms < 1000.0 and not args.no_sustained:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(2000):
            gemm(sets[i % N_SETS])
        b.record(stream)
        torch.cuda.synchronize()
        sus_ms += a.elapsed_time(b)
        n_sus += 2000
    clocks.__exit__()
    ops = 2.0 * M * N * K
    value = whole_job_tops(ops, world, ms_per_step)
    gemm_tops = ops / (gemm_ms * 1e-3) / 1e12
    sus_tops = ops * n_sus / (sus_ms * 1e-3) / 1e12 if n_sus else None
    quant_bytes = 2.0 * M * K + M * K + 4.0 * M
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    if W.w8a8_check_device_error() != 0:
        raise RuntimeError("device status word set during the benchmark")
    c1 = None if args.no_c1 else bench_c1(dev)

    # ---------------------------------------------------------------- e2e
    # The same step through the public API from and to pinned host memory:
    # each step copies its X in (host -> device) and its bf16 output back
    # (device -> host). Three streams with two device buffer sets let the
    # input copy of step i+1 and the output copy of step i-1 run while step i
    # computes (PCIe is full duplex); events order every buffer's reuse.
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(2 * N_SETS, min(args.steps, 50))
        nb = 2
        hostX = [sets[i]["X"].cpu().pin_memory() for i in range(N_SETS)]
        hostOut = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(N_SETS)]
        # one layer (the weight of set 0) serves every step, as in a serving loop
        bufs = [dict(sets[0], X=torch.empty_like(sets[0]["X"]), out=torch.empty_like(sets[0]["out"]))
                for _ in range(nb)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_run(n):
            copied_in = [None] * nb    # X[b] holds step i's input
            computed = [None] * nb     # out[b] holds step i's output
            drained = [None] * nb      # out[b] has been copied to the host
            used = [None] * nb         # step i's kernels have read X[b]
            for i in range(n):
                b = i % nb
                with torch.cuda.stream(s_in):
                    if used[b] is not None:
                        s_in.wait_event(used[b])
                    bufs[b]["X"].copy_(hostX[i % N_SETS], non_blocking=True)
                    copied_in[b] = torch.cuda.Event()
                    copied_in[b].record(s_in)
                stream.wait_event(copied_in[b])
                if drained[b] is not None:
                    stream.wait_event(drained[b])
                step(bufs[b])
                used[b] = computed[b] = torch.cuda.Event()
                computed[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[b])
                    hostOut[i % N_SETS].copy_(bufs[b]["out"], non_blocking=True)
                    drained[b] = torch.cuda.Event()
                    drained[b].record(s_out)
            for ev_ in drained:
                if ev_ is not None:
                    stream.wait_event(ev_)

        e2e_run(3)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_ranks(e0.elapsed_time(e1) / e2e_steps)
        ok = True
        for j in range(N_SETS):  # the last step that used input j, recomputed on the device
            ref = dict(bufs[0], X=sets[j]["X"], out=torch.empty_like(bufs[0]["out"]))
            step(ref)
            ok = ok and torch.equal(hostOut[j], ref["out"].cpu())
        e2e = {"value": whole_job_tops(ops, world, e2e_ms), "unit": "TOPS",
               "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": e2e_ms,
               "steps": e2e_steps, "outputs_match_device_run": ok,
               "timing": "pinned host X -> device, quant + GEMM, bf16 out -> pinned host, every step; input, "
                         "compute and output copies on three streams with two device buffer sets"}
        del bufs

    del sets
    torch.cuda.empty_cache()
    # ---------------------------------------------------------------- the other rows of the path
    decode = llm = block = kv = None
    quant_stream = None if args.no_quant_stream else bench_quant_stream(dev, peaks)
    if not args.no_decode:
        decode = bench_decode(args, dev, rank, peaks)
        kv = bench_kv_cache(dev, peaks)
    if not args.no_llm_int8:
        llm = bench_llm_int8(args, dev, rank, peaks, int8_peak)
    if not args.no_block:
        block = bench_block(args, dev, rank, peaks, int8_peak)
    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            dt, sops = cpu_baseline_sample(8)
            rows = int(min(M, max(8, 8 * args.cpu_seconds / max(dt, 1e-3))))
            dt, sops = cpu_baseline_sample(rows)
            cpu = {"value": sops / dt / 1e12, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                   "sample": f"{rows} of {M} tokens (full K={K}, N={N}), quant + int64 GEMM + epilogue, {dt:.1f} s"}
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": workload_config(world),
            "roofline": {"bound": "tensor", "kernel": "gemm_i8_tc2_kernel", "achieved": gemm_tops,
                         "peak": int8_peak, "unit": "TOPS", "frac": gemm_tops / int8_peak,
                         "peak_source": f"{peaks['source']} burst bf16 {peaks['bf16_tflops']} TFLOP/s x 2 "
                                        "(int8/bf16 nominal ratio); the kernel is timed in 200 launches with "
                                        "events around each",
                         "traffic": profiled_traffic(TC2_TRAFFIC), "traffic_unit": "B per launch",
                         "traffic_profile": TC2_TRAFFIC["profile"],
                         "algorithmic_ops": ops,
                         "algorithmic_bytes": M * K + N * K + 2 * M * N + 4 * M + 8 * N,
                         "sustained": None if sus_tops is None else {
                             "achieved": sus_tops, "peak": int8_sustained, "frac": sus_tops / int8_sustained,
                             "launches": n_sus, "ms": sus_ms,
                             "peak_source": f"{peaks['source']} sustained bf16 {peaks['bf16_tflops_sustained']} "
                                            "TFLOP/s x 2; the GEMM alone back to back for >= 1 s"}},
            "quant": {"kernel": "quant_per_token_kernel", "ms": quant_ms, "achieved": quant_gbs,
                      "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": quant_gbs / peaks["hbm_gbs"],
                      "C_s_over_C_g": quant_ms / gemm_ms, "timing": "events around each launch in the step",
                      "stream": quant_stream},
            "gemm_ms": gemm_ms,
            "prefill_small": c1,
            "decode": decode,
            "kv_cache": kv,
            "llm_int8": llm,
            "pdmix_block": block,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 2 * args.steps,
            "timing": {"value": "K back-to-back steps between two CUDA events (kernels overlap through "
                                "programmatic dependent launch)",
                       "per_kernel": f"{n_bd} further steps with events around each kernel (serialised); "
                                     "roofline.achieved and quant use these",
                       "clocks": "NVML samples every 2 ms over the timed steps, the per-kernel pass and the "
                                 ">= 1 s sustained GEMM pass"},
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    return 0


def graph_time_us(fn, n_calls, reps=10):
    """Per-call device time of fn(i), i < n_calls, captured once in a CUDA
    graph and replayed `reps` times between two events (no host overhead)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(min(3, n_calls)):
            fn(i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n_calls):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) * 1e3 / (reps * n_calls)


def bench_c1(dev):
    """The small single-linear Prefill workload (16 tokens x 256 -> 512, seed
    0): per-token quantization + GEMM + dequant, launch-latency bound. Per
    call: back to back in a CUDA graph, and one call with events around it."""
    import torch

    from int8_gemm_token_b200 import synth
    from int8_gemm_token_b200 import w8a8 as W
    case = synth.prefill_small(0)
    X = torch.from_numpy(case.X.view(np.int16)).view(torch.bfloat16).to(dev)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(torch.from_numpy(case.W).to(dev))
    bias = torch.from_numpy(case.bias).to(dev)
    Xq = torch.empty((16, 256), dtype=torch.int8, device=dev)
    S = torch.empty((16,), dtype=torch.float32, device=dev)
    out = torch.empty((16, 512), dtype=torch.bfloat16, device=dev)

    def call(i):
        W.w8a8_quant_per_token(X, Xq=Xq, S_x=S)
        W.w8a8_gemm_dequant(Xq, S, Wq, s_w, bias=bias, out=out)
    graph_us = graph_time_us(call, 20)
    single = []
    for _ in range(50):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        call(0)
        b.record()
        torch.cuda.synchronize()
        single.append(a.elapsed_time(b) * 1e3)
    return {"workload": "prefill single linear: X bf16 [16 x 256] row-scaled N(0,1) -> per-token quant -> INT8 "
                        "GEMM vs W [256 x 512] + bias -> bf16 [16 x 512]",
            "us_per_linear_graph": graph_us, "us_per_linear_single_call_median": statistics.median(single),
            "ops": 2.0 * 16 * 256 * 512, "bound": "launch latency (4.2 MOP, 8 KB of activation)"}


def bench_quant_stream(dev, peaks):
    """Per-token quantization alone: per-launch device time of back-to-back
    launches in a CUDA graph, inputs and outputs rotated over > 2x L2, at the
    step's shape and at the block's widest input (4096 tokens x 11008). One
    event pair around a single 25 MB launch mostly measures its launch and
    ramp; this measures the kernel's streaming rate."""
    import torch

    from int8_gemm_token_b200 import w8a8 as W
    rows = []
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    for (Mq, Kq) in ((M, K), (4096, 11008)):
        per = 3.0 * Mq * Kq
        n = max(3, int(400e6 // per) + 1)
        # rows of N(0,1) scaled by exp(N(0, 0.5)), as the step's activations
        X0 = (torch.randn((Mq, Kq), device=dev, generator=g)
              * torch.exp(0.5 * torch.randn((Mq, 1), device=dev, generator=g))).to(torch.bfloat16)
        Xs = [X0.clone() for _ in range(n)]
        Xqs = [torch.empty((Mq, Kq), dtype=torch.int8, device=dev) for _ in range(n)]
        Ss = [torch.empty((Mq,), dtype=torch.float32, device=dev) for _ in range(n)]
        us = graph_time_us(lambda i: W.w8a8_quant_per_token(Xs[i % n], Xq=Xqs[i % n], S_x=Ss[i % n]), 2 * n)
        nbytes = 2.0 * Mq * Kq + Mq * Kq + 4.0 * Mq
        gbs = nbytes / (us * 1e-6) / 1e9
        rows.append({"M": Mq, "K": Kq, "us": us, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]})
        del Xs, Xqs, Ss, X0
    torch.cuda.empty_cache()
    return {"workload": "quant_per_token_kernel alone, back-to-back launches in a CUDA graph, inputs and outputs "
                        "rotated over > 400 MB", "rows": rows, "unit": "GB/s", "peak": peaks["hbm_gbs"],
            "algorithmic_bytes": "2MK + MK + 4M per launch"}


def bench_kv_cache(dev, peaks):
    """INT8 KV cache kept in the Decode scheme: writing one cache tensor
    (bf16 -> codes, w8a8_quant_per_tensor) and reading it back (codes -> bf16,
    w8a8_dequant_per_tensor), 8192 tokens x 4096 (32 heads x 128), back to
    back in a CUDA graph over tensors rotated beyond L2."""
    import torch

    from int8_gemm_token_b200 import w8a8 as W
    T, D = 8192, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    X0 = (torch.randn((T, D), device=dev, generator=g)
          * torch.exp(0.5 * torch.randn((T, 1), device=dev, generator=g))).to(torch.bfloat16)
    S, r, Z = W.w8a8_calibrate_static(X0[:512])
    n = 4
    Xs = [X0.clone() for _ in range(n)]
    Qs = [W.w8a8_quant_per_tensor(x, r, Z) for x in Xs]
    del X0
    write_us = graph_time_us(lambda i: W.w8a8_quant_per_tensor(Xs[i % n], r, Z, Xq=Qs[i % n]), 2 * n)
    read_us = graph_time_us(lambda i: W.w8a8_dequant_per_tensor(Qs[i % n], S, Z, out=Xs[i % n]), 2 * n)
    nbytes = 3.0 * T * D
    rows = []
    for name, us in (("write (quant_per_tensor)", write_us), ("read (dequant_per_tensor)", read_us)):
        gbs = nbytes / (us * 1e-6) / 1e9
        rows.append({"op": name, "tokens": T, "width": D, "us": us, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]})
    del Xs, Qs
    torch.cuda.empty_cache()
    return {"workload": "INT8 KV cache tensor, 8192 tokens x 4096, static per-tensor scheme; graph-timed, "
                        "4 rotating tensors (> 2x L2 with their codes)", "rows": rows, "unit": "GB/s",
            "peak": peaks["hbm_gbs"], "algorithmic_bytes": "3 * tokens * width per call"}


def bench_decode(args, dev, rank, peaks):
    """Fused static-quant Decode linear (PDMIX decode: per-tensor static
    asymmetric quant + INT8 GEMM + zero-point corrected epilogue), for the
    token counts and weight shapes of the Decode workload, weights rotated so
    every call streams its weight from HBM; graph-timed."""
    import torch

    from int8_gemm_token_b200 import synth
    from int8_gemm_token_b200 import w8a8 as W

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    rows, requant = [], []
    for N in (11008, 4096):
        case = synth.decode_static(M=32, N=N, K=DEC_K, seed=rank)
        S, r, Z = W.w8a8_calibrate_static(bf(case.Xcal))
        Wq, s_w, cs = W.w8a8_quant_weight_per_channel(torch.from_numpy(case.W).to(dev))
        n_w = max(3, int(600e6 // (N * DEC_K)) + 1)
        ws = [(Wq.clone(), s_w.clone(), cs.clone()) for _ in range(n_w)]
        Xall = bf(case.X)
        for M in (32, 16, 4, 1):
            X = Xall[:M].contiguous()
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            work = W.new_workspace(M, N, DEC_K, device=dev)
            us = graph_time_us(lambda i: W.w8a8_linear_static(X, S, r, Z, *ws[i % n_w], out=out, workspace=work), 2 * n_w)
            nbytes = N * DEC_K + 8.0 * N + 2.0 * M * DEC_K + 2.0 * M * N
            gbs = nbytes / (us * 1e-6) / 1e9
            rows.append({"M": M, "K": DEC_K, "N": N, "us": us, "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]})
            # the int8 codes of the next linear straight from the epilogue, vs
            # the bf16 output followed by the static quantization kernel (the
            # next linear's r, Z stood in by this one's: same arithmetic)
            q = torch.empty((M, N), dtype=torch.int8, device=dev)
            rq_us = graph_time_us(lambda i: W.w8a8_linear_static_requant(X, S, r, Z, *ws[i % n_w], r, Z, out=q,
                                                                         workspace=work), 2 * n_w)

            def pair(i):
                W.w8a8_linear_static(X, S, r, Z, *ws[i % n_w], out=out, workspace=work)
                W.w8a8_quant_per_tensor(out, r, Z, Xq=q)
            pair_us = graph_time_us(pair, 2 * n_w)
            rq_bytes = N * DEC_K + 8.0 * N + 2.0 * M * DEC_K + 1.0 * M * N
            rq_gbs = rq_bytes / (rq_us * 1e-6) / 1e9
            requant.append({"M": M, "K": DEC_K, "N": N, "us": rq_us, "GB/s": rq_gbs, "frac": rq_gbs / peaks["hbm_gbs"],
                            "unfused_us": pair_us})
        del ws
    # static quant alone vs GEMM alone (the C_s / C_g of the PDMIX cost model) at the largest shape
    return {"workload": "decode: static-quant W8A8 linear, w8a8_linear_static (one kernel with the quantization fused "
                        "into the weight-streaming GEMM for M <= 16 or N <= 4096, else quantization kernel + GEMM), "
                        "back-to-back calls, rotating weights > L2, CUDA-graph timed", "rows": rows,
            "unit": "GB/s", "peak": peaks["hbm_gbs"], "algorithmic_bytes": "N*K + 8N + 2MK + 2MN per call",
            "requant": {"workload": "w8a8_linear_static_requant: the same Decode linear writing the next linear's "
                                    "static int8 codes from its epilogue; unfused_us = w8a8_linear_static (bf16) + "
                                    "w8a8_quant_per_tensor", "rows": requant,
                        "algorithmic_bytes": "N*K + 8N + 2MK + MN per call"}}


def bench_llm_int8(args, dev, rank, peaks, int8_peak):
    """LLM.int8() mode at 4096 x 8192 x 8192: the outlier split, and the mixed
    GEMM with the side product on CUDA cores (fixed-order fmaf chain) and on
    the tensor cores, at the workload's own 6-8 outlier columns and with 64
    and 512 planted ones; the plain pair GEMM of the same shape for scale."""
    import torch

    from int8_gemm_token_b200 import synth
    from int8_gemm_token_b200 import w8a8 as W
    case = synth.llm_int8(seed=rank)
    bf = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    X, Wd = bf(case.X), bf(case.W)
    Mq, Kq = case.X.shape
    Nq = case.W.shape[1]
    ops = 2.0 * Mq * Nq * Kq
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq = torch.empty((Mq, Kq), dtype=torch.int8, device=dev)
    S = torch.empty((Mq,), dtype=torch.float32, device=dev)
    out = torch.empty((Mq, Nq), dtype=torch.bfloat16, device=dev)
    wsb = torch.zeros((W.lib().int8_outlier_split_workspace_size(Kq),), dtype=torch.uint8, device=dev)
    res = {"workload": f"LLM.int8() X [{Mq} x {Kq}], W bf16 [{Kq} x {Nq}], threshold 6.0", "rows": []}
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    for label in ("workload", 64, 512):
        if label == "workload":
            Xl, cap = X, 64
        else:  # N(0,1) clipped to +-5.5 with `label` planted columns of random sign x U(20, 100)
            cap = label
            Xl = torch.randn((Mq, Kq), device=dev, generator=g).clamp_(-5.5, 5.5)  # only planted columns exceed 6
            cols = torch.randperm(Kq, device=dev, generator=g)[:label]
            mag = 20.0 + 80.0 * torch.rand((Mq, label), device=dev, generator=g)
            sign = torch.where(torch.rand((Mq, label), device=dev, generator=g) < 0.5, -1.0, 1.0)
            Xl[:, cols] = sign * mag
            Xl = Xl.to(torch.bfloat16)
        idx = torch.empty((cap,), dtype=torch.int32, device=dev)
        n_out = torch.empty((1,), dtype=torch.int32, device=dev)
        Xo = torch.empty((Mq, cap), dtype=torch.bfloat16, device=dev)
        split = lambda i: W.int8_outlier_split(Xl, case.threshold, cap, Xq=Xq, S_x=S, idx=idx, n_out=n_out, Xo=Xo,
                                               workspace=wsb)
        split_us = graph_time_us(split, 4)
        n = int(n_out.item())
        cuda_us = graph_time_us(lambda i: W.int8_mixed_decomp_gemm(Xq, S, Xo, idx, n_out, cap, Wq, s_w, Wd, out=out),
                                4, reps=3 if n > 64 else 10)
        tc_us = graph_time_us(lambda i: W.int8_mixed_decomp_gemm_tc(Xq, S, Xo, idx, n_out, cap, Wq, s_w, Wd, out=out), 4)
        split_bytes = 2.0 * Mq * Kq + Mq * Kq + 4.0 * Mq + 2.0 * Mq * n
        res["rows"].append({"outlier_columns": n, "cap": cap,
                            "split_us": split_us, "split_GB/s": split_bytes / (split_us * 1e-6) / 1e9,
                            "split_frac_hbm": split_bytes / (split_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                            "mixed_cuda_core_side_us": cuda_us,
                            "mixed_cuda_core_side_frac_int8": ops / (cuda_us * 1e-6) / 1e12 / int8_peak,
                            "mixed_tensor_core_side_us": tc_us,
                            "mixed_tensor_core_side_frac_int8": ops / (tc_us * 1e-6) / 1e12 / int8_peak})
        if label == "workload":
            res.update({"outlier_columns": n, "split_us": split_us,
                        "split_frac_hbm": res["rows"][0]["split_frac_hbm"], "split_algorithmic_bytes": split_bytes})
        del Xl
    # the plain pair GEMM of the same shape (no side product), for the overhead of the side path
    plain_us = graph_time_us(lambda i: W.w8a8_gemm_dequant(Xq, S, Wq, s_w, out=out), 4)
    res["plain_gemm_us"] = plain_us
    res["plain_gemm_frac_int8"] = ops / (plain_us * 1e-6) / 1e12 / int8_peak
    for r in res["rows"]:
        r["tensor_core_side_over_plain"] = r["mixed_tensor_core_side_us"] / plain_us
        r["cuda_core_side_over_plain"] = r["mixed_cuda_core_side_us"] / plain_us
    assert W.w8a8_check_device_error() == 0
    return res


def bench_block(args, dev, rank, peaks, int8_peak):
    """PDMIX block sequence (Llama-7B-like linears): one Prefill pass of 4096
    tokens (per-token quant + GEMM per linear) and 64 Decode steps of 32 tokens
    (fused static-quant linear per linear), one INT8 weight per linear shared
    by both phases; decode steps captured in one CUDA graph."""
    import torch

    from int8_gemm_token_b200 import synth
    from int8_gemm_token_b200 import w8a8 as W
    bf = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    lin = synth.pdmix_block(seed=rank)
    layers = []
    for L_ in lin:
        Wq, s_w, cs = W.w8a8_quant_weight_per_channel(torch.from_numpy(L_.weight()).to(dev))
        S, r, Z = W.w8a8_calibrate_static(bf(L_.calibration()))
        Xp = bf(L_.prefill_input(4096))
        dec = torch.stack([bf(L_.decode_input(step, 32)) for step in range(64)])
        layers.append(dict(K=L_.K, N=L_.N, Wq=Wq, s_w=s_w, cs=cs, S=S, r=r, Z=Z, Xp=Xp, dec=dec,
                           Xq=torch.empty((4096, L_.K), dtype=torch.int8, device=dev),
                           Sx=torch.empty((4096,), dtype=torch.float32, device=dev),
                           outp=torch.empty((4096, L_.N), dtype=torch.bfloat16, device=dev),
                           outd=torch.empty((32, L_.N), dtype=torch.bfloat16, device=dev),
                           work=W.new_workspace(32, L_.N, L_.K, device=dev)))
    stream = torch.cuda.current_stream()
    # prefill: events around each kernel, a few repetitions
    q_ms = g_ms = 0.0
    reps = 5
    for rep in range(reps + 2):
        evs = []
        for Ly in layers:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            W.w8a8_quant_per_token(Ly["Xp"], Xq=Ly["Xq"], S_x=Ly["Sx"])
            e[1].record(stream)
            W.w8a8_gemm_dequant(Ly["Xq"], Ly["Sx"], Ly["Wq"], Ly["s_w"], out=Ly["outp"])
            e[2].record(stream)
            evs.append(e)
        torch.cuda.synchronize()
        if rep >= 2:
            q_ms += sum(e[0].elapsed_time(e[1]) for e in evs) / reps
            g_ms += sum(e[1].elapsed_time(e[2]) for e in evs) / reps
    prefill_ops = sum(2.0 * 4096 * Ly["K"] * Ly["N"] for Ly in layers)
    # the whole Prefill pass back to back (events only at both ends, so the
    # kernels overlap through programmatic dependent launch)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for rep in range(reps):
        for Ly in layers:
            W.w8a8_quant_per_token(Ly["Xp"], Xq=Ly["Xq"], S_x=Ly["Sx"])
            W.w8a8_gemm_dequant(Ly["Xq"], Ly["Sx"], Ly["Wq"], Ly["s_w"], out=Ly["outp"])
    b.record(stream)
    torch.cuda.synchronize()
    pass_ms = a.elapsed_time(b) / reps

    def decode_all(step):
        for Ly in layers:
            W.w8a8_linear_static(Ly["dec"][step], Ly["S"], Ly["r"], Ly["Z"], Ly["Wq"], Ly["s_w"], Ly["cs"],
                                 out=Ly["outd"], workspace=Ly["work"])
    step_us = graph_time_us(decode_all, 64, reps=3)
    w_bytes = sum(Ly["K"] * Ly["N"] for Ly in layers)
    # the PDMIX cost model: static quant alone vs the decode GEMM alone, per step
    dq_us = graph_time_us(lambda i: [W.w8a8_quant_per_tensor(Ly["dec"][i % 64], Ly["r"], Ly["Z"], Xq=Ly["Xq"][:32]) for Ly in layers], 16)
    assert W.w8a8_check_device_error() == 0
    return {"workload": "PDMIX block: QKV 4096->12288, O 4096->4096, gate+up 4096->22016, down 11008->4096; "
                        "prefill 4096 tokens, then 64 decode steps x 32 tokens",
            "prefill_us": pass_ms * 1e3, "prefill_TOPS": prefill_ops / (pass_ms * 1e-3) / 1e12,
            "prefill_kernels_serialised_us": (q_ms + g_ms) * 1e3,
            "prefill_gemm_frac_int8": prefill_ops / (g_ms * 1e-3) / 1e12 / int8_peak,
            "prefill_C_s_over_C_g": q_ms / g_ms,
            "decode_total_us": 64 * step_us, "decode_step_us": step_us,
            "decode_weight_GB/s": w_bytes / (step_us * 1e-6) / 1e9,
            "decode_frac_hbm": w_bytes / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
            "decode_static_quant_us_per_step": dq_us,
            "decode_C_s_over_C_g": dq_us / max(step_us - dq_us, 1e-9)}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-llm-int8", action="store_true")
    ap.add_argument("--no-block", action="store_true")
    ap.add_argument("--no-quant-stream", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sustained", action="store_true")
    ap.add_argument("--no-c1", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-rows", type=int, default=16)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.impl == "reference":
        world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
        return run_reference(args, world, rank)
    world, rank, local = dist_setup("nccl")
    try:
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
