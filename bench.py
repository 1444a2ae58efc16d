#!/usr/bin/env python
"""Benchmark of the BitLinear W1.58·A8 decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Workload (default): one 7B-shaped decoder layer set at M = 1 token — q, k, v, o
(4096→4096), gate, up (4096→11008), down (11008→4096) — each with its own
bfloat16 input (0.1% ×20 outlier channels) and W ~ N(0, 0.02) weights that are
absmean-ternarised once (not timed).  One step = the whole path over that set:
per-token int8 activation quantisation of the seven inputs (one grouped
launch) and the ternary GEMV + dequant of the seven matrices (one grouped
launch), issued as one bitlinear_linear_grouped call (weights flagged static)
whose kernels chain by programmatic dependent launch: each step's GEMV starts
streaming its weights while the previous step drains.  The metric is algorithmic HBM
bytes per step ÷ time per step.

Timing: W warm-up steps, then exactly K steps captured in one CUDA graph and
replayed between a barrier + synchronize on both sides, timed with CUDA events
on the replay stream (no events inside the graph: they would break the
overlap of consecutive steps).  Weight copies rotate across steps so every step reads its weights from
HBM (the replicas together exceed 4× the L2).  Multi-GPU: one process per GPU,
each runs its own replica of the workload (weak scaling, no data-path
collective); the step time is the max over ranks.

Prefill leg (same JSON line, key "prefill"): M = 2048 tokens through the three
prefill shapes (K, N) = (4096, 4096), (4096, 11008), (11008, 4096), bf16 inputs
with outliers; one step = one bitlinear_linear_grouped call over the three
(grouped act quant + one tcgen05 int8 GEMM launch per matrix), K steps in one
CUDA graph.  Its roofline is the GEMM's int8 TOPS (each launch timed with CUDA
events, the three shapes rotating) against the measured bf16 tensor peak × 2.

``--impl reference`` times the CPU oracle (the method written out in plain C)
on the host cores over a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time
import hashlib

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMV HBM GB/s (% of 8 TB/s); prefill int8 TOPS (% of peak)"
GEMV_SOURCES = ("gemv_ternary.cu", "bl_ptx.cuh", "bl_common.cuh")
GEMM_SOURCES = ("gemm_tcgen05.cu", "bl_ptx.cuh", "bl_common.cuh")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------- workload
def workload_specs():
    from bitlinear_w1_a8_03_b200 import workloads
    return workloads.decode_7b_layer_set(M=1)


def bytes_per_step(specs) -> int:
    """Algorithmic HBM bytes of one step: the packed weights once, plus the
    activation quantisation (x bf16 in, x̃ + β out) and the GEMV's x̃ + β in and
    fp32 y out, for every matrix."""
    total = 0
    for s in specs:
        rb = 16 * ((s.K + 63) // 64)
        total += s.N * rb                      # packed ternary weights
        total += s.M * s.K * 2 + s.M * s.K + 4 * s.M   # act quant: x in, x̃ out, β out
        total += s.M * s.K + 4 * s.M + 4 * s.M * s.N   # GEMV: x̃, β in; y out
    return total


def prefill_specs():
    from bitlinear_w1_a8_03_b200 import workloads
    return [workloads.prefill(4096, 4096), workloads.prefill(4096, 11008), workloads.prefill(11008, 4096)]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_sources_sha256(sources) -> str | None:
    """sha256 over the kernel's source file and the device headers it includes,
    in the order given (the key a recorded ncu traffic figure is valid for)."""
    m = hashlib.sha256()
    for name in sources:
        src = os.path.join(ROOT, "bitlinear_w1_a8_03_b200", "csrc", name)
        if not os.path.exists(src):
            return None
        m.update(open(src, "rb").read())
    return m.hexdigest()


def recorded_traffic(kernel_tag: str, sources):
    """DRAM bytes per launch recorded from an ncu capture in profiles/, valid
    only while the kernel's sources are unchanged (sha256 recorded beside it)."""
    sha = kernel_sources_sha256(sources)
    pdir = os.path.join(ROOT, "profiles")
    if sha is None or not os.path.isdir(pdir):
        return None
    pat = re.compile(rf"^traffic\[{re.escape(kernel_tag)}\]:\s*(\d+)\s+bytes/launch\s+source_sha256:\s*([0-9a-f]+)", re.M)
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".md", ".txt")):
            continue
        for m in pat.finditer(open(os.path.join(pdir, name), encoding="utf-8").read()):
            if m.group(2) == sha:
                return int(m.group(1))
    return None


def decode_config(specs) -> dict:
    """The decode workload's config, identical in the native and reference arms."""
    return {
        "workload": "7B decode layer set, M=1: q,k,v,o 4096->4096; gate,up 4096->11008; down 11008->4096",
        "bytes_per_step": bytes_per_step(specs),
        "weight_bytes_per_step": sum(s.N * 16 * ((s.K + 63) // 64) for s in specs),
        "l2": "inputs larger than L2: weight replicas rotate across steps, together more than 4x the L2",
        "parallelism": "replicas (one independent replica of the workload per GPU, weak scaling)",
    }


def kernels_per_call(fn, stream) -> int:
    """CUDA kernels one eager call of fn launches, counted by the torch
    profiler outside any timed region (the library picks launch shapes at
    run time, e.g. one act-quant launch per CTA size)."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    stream.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        with torch.cuda.stream(stream):
            fn()
        stream.synchronize()
    return sum(1 for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA)


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values, device, world: int):
    """Element-wise max of per-rank timings (ms) over all ranks; identity at N=1."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def replica_throughput(units_per_rank: float, max_ms: float, world: int) -> float:
    """Whole-job units per second: every rank runs its own replica of the same
    work (weak scaling), timed as the slowest rank."""
    return world * units_per_rank / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sms, maxes, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


def gpu_id(props, local_rank) -> str:
    return "GPU-" + str(props.uuid) if hasattr(props, "uuid") else str(local_rank)


SETTLE_SECONDS = 1.0  # --settle-seconds; 0 only for profiler runs, whose numbers are not bench values


def settle(stream, replay, props, local_rank, seconds: float | None = None) -> ClockSampler:
    """Starts the clock sampler, then runs about `seconds` of identical replays
    so the timed region that follows runs at settled clocks; the caller stops
    the sampler after its timed region (and a few more replays)."""
    import torch
    sampler = ClockSampler(gpu_id(props, local_rank))
    t_end = time.time() + (SETTLE_SECONDS if seconds is None else seconds)
    with torch.cuda.stream(stream):
        while time.time() < t_end:
            replay()
            stream.synchronize()
    return sampler


# ----------------------------------------------------------------------------- native arm
def run_native(args, rank, world, local_rank):
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    specs = workload_specs()

    # weights: generate, quantise once on the device (cached, not timed)
    packed0, alphas = [], []
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        p, a = bl.bitlinear_quantize_weights(W)
        packed0.append(p)
        alphas.append(a)
        del W
    torch.cuda.synchronize()
    set_bytes = sum(p.numel() for p in packed0)
    replicas = max(2, math.ceil(4 * props.L2_cache_size / set_bytes) + 1)
    packed = [packed0] + [[p.clone() for p in packed0] for _ in range(replicas - 1)]

    # inputs (bf16, M = 1) in one buffer so the end-to-end leg copies them at once
    x_host = np.concatenate([synth.f32_to_bf16_bits(synth.activations(s.x_seed, s.M, s.K, outliers=s.outliers)).ravel()
                             for s in specs])
    x_dev = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).to(dev)
    xs, xq, beta, ys = [], [], [], []
    y_dev = torch.empty(sum(s.M * s.N for s in specs), dtype=torch.float32, device=dev)
    ox = oy = 0
    for s in specs:
        xs.append(x_dev[ox:ox + s.M * s.K].view(s.M, s.K))
        xq.append(torch.empty((s.M, s.K), dtype=torch.int8, device=dev))
        beta.append(torch.empty(s.M, dtype=torch.float32, device=dev))
        ys.append(y_dev[oy:oy + s.M * s.N].view(s.M, s.N))
        ox += s.M * s.K
        oy += s.M * s.N
    lin_arrs = [bl.make_linear_problems([dict(x=xs[i], x_q=xq[i], beta=beta[i], W_packed=packed[r][i],
                                              alpha=alphas[i], N=s.N, y=ys[i]) for i, s in enumerate(specs)])
                for r in range(replicas)]
    L = bl.lib()
    nprob = len(specs)

    def step(i, stream_handle, ev=None):
        if ev is not None:
            ev[0].record()
        bl.check(L.bitlinear_linear_grouped(lin_arrs[i % replicas], nprob, bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                            stream_handle), "linear")
        if ev is not None:
            ev[1].record()

    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):  # first calls also initialise the library's caches
            step(i, sh)
    stream.synchronize()

    K = args.steps
    g_warm, g_timed = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        for i in range(replicas):
            step(i, sh)
    with torch.cuda.graph(g_timed, stream=stream):
        for i in range(K):
            step(i, sh)

    # warm-up: W steps in the graph form, one untimed replay of the timed graph
    # (its first launch also uploads it to the device), then ≈1 s of identical
    # replays while the clock sampler runs
    with torch.cuda.stream(stream):
        for _ in range(max(1, math.ceil(args.warmup / replicas))):
            g_warm.replay()
        g_timed.replay()
    stream.synchronize()
    sampler = settle(stream, g_warm.replay, props, local_rank)

    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g_timed.replay()
        t1.record()
    t1.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    # a little more identical load for the clock window, then stop sampling
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_warm.replay()
    stream.synchronize()
    clocks = sampler.stop()

    # end to end through the C ABI with host buffers: every step is one
    # bitlinear_linear_grouped_host call that copies the step's inputs from
    # pinned host memory, runs the linear and copies the results back (one
    # merged copy each way). Steps rotate over three streams with their own
    # buffers, so a step's copies overlap the other steps' kernels.
    NB = 3
    x_pinned = [torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory() for _ in range(NB)]
    y_pinned = [torch.empty(y_dev.numel(), dtype=torch.float32).pin_memory() for _ in range(NB)]
    x_dev2 = [x_dev] + [torch.empty_like(x_dev) for _ in range(NB - 1)]
    y_dev2 = [y_dev] + [torch.empty_like(y_dev) for _ in range(NB - 1)]
    xq2 = [xq] + [[torch.empty_like(t) for t in xq] for _ in range(NB - 1)]
    beta2 = [beta] + [[torch.empty_like(t) for t in beta] for _ in range(NB - 1)]

    def e2e_problems(bi, r):
        out, io, ox, oy = [], [], 0, 0
        for i, s in enumerate(specs):
            out.append(dict(x=x_dev2[bi][ox:ox + s.M * s.K].view(s.M, s.K), x_q=xq2[bi][i], beta=beta2[bi][i],
                            W_packed=packed[r][i], alpha=alphas[i], N=s.N, y=y_dev2[bi][oy:oy + s.M * s.N].view(s.M, s.N)))
            io.append((x_pinned[bi][ox:ox + s.M * s.K], y_pinned[bi][oy:oy + s.M * s.N]))
            ox += s.M * s.K
            oy += s.M * s.N
        return bl.make_linear_problems(out), bl.make_host_io(io)
    e2e_arr = [[e2e_problems(bi, r) for r in range(replicas)] for bi in range(NB)]
    e2e_streams = [torch.cuda.Stream(device=dev) for _ in range(NB)]

    def e2e_step(i):
        bi = i % NB
        arr, io = e2e_arr[bi][i % replicas]
        bl.check(L.bitlinear_linear_grouped_host(arr, io, nprob, bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                                 e2e_streams[bi].cuda_stream), "linear_host")

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(e2e_streams[0])
    for s_ in e2e_streams[1:]:
        s_.wait_event(e0)
    for i in range(K):
        e2e_step(i)
    for s_ in e2e_streams[1:]:
        e2e_streams[0].wait_stream(s_)
    e1.record(e2e_streams[0])
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], dev, world)

    bps = bytes_per_step(specs)
    value = replica_throughput(bps * K, elapsed_ms, world) / 1e9
    e2e_value = replica_throughput(bps * K, e2e_ms, world) / 1e9
    # one launch per step (the fused GEMV; consecutive steps overlap by PDL),
    # so the per-launch duration is the timed region over K (an upper bound)
    kavg = elapsed_ms / K
    achieved = bps / (kavg * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    traffic = recorded_traffic("gemv_stream:decode7b", GEMV_SOURCES)
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / K, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 x ternary(2-bit) -> int32, fp32 dequant",
        "data": "synthetic (seeded SplitMix64/Box-Muller; W ~ N(0,0.02) ternarised once, x bf16 ~ N(0,1) + 0.1% x20 outliers)",
        "config": decode_config(specs),
        "timing": {
            "l2": f"{replicas} rotating weight replicas, {replicas * set_bytes / 1e6:.0f} MB "
                  f"(L2 {props.L2_cache_size / 1e6:.0f} MB)",
            "launch": "K steps captured in one CUDA graph; per step one bitlinear_linear_grouped call "
                      "(BL_LINEAR_WEIGHTS_STATIC) = one fused quantise + GEMV launch, steps chained by PDL",
            "pct_of_8TBps": round(100 * value / world / 8000.0, 2),
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "gemv_stream_kernel<1, fused> (one bitlinear_linear_grouped call over the 7 matrices = one "
                      "launch that quantises its inputs in its prologue; consecutive steps chained by PDL)",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json copy bandwidth)" if peak_src == "measured"
                           else "fallback 6650 GB/s",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "bytes_per_launch": bps,
            "avg_launch_us": round(kavg * 1e3, 3),
        },
        "e2e": {
            "value": round(e2e_value, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": int(x_host.nbytes),
            "d2h_bytes_per_step": int(y_dev.numel() * 4),
            "how": "per step one C-ABI call with host buffers, bitlinear_linear_grouped_host: pinned x -> device "
                   "(one merged copy), the grouped linear, y -> pinned host (one merged copy); steps rotate "
                   "over three streams with their own buffers",
        },
        "gpu_launches": K,
        "clocks": clocks,
    }
    return result


# ----------------------------------------------------------------------------- prefill leg
def run_prefill(args, world, local_rank):
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    specs = prefill_specs()
    probs, fwd = [], []
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        p, a = bl.bitlinear_quantize_weights(W)
        del W
        xb = synth.f32_to_bf16_bits(synth.activations(s.x_seed, s.M, s.K, outliers=s.outliers))
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        pr = dict(x=x, x_q=torch.empty((s.M, s.K), dtype=torch.int8, device=dev),
                  beta=torch.empty(s.M, dtype=torch.float32, device=dev), W_packed=p, alpha=a, N=s.N,
                  y=torch.empty((s.M, s.N), dtype=torch.float32, device=dev))
        probs.append(pr)
    torch.cuda.synchronize()
    ops = [2 * s.M * s.N * s.K for s in specs]
    L = bl.lib()
    arr = bl.make_linear_problems(probs)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step():
        bl.check(L.bitlinear_linear_grouped(arr, len(specs), bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC, sh), "linear")

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            step()
    stream.synchronize()
    launches_per_step = kernels_per_call(step, stream)
    K = args.steps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(K):
            step()
    with torch.cuda.stream(stream):
        g.replay()  # warm replay (W steps already ran eagerly)
    stream.synchronize()
    sampler = settle(stream, g.replay, props, local_rank)  # ≈1 s of identical steps under the clock sampler
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    t1.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = max_over_ranks([t0.elapsed_time(t1) / K], dev, world)[0]

    # the product alone: one grouped tcgen05 launch over the three matrices
    # (x̃ ready), as in the step; and each shape on its own for context
    reps = max(5, min(50, K // 4))
    fwd_arr = bl.make_forward_problems([dict(x_q=pr["x_q"], beta=pr["beta"], W_packed=pr["W_packed"],
                                             alpha=pr["alpha"], N=pr["N"], y=pr["y"]) for pr in probs])
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            bl.check(L.bitlinear_forward_grouped(fwd_arr, len(specs), sh), "forward_grouped")
        g0.record()
        for _ in range(reps):
            bl.check(L.bitlinear_forward_grouped(fwd_arr, len(specs), sh), "forward_grouped")
        g1.record()
    stream.synchronize()
    grouped_ms = g0.elapsed_time(g1) / reps
    gemm_ms = [0.0] * len(specs)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in specs]
           for _ in range(reps)]
    with torch.cuda.stream(stream):
        for r in range(reps):
            for i, (s, pr) in enumerate(zip(specs, probs)):
                evs[r][i][0].record()
                bl.check(L.bitlinear_forward(bl._ptr(pr["x_q"]), bl._ptr(pr["beta"]), s.M, s.K, bl._ptr(pr["W_packed"]),
                                             bl._ptr(pr["alpha"]), s.N, None, bl._ptr(pr["y"]), None, sh), "forward")
                evs[r][i][1].record()
    stream.synchronize()
    for r in range(reps):
        for i in range(len(specs)):
            gemm_ms[i] += evs[r][i][0].elapsed_time(evs[r][i][1]) / reps
    # the grouped activation quantisation alone
    aq = (bl.ActProblem * len(specs))()
    for i, (s, pr) in enumerate(zip(specs, probs)):
        aq[i] = bl.ActProblem(bl._ptr(pr["x"]), bl._ptr(pr["x_q"]), bl._ptr(pr["beta"]), s.M, s.K)
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            bl.check(L.bitlinear_quantize_act_grouped(aq, len(specs), bl.BL_BF16, sh), "act")
        q0.record()
        for _ in range(reps):
            bl.check(L.bitlinear_quantize_act_grouped(aq, len(specs), bl.BL_BF16, sh), "act")
        q1.record()
    stream.synchronize()
    clocks = sampler.stop()
    aq_ms = q0.elapsed_time(q1) / reps
    aq_bytes = sum(s.M * s.K * 3 + 4 * s.M for s in specs)

    # the one-off weight quantisation (absmean + ternarise + pack) of the
    # prefill matrices, fp32 W: algorithmic bytes = 2 reads of W + packed write
    wq_bytes, wq_ms = 0, 0.0
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        ws = torch.empty(L.bitlinear_quantize_weights_workspace_bytes(s.N, s.K), dtype=torch.uint8, device=dev)
        pk = torch.empty((s.N, int(L.bitlinear_packed_row_bytes(s.K))), dtype=torch.uint8, device=dev)
        al = torch.empty(1, dtype=torch.float32, device=dev)
        def wq():
            bl.check(L.bitlinear_quantize_weights(bl._ptr(W), bl.BL_F32, s.N, s.K, bl._ptr(pk), bl._ptr(al),
                                                  bl._ptr(ws), ws.numel(), sh), "quantize_weights")
        with torch.cuda.stream(stream):
            wq()
            w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            w0.record()
            for _ in range(5):
                wq()
            w1.record()
        w1.synchronize()
        wq_ms += w0.elapsed_time(w1) / 5
        wq_bytes += 2 * s.N * s.K * 4 + pk.numel()
        del W, ws, pk

    # context: cuBLAS int8 GEMM (torch._int_mm) on int8 operands of the same shapes
    cublas = {}
    try:
        for s in specs:
            a8 = torch.randint(-127, 128, (s.M, s.K), dtype=torch.int8, device=dev)
            b8 = torch.randint(-1, 2, (s.N, s.K), dtype=torch.int8, device=dev).t()
            for _ in range(3):
                torch._int_mm(a8, b8)
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record()
            for _ in range(10):
                torch._int_mm(a8, b8)
            c1.record()
            c1.synchronize()
            cublas[f"{s.M}x{s.K}x{s.N}"] = round(2 * s.M * s.N * s.K / (c0.elapsed_time(c1) / 10 * 1e-3) / 1e12, 1)
            del a8, b8
    except RuntimeError as e:  # context only
        cublas = {"unavailable": str(e).splitlines()[0]}

    peaks, peak_src = load_peaks()
    peak = 2.0 * float(peaks["bf16_tflops"])
    achieved = sum(ops) / (grouped_ms * 1e-3) / 1e12
    value = world * sum(ops) / (step_ms * 1e-3) / 1e12
    return {
        "metric": "prefill int8 TOPS",
        "value": round(value, 1),
        "unit": "TOPS",
        "ms_per_step": round(step_ms, 5),
        "steps": K,
        "workload": "prefill M=2048 tokens: (K,N) = (4096,4096), (4096,11008), (11008,4096); bf16 x ~ N(0,1) + 0.1% "
                    "x20 outliers; per step grouped act quant + one tcgen05 GEMM (+dequant) per matrix",
        "ops_per_step": sum(ops),
        "l2": "per step the three problems hold x 79 MB, x_q 39 MB, packed W 27 MB, y 157 MB (>2x the L2)",
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_tc_kernel<256> (tcgen05.mma kind::i8, persistent, one CTA per SM), one grouped launch "
                      "over the three matrices",
            "achieved": round(achieved, 1),
            "peak": round(peak, 1),
            "peak_source": (f"{peak_src} bf16_tflops {peaks['bf16_tflops']} (cuBLAS bf16 burst) x 2, the nominal "
                            "int8/bf16 dense ratio (4.5/2.25 PFLOP/s)"),
            "unit": "TOPS",
            "frac": round(achieved / peak, 4),
            "traffic": recorded_traffic("gemm_tc:prefill_grouped", GEMM_SOURCES),
            "avg_launch_us": round(grouped_ms * 1e3, 2),
            "single_launch_us": {f"{s.M}x{s.K}x{s.N}": round(t * 1e3, 2) for s, t in zip(specs, gemm_ms)},
            "tops_by_shape": {f"{s.M}x{s.K}x{s.N}": round(o / (t * 1e-3) / 1e12, 1)
                              for s, o, t in zip(specs, ops, gemm_ms)},
        },
        "act_quant": {"us_per_step": round(aq_ms * 1e3, 2), "GB/s": round(aq_bytes / (aq_ms * 1e-3) / 1e9, 1),
                      "bytes_per_step": aq_bytes},
        "weight_quant": {"us_for_3_matrices": round(wq_ms * 1e3, 1), "GB/s": round(wq_bytes / (wq_ms * 1e-3) / 1e9, 1),
                         "bytes": wq_bytes, "what": "absmean (exact sum) + ternarise + 2-bit pack of the three fp32 "
                                                   "prefill matrices, once per matrix (not on the step path)"},
        "cublas_int8_tops_context": cublas,
        "gpu_launches": launches_per_step * K,  # act quant (one launch per CTA size) + one grouped GEMM per step
        "clocks": clocks,
    }


# ----------------------------------------------------------------------------- 100B batched-decode leg
def run_batched_100b(args, world, local_rank):
    """The 100B-shaped batched decode sweep: (K, N) = (8192, 28672) and
    (28672, 8192), M in {1, 2, 4, 8, 16, 32, 64}.  One step is one
    bitlinear_linear_grouped call on one matrix (act quant + product, flagged
    BL_LINEAR_WEIGHTS_STATIC); K steps per M in one CUDA graph over weight
    replicas that together exceed 4x the L2.  GB/s = algorithmic bytes per
    step (as for the decode leg) / time per step."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth, workloads

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    peak = float(load_peaks()[0]["hbm_gbs"])
    L = bl.lib()
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream
    Ms = (1, 2, 4, 8, 16, 32, 64)
    K_steps = max(12, args.steps)
    out, sampler, graphs = {}, None, []
    for (K, N) in ((8192, 28672), (28672, 8192)):
        spec0 = workloads.batched_decode_100b(K, N, 1)
        W = torch.from_numpy(synth.weights(spec0.seed, N, K, spec0.w_std)).to(dev)
        p0, alpha = bl.bitlinear_quantize_weights(W)
        del W
        wbytes = p0.numel()
        replicas = max(2, math.ceil(4 * props.L2_cache_size / wbytes) + 1)
        packed = [p0] + [p0.clone() for _ in range(replicas - 1)]
        per_m = {}
        for M in Ms:
            spec = workloads.batched_decode_100b(K, N, M)
            xb = synth.f32_to_bf16_bits(synth.activations(spec.x_seed, M, K))
            x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
            xq = torch.empty((M, K), dtype=torch.int8, device=dev)
            beta = torch.empty(M, dtype=torch.float32, device=dev)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            arrs = [bl.make_linear_problems([dict(x=x, x_q=xq, beta=beta, W_packed=packed[r], alpha=alpha, N=N, y=y)])
                    for r in range(replicas)]

            def step(i):
                bl.check(L.bitlinear_linear_grouped(arrs[i % replicas], 1, bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                                    sh), "linear")

            with torch.cuda.stream(stream):
                for i in range(3):
                    step(i)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(K_steps):
                    step(i)
            graphs.append(g)
            if sampler is None:
                sampler = settle(stream, g.replay, props, local_rank)
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
            if world > 1:
                import torch.distributed as dist
                dist.barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                t0.record()
                g.replay()
                t1.record()
            t1.synchronize()
            ms = max_over_ranks([t0.elapsed_time(t1) / K_steps], dev, world)[0]
            bps = bytes_per_step([spec])
            gbs = bps / (ms * 1e-3) / 1e9
            per_m[f"M{M}"] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1),
                              "frac": round(gbs / peak, 4), "pct_of_8TBps": round(100 * gbs / 8000.0, 2),
                              "kernel": ("gemv_stream_kernel (CUDA cores)" if M <= 2 else
                                         "gemm_tm_kernel (tcgen05 i8, codes expanded into tensor memory)")}
        out[f"K{K}_N{N}"] = {"weight_bytes": wbytes, "replicas": replicas, **per_m}
        del packed, p0
    with torch.cuda.stream(stream):
        graphs[-1].replay()
    stream.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    del graphs
    worst = min((v["frac"], k, m) for k, d in out.items() for m, v in d.items() if isinstance(v, dict))
    return {
        "metric": "ternary GEMV/GEMM HBM GB/s, 100B-shaped batched decode",
        "workload": "100B-shaped batched decode: (K,N) = (8192,28672) and (28672,8192), M in {1,2,4,8,16,32,64}; "
                    "W ~ N(0,0.015) ternarised once, x bf16 ~ N(0,1); per step one bitlinear_linear_grouped call "
                    "(act quant + product + dequant), K steps in one CUDA graph",
        "l2": "weight replicas rotate across steps, together more than 4x the L2",
        "steps": K_steps,
        "peak": peak,
        "unit": "GB/s",
        **out,
        "roofline": {"bound": "hbm", "unit": "GB/s", "peak": peak,
                     "achieved_M1": {k: d["M1"]["GB/s"] for k, d in out.items()},
                     "frac_M1": {k: d["M1"]["frac"] for k, d in out.items()},
                     "lowest_frac": {"frac": worst[0], "shape": worst[1], "M": worst[2]}},
        "clocks": clocks,
    }


# ----------------------------------------------------------------------------- shared timing
def time_steps(step, n_rep: int, K: int, stream, props, local_rank, world, dev):
    """Captures K calls of step(i) (i = 0..K-1, rotating over n_rep weight
    replicas inside step) in one CUDA graph, settles the clocks for ≈1 s of
    replays under the sampler, then times one replay with CUDA events on the
    replay stream.  Returns (ms per step, max over ranks; clocks)."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(K):
            step(i)
    sampler = settle(stream, g.replay, props, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        g.replay()
        t1.record()
    t1.synchronize()
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    clocks = sampler.stop()
    ms = max_over_ranks([t0.elapsed_time(t1) / K], dev, world)[0]
    del g
    return ms, clocks


def decode_inputs(specs, dev):
    """bf16 inputs (with outliers) and output buffers of the 7B decode set."""
    import torch
    from bitlinear_w1_a8_03_b200 import synth
    out = []
    for s in specs:
        xb = synth.f32_to_bf16_bits(synth.activations(s.x_seed, s.M, s.K, outliers=s.outliers))
        out.append(dict(x=torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev).view(s.M, s.K),
                        x_q=torch.empty((s.M, s.K), dtype=torch.int8, device=dev),
                        beta=torch.empty(s.M, dtype=torch.float32, device=dev),
                        y=torch.empty((s.M, s.N), dtype=torch.float32, device=dev), N=s.N))
    return out


# ----------------------------------------------------------------------------- rotation leg
def run_hadamard(args, world, local_rank):
    """The 7B decode set with the Hadamard rotation before the absmax
    quantisation ("1.58-bit 大模型极限量化实战" §6.2): weights quantised once from
    W·H/b (not timed); one step = one bitlinear_linear_grouped call flagged
    BL_LINEAR_HADAMARD | BL_LINEAR_WEIGHTS_STATIC: one GEMV launch whose CTAs
    rotate and quantise their input rows in the prologue; steps chained by PDL)."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    specs = workload_specs()
    packed0, alphas = [], []
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        p, a = bl.bitlinear_quantize_weights_rotated(W, bl.hadamard_block(s.K))
        packed0.append(p)
        alphas.append(a)
        del W
    torch.cuda.synchronize()
    set_bytes = sum(p.numel() for p in packed0)
    replicas = max(2, math.ceil(4 * props.L2_cache_size / set_bytes) + 1)
    packed = [packed0] + [[p.clone() for p in packed0] for _ in range(replicas - 1)]
    ins = decode_inputs(specs, dev)
    arrs = [bl.make_linear_problems([dict(io, W_packed=packed[r][i], alpha=alphas[i]) for i, io in enumerate(ins)])
            for r in range(replicas)]
    L = bl.lib()
    stream = torch.cuda.Stream(device=dev)
    flags = bl.BL_LINEAR_HADAMARD | bl.BL_LINEAR_WEIGHTS_STATIC

    def step(i):
        bl.check(L.bitlinear_linear_grouped(arrs[i % replicas], len(specs), bl.BL_BF16, flags, stream.cuda_stream),
                 "linear")

    K = max(12, args.steps)
    ms, clocks = time_steps(step, replicas, K, stream, props, local_rank, world, dev)
    bps = bytes_per_step(specs)
    peak = float(load_peaks()[0]["hbm_gbs"])
    gbs = bps / (ms * 1e-3) / 1e9
    return {"metric": "decode GB/s with the Hadamard rotation before the act quant",
            "workload": "7B decode layer set, M=1, bf16 x with 0.1% x20 outliers; weights from W*H/b; block = largest "
                        "power of two dividing K (4096 for K=4096, 256 for K=11008)",
            "us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
            "bytes_per_step": bps, "steps": K, "replicas": replicas,
            "launches_per_step": 1, "clocks": clocks}


# ----------------------------------------------------------------------------- scale-granularity leg
def run_scales(args, world, local_rank):
    """The 7B decode set with one α per row and one α per 128-block of a row
    (bitlinear_linear_scaled: grouped act quant, then the scaled GEMV).  The α
    table (N·ceil(K/group)·4 bytes) counts as weight traffic."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    specs = workload_specs()
    peak = float(load_peaks()[0]["hbm_gbs"])
    L = bl.lib()
    stream = torch.cuda.Stream(device=dev)
    out = {}
    for name, group in (("per_row", 1 << 30), ("per_block128", 128)):
        packed0, alphas = [], []
        for s in specs:
            W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
            p, a = bl.bitlinear_quantize_weights_scaled(W, group)
            packed0.append(p)
            alphas.append(a)
            del W
        torch.cuda.synchronize()
        set_bytes = sum(p.numel() + 4 * a.numel() for p, a in zip(packed0, alphas))
        replicas = max(2, math.ceil(4 * props.L2_cache_size / set_bytes) + 1)
        reps = [(packed0, alphas)] + [([p.clone() for p in packed0], [a.clone() for a in alphas])
                                      for _ in range(replicas - 1)]
        ins = decode_inputs(specs, dev)
        arrs = [bl.make_scaled_problems([dict(io, W_packed=reps[r][0][i], alpha=reps[r][1][i], group=group)
                                         for i, io in enumerate(ins)]) for r in range(replicas)]

        def step(i):
            bl.check(L.bitlinear_linear_scaled(arrs[i % replicas], len(specs), bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                               stream.cuda_stream), "linear_scaled")

        K = max(12, args.steps)
        ms, clocks = time_steps(step, replicas, K, stream, props, local_rank, world, dev)
        bps = bytes_per_step(specs) + sum(4 * a.numel() for a in alphas)
        gbs = bps / (ms * 1e-3) / 1e9
        out[name] = {"us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
                     "bytes_per_step": bps, "alpha_bytes": sum(4 * a.numel() for a in alphas), "steps": K,
                     "replicas": replicas, "clocks": clocks}
        del reps, arrs
    return {"metric": "decode GB/s with one alpha per row / per 128-block",
            "workload": "7B decode layer set, M=1, bf16 x with outliers; bitlinear_linear_scaled: one alpha per row "
                        "runs as one launch (the streaming GEMV quantises x in its prologue, the epilogue applies "
                        "the row's alpha); per 128-block as act quant + scaled GEMV (2 launches per step)", **out}


# ----------------------------------------------------------------------------- 4-bit activation leg
def run_a4(args, world, local_rank):
    """The 7B decode set with 4-bit activations: one step = one
    bitlinear_linear_a4 call (grouped 4-bit act quant, then the CUDA-core
    product on packed 4-bit x̃), weights flagged static."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    specs = workload_specs()
    packed0, alphas = [], []
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        p, a = bl.bitlinear_quantize_weights(W)
        packed0.append(p)
        alphas.append(a)
        del W
    torch.cuda.synchronize()
    set_bytes = sum(p.numel() for p in packed0)
    replicas = max(2, math.ceil(4 * props.L2_cache_size / set_bytes) + 1)
    packed = [packed0] + [[p.clone() for p in packed0] for _ in range(replicas - 1)]
    ins = decode_inputs(specs, dev)
    for io, s in zip(ins, specs):
        io["x_q"] = torch.empty((s.M, (s.K + 1) // 2), dtype=torch.uint8, device=dev)
    arrs = [bl.make_linear_a4_problems([dict(io, W_packed=packed[r][i], alpha=alphas[i]) for i, io in enumerate(ins)])
            for r in range(replicas)]
    L = bl.lib()
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        bl.check(L.bitlinear_linear_a4(arrs[i % replicas], len(specs), bl.BL_BF16, bl.BL_LINEAR_WEIGHTS_STATIC,
                                       stream.cuda_stream), "linear_a4")

    K = max(12, args.steps)
    ms, clocks = time_steps(step, replicas, K, stream, props, local_rank, world, dev)
    bps = sum(s.N * 16 * ((s.K + 63) // 64) + s.M * s.K * 2 + 2 * s.M * ((s.K + 1) // 2) + 8 * s.M + 4 * s.M * s.N
              for s in specs)
    peak = float(load_peaks()[0]["hbm_gbs"])
    gbs = bps / (ms * 1e-3) / 1e9
    return {"metric": "decode GB/s with 4-bit activations",
            "workload": "7B decode layer set, M=1, bf16 x with outliers; bitlinear_linear_a4 (one launch per step: "
                        "the streaming GEMV quantises x to 4 bits in its prologue)",
            "us_per_step": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
            "bytes_per_step": bps, "steps": K, "replicas": replicas, "clocks": clocks}


# ----------------------------------------------------------------------------- training leg
FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs × FP32 FMA lanes/clk × 2 flops × max SM clock


def run_train(args, world, local_rank):
    """One training step with the straight-through estimator on the three
    prefill shapes at M = 2048 tokens: bitlinear_train_forward (quantise the
    float32 latent weights afresh, quantise x, tensor-core product) then
    bitlinear_ste_backward (grad_x and grad_W, float32 CUDA-core GEMMs)."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    specs = prefill_specs()
    L = bl.lib()
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream
    items = []
    for s in specs:
        W = torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev)
        xb = synth.f32_to_bf16_bits(synth.activations(s.x_seed, s.M, s.K, outliers=True))
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        g = torch.randn((s.M, s.N), generator=torch.Generator(device=dev).manual_seed(s.seed), device=dev) * 1e-3
        ws = torch.empty(L.bitlinear_quantize_weights_workspace_bytes(s.N, s.K), dtype=torch.uint8, device=dev)
        it = dict(W=W, x=x, g=g, ws=ws, s=s,
                  Wp=torch.empty((s.N, int(L.bitlinear_packed_row_bytes(s.K))), dtype=torch.uint8, device=dev),
                  a=torch.empty(1, dtype=torch.float32, device=dev),
                  xq=torch.empty((s.M, s.K), dtype=torch.int8, device=dev),
                  b=torch.empty(s.M, dtype=torch.float32, device=dev),
                  y=torch.empty((s.M, s.N), dtype=torch.float32, device=dev),
                  gx=torch.empty((s.M, s.K), dtype=torch.float32, device=dev),
                  gw=torch.empty((s.N, s.K), dtype=torch.float32, device=dev))
        items.append(it)
    P = bl._ptr

    def fwd():
        for it in items:
            s = it["s"]
            bl.check(L.bitlinear_train_forward(P(it["W"]), bl.BL_F32, s.N, s.K, P(it["x"]), bl.BL_BF16, s.M, P(it["Wp"]),
                                               P(it["a"]), P(it["xq"]), P(it["b"]), P(it["y"]), P(it["ws"]),
                                               it["ws"].numel(), sh), "train_forward")

    def bwd():
        for it in items:
            s = it["s"]
            bl.check(L.bitlinear_ste_backward(P(it["g"]), s.M, s.N, s.K, P(it["Wp"]), P(it["a"]), P(it["xq"]), P(it["b"]),
                                              P(it["W"]), bl.BL_F32, P(it["gx"]), P(it["gw"]), sh), "ste_backward")

    K = max(3, args.steps // 4)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        for _ in range(2):
            fwd()
            bwd()
    stream.synchronize()
    sampler = ClockSampler(gpu_id(props, local_rank))
    fwd_ms = bwd_ms = 0.0
    with torch.cuda.stream(stream):
        for _ in range(K):
            ev[0].record()
            fwd()
            ev[1].record()
            bwd()
            ev[2].record()
            ev[2].synchronize()
            fwd_ms += ev[0].elapsed_time(ev[1]) / K
            bwd_ms += ev[1].elapsed_time(ev[2]) / K
    clocks = sampler.stop()
    fwd_ms, bwd_ms = max_over_ranks([fwd_ms, bwd_ms], dev, world)
    bwd_flops = sum(4 * s.M * s.N * s.K for s in specs)
    fwd_ops = sum(2 * s.M * s.N * s.K for s in specs)
    achieved = bwd_flops / (bwd_ms * 1e-3) / 1e12
    return {"metric": "training step (straight-through estimator) on the prefill shapes",
            "workload": "M=2048 tokens; (K,N) = (4096,4096), (4096,11008), (11008,4096); float32 latent W, bf16 x, "
                        "float32 upstream gradient",
            "ms_per_step": round(fwd_ms + bwd_ms, 3), "forward_ms": round(fwd_ms, 3), "backward_ms": round(bwd_ms, 3),
            "forward_TOPS": round(fwd_ops / (fwd_ms * 1e-3) / 1e12, 1),
            "roofline": {"bound": "alu", "kernel": "ste_grad_x_kernel + ste_grad_w_kernel (float32 FMA on CUDA cores)",
                         "achieved": round(achieved, 2), "peak": round(FFMA_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
                         "frac": round(achieved / FFMA_PEAK_TFLOPS, 4),
                         "peak_source": "148 SMs x 128 FP32 FMA lanes/clk x 2 flops x 1.965 GHz"},
            "steps": K, "clocks": clocks}


# ----------------------------------------------------------------------------- tiny leg
def run_tiny(args, world, local_rank):
    """Config 1: M = 1, K = N = 256, float32 x and W (seed 0).  A latency line:
    each bitlinear_linear call timed alone with CUDA events, an L2 flush (a
    write larger than the L2) between calls outside the timed events."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth, workloads

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    s = workloads.tiny()
    packed, alpha = bl.bitlinear_quantize_weights(torch.from_numpy(synth.weights(s.seed, s.N, s.K, s.w_std)).to(dev))
    x = torch.from_numpy(synth.activations(s.x_seed, s.M, s.K)).to(dev)
    xq = torch.empty((s.M, s.K), dtype=torch.int8, device=dev)
    beta = torch.empty(s.M, dtype=torch.float32, device=dev)
    y = torch.empty((s.M, s.N), dtype=torch.float32, device=dev)
    flush = torch.empty(2 * props.L2_cache_size // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    reps = max(20, args.steps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            bl.bitlinear_linear(x, packed, alpha, s.N, x_q=xq, beta=beta, y=y, stream=stream)
        for e0, e1 in evs:
            flush.fill_(1.0)
            e0.record()
            bl.bitlinear_linear(x, packed, alpha, s.N, x_q=xq, beta=beta, y=y, stream=stream)
            e1.record()
    stream.synchronize()
    us = sorted(e0.elapsed_time(e1) * 1e3 for e0, e1 in evs)
    med = statistics.median(us)
    bytes_call = s.N * 16 * ((s.K + 63) // 64) + s.M * s.K * 4 + s.M * s.K + 4 * s.M + s.M * s.K + 4 * s.M + 4 * s.M * s.N
    us = max_over_ranks([med], dev, world)[0]
    return {"metric": "latency of one bitlinear_linear call (act quant + GEMV + dequant), L2 flushed between calls",
            "workload": "tiny: M=1, K=N=256, fp32 x ~ N(0,1), W ~ N(0,0.02), seed 0",
            "us_per_call_median": round(us, 3), "GB/s": round(bytes_call / (us * 1e-6) / 1e9, 2),
            "bytes_per_call": bytes_call, "calls": reps}


# ----------------------------------------------------------------------------- stack leg
def run_stack(args, world, local_rank):
    """The 32-layer 7B-shaped linear stack per decode step (M = 1 and 16)."""
    import torch
    import bitlinear_w1_a8_03_b200 as bl
    from bitlinear_w1_a8_03_b200 import synth
    from bitlinear_w1_a8_03_b200.stack import MATRICES, LinearStack, shapes

    dev = torch.device("cuda", local_rank)
    props = torch.cuda.get_device_properties(dev)
    hidden, ffn, L = 4096, 11008, 32
    sh = shapes(hidden, ffn)
    g = torch.Generator(device=dev)
    layers = []
    for l in range(L):
        d = {}
        for i, n in enumerate(MATRICES):
            g.manual_seed(5000 + 7 * l + i)
            W = torch.randn(sh[n], generator=g, device=dev) * 0.02
            d[n] = bl.bitlinear_quantize_weights(W)
            del W
        layers.append(d)
    torch.cuda.synchronize()
    out = {}
    stream = torch.cuda.Stream(device=dev)
    for M in (1, 16):
        st = LinearStack(layers, hidden, ffn, M, dev)
        st.h0.copy_(torch.from_numpy(synth.activations(5999, M, hidden, outliers=True)).to(dev))
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                st.run(stream)
        stream.synchronize()
        stack_launches = kernels_per_call(lambda: st.run(stream), stream)
        K = max(10, args.steps // 4)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for _ in range(K):
                st.run(stream)
        with torch.cuda.stream(stream):
            gr.replay()
        stream.synchronize()
        sampler = settle(stream, gr.replay, props, local_rank)
        import torch.distributed as dist
        if world > 1:
            dist.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record()
            gr.replay()
            t1.record()
        t1.synchronize()
        with torch.cuda.stream(stream):
            gr.replay()
        stream.synchronize()
        clocks = sampler.stop()
        ms = max_over_ranks([t0.elapsed_time(t1) / K], dev, world)[0]
        # per token and layer: quant(y_o + y_down) 8H in, H out; x_h read once, y_q,k,v 12H and y_gate,up
        # 8F out; quant(y_v, y_up) 4H + 4F in, H + F out; x_v + x_up read, y_o + y_down 8H out
        act_bytes = L * M * (36 * hidden + 14 * ffn)
        bytes_step = st.weight_bytes + act_bytes
        err = bl.bitlinear_device_error()
        out[f"M{M}"] = {
            "tokens_per_s": round(world * M / (ms * 1e-3), 1),
            "ms_per_step": round(ms, 4),
            "effective_GBps": round(bytes_step / (ms * 1e-3) / 1e9, 1),
            "frac_of_hbm": round(bytes_step / (ms * 1e-3) / 1e9 / float(load_peaks()[0]["hbm_gbs"]), 4),
            "bytes_per_step": bytes_step,
            "steps": K,
            "gpu_launches_per_step": stack_launches,
            "device_error": err,
            "clocks": clocks,
        }
        del gr, st
    return {
        "metric": "decode tokens/s through the 32-layer linear stack",
        "workload": "7B-shaped stack: 32 layers x {q,k,v,o 4096->4096; gate,up 4096->11008; down 11008->4096}, "
                    "1.62 GB packed weights (W ~ N(0,0.02) from the device generator, seed 5000+7*layer+matrix); "
                    "per layer q,k,v,gate,up read quant(h), o reads quant(y_v), down reads quant(y_up), "
                    "h' = y_o + y_down summed inside the next quantisation; one CUDA graph of K steps",
        "l2": "weights 1.62 GB (13x the L2) streamed once per step",
        **out,
    }


# ----------------------------------------------------------------------------- oracle timing
def oracle_full():
    """Oracle inputs for the same workload: α and codes from the oracle's own
    weight quantisation of the full matrices (not timed)."""
    import oracle
    from bitlinear_w1_a8_03_b200 import synth
    items = []
    for s in workload_specs():
        W = synth.weights(s.seed, s.N, s.K, s.w_std)
        alpha = oracle.absmean(W)
        codes = oracle.ternarize(W, alpha)
        del W
        x = synth.f32_to_bf16_bits(synth.activations(s.x_seed, s.M, s.K, outliers=s.outliers))
        items.append((s, x, codes, alpha))
    return items


def oracle_sample(full, rows_frac: float):
    """The first round(N·rows_frac) output rows of every matrix (full K)."""
    out = []
    for s, x, codes, alpha in full:
        n = max(1, int(round(s.N * rows_frac)))
        out.append((s, x, np.ascontiguousarray(codes[:n]), alpha, n))
    return out


def oracle_bytes(items) -> int:
    total = 0
    for s, x, codes, alpha, n in items:
        rb = 16 * ((s.K + 63) // 64)
        total += n * rb + s.M * s.K * 3 + 4 * s.M + s.M * s.K + 4 * s.M + 4 * s.M * n
    return total


def time_oracle(items, threads: int, steps: int, budget_s: float):
    import oracle
    done, t_total = 0, 0.0
    while done < steps:
        t = time.perf_counter()
        for s, x, codes, alpha, n in items:
            oracle.forward(x, codes, alpha, threads=threads)
        t_total += time.perf_counter() - t
        done += 1
        if t_total >= budget_s:
            break
    return done, t_total


def sized_sample(full, threads: int, step_seconds: float):
    """Row fraction whose oracle step takes about ``step_seconds`` here."""
    probe = oracle_sample(full, 0.02)
    _, tp = time_oracle(probe, threads, 1, 0.0)
    frac = min(1.0, max(1e-4, 0.02 * step_seconds / max(tp, 1e-4)))
    return frac, oracle_sample(full, frac)


def cpu_baseline(args):
    threads = os.cpu_count() or 1
    full = oracle_full()
    frac, items = sized_sample(full, threads, 1.0)
    steps, secs = time_oracle(items, threads, 1000, 12.0)
    gbs = oracle_bytes(items) * steps / secs / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {frac:.4f} of the output rows of each of the 7 matrices (full K), {steps} whole steps "
                      f"in {secs:.1f} s; act quant + add/sub/skip product + dequant, OpenMP over output elements"}


def run_reference(args):
    threads = os.cpu_count() or 1
    total_steps = args.steps + args.warmup
    budget = 150.0  # seconds for the whole timed + warm-up run
    full = oracle_full()
    frac, items = sized_sample(full, threads, budget / max(total_steps, 1))
    for _ in range(args.warmup):
        time_oracle(items, threads, 1, 0.0)
    steps, secs = time_oracle(items, threads, args.steps, float("inf"))
    value = oracle_bytes(items) * steps / secs / 1e9
    sample = (f"first {frac:.5f} of the output rows of each of the 7 matrices (full K) per step; "
              "act quant + add/sub/skip product + dequant, OpenMP over output elements")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": 1,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 x ternary -> int64 (checked into int32), fp32 dequant",
        "data": "synthetic (same seeds as the native arm)",
        "config": decode_config(workload_specs()),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--legs", default="decode,tiny,batched_100b,prefill,stack,hadamard,scales,a4,train",
                    help="comma list: decode (the headline line); tiny, batched_100b, prefill, stack, hadamard, "
                         "scales, a4 and train are added under their own keys")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle on the host")
    ap.add_argument("--settle-seconds", type=float, default=1.0,
                    help="seconds of identical replays before each timed region (0: profiler runs only)")
    args = ap.parse_args()
    global SETTLE_SECONDS
    SETTLE_SECONDS = max(0.0, args.settle_seconds)
    legs = [x for x in args.legs.split(",") if x]
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    result = run_native(args, rank, world, local_rank) if "decode" in legs else {"metric": METRIC}
    if "prefill" in legs:
        pre = run_prefill(args, world, local_rank)
        result["prefill"] = pre
        if "decode" not in legs:
            result.update({"value": pre["value"], "unit": pre["unit"], "n_gpus": world, "steps": args.steps,
                           "warmup": args.warmup, "ms_per_step": pre["ms_per_step"], "higher_is_better": True,
                           "scaling": "weak", "vs_baseline": None})
    if "tiny" in legs:
        result["tiny"] = run_tiny(args, world, local_rank)
    if "batched_100b" in legs:
        result["batched_100b"] = run_batched_100b(args, world, local_rank)
    if "stack" in legs:
        result["stack"] = run_stack(args, world, local_rank)
    if "hadamard" in legs:
        result["hadamard"] = run_hadamard(args, world, local_rank)
    if "scales" in legs:
        result["scales"] = run_scales(args, world, local_rank)
    if "a4" in legs:
        result["a4"] = run_a4(args, world, local_rank)
    if "train" in legs:
        result["train"] = run_train(args, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(args)
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
