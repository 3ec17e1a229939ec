"""Benchmark of the W4A16 fused GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode70b|decode70b_sym|decode7b|prefill|decode7b_pc|prefill_pc]
                    [--no-extras] [--no-cpu-baseline] [--crossover]

Metric: W4A16 GEMM HBM GB/s at M=1 and TFLOPS at M=2048, as % of the B200
roofline.  The headline line (default workload) is the M=1 decode of the two
Llama-2-70B-shaped layers (K=8192,N=28672 and K=28672,N=8192; g=128, asym),
the largest single-GPU M=1 configuration: one step = both fused GEMMs,
through the library's dispatch, on synthetic seeded weights/activations of
that shape.  `value` is algorithmic bytes per step (packed weights + scales +
zeros + X read once + Y written once) times steps, over the device time of the
timed region, summed over ranks and divided by the max over ranks.  The same
JSON line carries, each with its own roofline object, the other M=1 decode
workloads (the 70B-shaped layers with symmetric codes, the 7B-shaped layers),
the M=2048 prefill TFLOPS (K=N=8192) against the tensor-core roofline, dense
bf16 cuBLAS and the unfused dequantize-then-GEMM at the same shapes, the
crossover sweep (K=N=8192, every M, g and mode, each kernel the dispatch can
choose), the end-to-end number through the public API with host buffers, and
the host oracle on the CPU.  Further extras: standalone quantize/dequantize
bandwidth, the per-channel (g = K) decode and prefill, the W8A16 (8-bit
code) quantize, dequantize, M=1 GEMV and M=2048 GEMM, and the cost of the fused
per-input-channel activation scale.

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs (one
graph holds a full rotation over the weight copies, so graph launches are
amortized; leftover steps replay one-step graphs), bracketed by a barrier and
torch.cuda.synchronize() on both sides, CUDA events on the launching stream.
Weight copies rotate so the bytes touched between reuses exceed twice the L2
size: every step streams its weights from HBM.  The timed region contains only
the workload's GEMM launches, so the average launch duration behind the
roofline figure is the region's time over its launches.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "W4A16 GEMM HBM GB/s at M=1 and TFLOPS at M=2048, as % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES_FALLBACK = 126 * 1024 * 1024


# ---------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def group_of(g: int, K: int) -> int:
    """g = 0 in a workload definition means per-channel granularity: one group
    spanning each row (g = K), one scale and zero per output feature."""
    return K if g == 0 else g


def input_bytes(M: int, N: int, K: int, g: int, sym: bool, bits: int = 4) -> int:
    """Packed codes (bits per weight) + scales (+ zeros if asymmetric) + X."""
    return N * K * bits // 8 + 2 * N * (K // g) * (1 if sym else 2) + 2 * M * K


def algorithmic_bytes(M: int, N: int, K: int, g: int, sym: bool, bits: int = 4) -> int:
    """Packed codes + scales (+ zeros if asymmetric) + X read once + Y written once."""
    return input_bytes(M, N, K, g, sym, bits) + 2 * M * N


# Sources each timed kernel is built from (its device code, the shared device
# helpers, and the host file that chooses its launch configuration).
KERNEL_SOURCES = {
    "gemv_decode_kernel": ("common.cuh", "gemv_decode.cuh", "w4a16.cu"),
    "gemm_tc_kernel": ("common.cuh", "gemm_tcgen05.cuh", "w4a16.cu"),
    "gemm_w8a8_kernel": ("common.cuh", "gemm_w8a8.cuh", "w4a16.cu"),
}


def kernel_source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_quantization_rtn_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu capture of the current kernel
    source (profiles/ncu_traffic.json, key "<kernel>:<workload>"), or None when
    the capture is missing or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
        entry = table[kernel_key]
        if entry.get("kernel_source_digest") != kernel_source_digest(kernel_key.split(":")[0]):
            return None
        return float(entry["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while it runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        self.t0 = time.time()
        return self

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.12)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        import datetime
        rows = []
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if self.t1 is not None and not (self.t0 - 0.06 <= ts <= self.t1 + 0.06):
                    continue                      # keep the samples taken in the timed region
                rows.append((float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------- dist
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce_scalar(world, value: float, op) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(world, value: float) -> float:
    """Timing is the slowest rank's: max of the per-rank device times."""
    import torch.distributed as dist
    return value if world == 1 else _reduce_scalar(world, value, dist.ReduceOp.MAX)


def sum_over_ranks(world, value: float) -> float:
    """Work is the whole job's: sum of the per-rank bytes or flops."""
    import torch.distributed as dist
    return value if world == 1 else _reduce_scalar(world, value, dist.ReduceOp.SUM)


def job_throughput(world, per_rank_work: float, per_rank_ms: float, scale: float) -> float:
    """Whole-job throughput: all ranks' work over the max of their times."""
    total = sum_over_ranks(world, per_rank_work)
    ms = max_over_ranks(world, per_rank_ms)
    return total / (ms / 1e3) / scale


# ---------------------------------------------------------------------------- workloads
class GemmCase:
    """One layer of a workload, resident on the device, with `copies` rotating
    copies of the quantized weights (and activations)."""

    def __init__(self, w4, layer, M, g, sym, copies, dev, bits=4):
        self.layer, self.M, self.g, self.sym, self.bits = layer, M, g, sym, bits
        self.N, self.K = layer.N, layer.K
        W = layer.weight().to(dev)
        P, S, Z = (w4.quantize8 if bits == 8 else w4.quantize)(W, g, sym)
        self.W_dense = W
        self.P = [P] + [P.clone() for _ in range(copies - 1)]
        self.S = [S] + [S.clone() for _ in range(copies - 1)]
        self.Z = [Z] + [Z.clone() for _ in range(copies - 1)]
        X = layer.activation(M).to(dev)
        self.X = [X] + [X.clone() for _ in range(copies - 1)]
        self.Y = [torch.empty(M, self.N, dtype=torch.bfloat16, device=dev) for _ in range(copies)]
        self.bytes = algorithmic_bytes(M, self.N, self.K, g, sym, bits)
        self.flops = 2 * M * self.N * self.K

    def call(self, w4, i):
        # The weights are fixed after set-up and no kernel in a step writes them, so
        # the decode kernel may stream them while the previous GEMM drains.
        j = i % len(self.P)
        gemm = w4.gemm8 if self.bits == 8 else w4.gemm
        gemm(self.X[j], self.P[j], self.S[j], self.Z[j], self.g, self.sym, out=self.Y[j],
             static_weights=True)


def launches_per_call(plan: dict) -> int:
    """Kernels one GEMM call launches (a host-side property of the plan): one for
    the decode path; one to three for the tensor-core path (unsplit head, K-split
    tail, the reduce of the tail's parts)."""
    return int(plan["kernels"])


def copies_for(bytes_per_step: int, l2: int) -> int:
    return max(2, -(-2 * l2 // max(bytes_per_step, 1)) + 1)


def capture_rotation_graph(w4, cases, copies):
    """One CUDA graph holding a full rotation: `copies` steps, step i running
    every case on weight copy i.  Replaying it back to back keeps consecutive
    steps on different copies, and amortizes the graph launch over the steps."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for i in range(copies):          # plans, tensor maps and kernel attributes before capture
            for c in cases:
                c.call(w4, i)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    rot = torch.cuda.CUDAGraph()
    with torch.cuda.graph(rot, stream=stream):
        for i in range(copies):
            for c in cases:
                c.call(w4, i)
    singles = []
    for i in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in cases:
                c.call(w4, i)
        singles.append(g)
    torch.cuda.synchronize()
    return rot, singles


def replay_steps(rot, singles, copies, steps):
    """Exactly `steps` steps: whole rotations, then single steps for the rest."""
    for _ in range(steps // copies):
        rot.replay()
    for i in range(steps % copies):
        singles[i].replay()


def run_timed(world, rot, singles, copies, steps, warmup, sampler_index=None):
    replay_steps(rot, singles, copies, warmup)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(sampler_index) if sampler_index is not None else None
    if sampler:
        sampler.__enter__()
    start.record()
    replay_steps(rot, singles, copies, steps)
    end.record()
    end.synchronize()
    if sampler:
        sampler.mark_end()
        sampler.__exit__(None, None, None)
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    return ms, (sampler.summary() if sampler else None)


def per_layer_ms(w4, cases, copies, reps=50):
    """Diagnostic outside the timed region: each case alone, replayed from a
    rotation graph, so its own average duration (launch gaps included)."""
    out = []
    for c in cases:
        rot, singles = capture_rotation_graph(w4, [c], copies)
        replay_steps(rot, singles, copies, copies * 3)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        replay_steps(rot, singles, copies, copies * reps)
        b.record()
        b.synchronize()
        out.append(a.elapsed_time(b) / (copies * reps))
        del rot, singles
    return out


def time_callable(fn, iters, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / iters


def graph_of(fn, copies):
    """CUDA graphs of fn(i) for each rotation slot i (for comparison timings)."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for i in range(copies):
            fn(i)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    gs = []
    for i in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn(i)
        gs.append(g)
    torch.cuda.synchronize()
    return gs


def time_graphs(gs, iters):
    for i in range(3):
        gs[i % len(gs)].replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(iters):
        gs[i % len(gs)].replay()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / iters


# ---------------------------------------------------------------------------- oracle baseline
def cpu_baseline(layers, M, g, sym, unit_bytes: bool, budget_s: float = 6.0):
    """The host oracle as it stands (dequantize + binary64 matmul from the packed
    form) on the same layer shapes; repeats the whole workload until budget_s."""
    import oracle
    oracle.build()
    prepared = []
    for layer in layers:
        Wb = workloads.bits(layer.weight())
        Xb = workloads.bits(layer.activation(M))
        P, S, Z = oracle.quantize(Wb, group_of(g, layer.K), sym)
        prepared.append((layer, Xb, P, S, Z))
    reps, t0 = 0, time.perf_counter()
    while True:
        for layer, Xb, P, S, Z in prepared:
            oracle.gemm_w4a16(Xb, P, S, Z, group_of(g, layer.K), sym)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 50:
            break
    per_step = el / reps
    if unit_bytes:
        work = sum(algorithmic_bytes(M, l.N, l.K, group_of(g, l.K), sym) for l in layers)
        value, unit = work / per_step / 1e9, "GB/s"
    else:
        work = sum(2 * M * l.N * l.K for l in layers)
        value, unit = work / per_step / 1e12, "TFLOP/s"
    return {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} full step(s) of the workload ({len(layers)} layer GEMM(s), "
                      f"dequantize + binary64 matmul from the packed form) in {el:.2f} s",
            "s_per_step": per_step}


def cpu_baseline_sampled(layer, M, g, sym, rows: int):
    """Oracle on a bounded sample of output rows (for workloads far beyond a
    minute of CPU time); throughput scaled per output row."""
    import numpy as np
    import oracle
    oracle.build()
    Wb = workloads.bits(layer.weight())
    Xb = workloads.bits(layer.activation(M))
    g = group_of(g, layer.K)
    P, S, Z = oracle.quantize(Wb, g, sym)
    ns = np.arange(rows, dtype=np.int64)
    ms = np.zeros(rows, dtype=np.int64)
    mm, nn = np.meshgrid(np.arange(M), ns, indexing="ij")
    t0 = time.perf_counter()
    oracle.gemm_sampled(Xb, P, S, Z, g, sym, mm.ravel(), nn.ravel())
    el = time.perf_counter() - t0
    frac = rows / layer.N
    flops = 2 * M * layer.N * layer.K * frac
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{rows} of {layer.N} output columns x all {M} rows "
                      f"({frac * 100:.2f}% of the outputs) in {el:.2f} s",
            "s_per_step": el / frac}


# ---------------------------------------------------------------------------- main arms
WORKLOAD_DEFS = {
    # name: (workload, M, g, sym, metric half, code bits); g = 0: per-channel (g = K)
    "decode7b": (workloads.DECODE_7B, 1, 128, False, "hbm", 4),
    "decode70b": (workloads.DECODE_70B, 1, 128, False, "hbm", 4),
    "decode70b_sym": (workloads.DECODE_70B, 1, 128, True, "hbm", 4),
    "prefill": (workloads.PREFILL, 2048, 128, False, "tensor", 4),
    "decode7b_pc": (workloads.DECODE_7B, 1, 0, False, "hbm", 4),
    "prefill_pc": (workloads.PREFILL, 2048, 0, False, "tensor", 4),
    # mid-M: the tensor-core kernel at 32 activation rows on the prefill matrix
    # (2 CTAs per SM, all tiles split over K); HBM-bound at this M (≈128 flop/B)
    "mid32": (workloads.PREFILL, 32, 128, False, "hbm", 4),
    # W8A16 (8-bit codes): for profiling the 8-bit kernels; no end-to-end leg
    "w8_decode70b": (workloads.DECODE_70B, 1, 128, False, "hbm", 8),
    "w8_prefill": (workloads.PREFILL, 2048, 128, False, "tensor", 8),
}


def workload_name(wl, M, g, sym=False, bits=4) -> str:
    return (("w8a16_" if bits == 8 else "") + f"{wl.name}_M{M}" + ("_per_channel" if g == 0 else "")
            + ("_sym" if sym else ""))


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    import weight_only_quantization_rtn_b200 as w4
    from weight_only_quantization_rtn_b200 import build as w4build
    if rank == 0:
        w4build.build()
    barrier(world)
    w4.lib()
    peaks, peak_src = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 0) or L2_BYTES_FALLBACK

    wl, M, g, sym, half, bits = WORKLOAD_DEFS[args.workload]
    bytes_step = sum(algorithmic_bytes(M, l.N, l.K, group_of(g, l.K), sym, bits) for l in wl.layers)
    flops_step = sum(2 * M * l.N * l.K for l in wl.layers)
    in_bytes_step = sum(input_bytes(M, l.N, l.K, group_of(g, l.K), sym, bits) for l in wl.layers)
    copies = copies_for(in_bytes_step, l2)
    cases = [GemmCase(w4, l, M, group_of(g, l.K), sym, copies, dev, bits) for l in wl.layers]
    rot, singles = capture_rotation_graph(w4, cases, copies)
    ms, clocks = run_timed(world, rot, singles, copies, args.steps, args.warmup, sampler_index=local)
    ms_max = max_over_ranks(world, ms)
    total_bytes = sum_over_ranks(world, bytes_step * args.steps)
    total_flops = sum_over_ranks(world, flops_step * args.steps)
    sec = ms_max / 1e3
    if half == "hbm":
        value, unit = total_bytes / sec / 1e9, "GB/s"
    else:
        value, unit = total_flops / sec / 1e12, "TFLOP/s"
    kms = per_layer_ms(w4, cases, copies)

    plans = [(w4.plan8 if bits == 8 else w4.plan)(M, c.N, c.K, c.g, sym) for c in cases]
    kernel_name = "gemv_decode_kernel" if plans[0]["path"] == "decode" else "gemm_tc_kernel"
    # The timed region holds only this workload's GEMM launches, so the kernel's
    # average launch duration is the region's time over its launches.
    launches = len(cases) * args.steps
    k_sec = (ms / 1e3) / args.steps
    if half == "hbm":
        achieved = bytes_step / k_sec / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src}
    else:
        achieved = flops_step / k_sec / 1e12
        pk = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                "frac": achieved / pk, "peak_source": peak_src + " (burst)"}
    traffic = ncu_traffic(f"{kernel_name}:{args.workload}")
    roof["traffic"] = traffic
    roof["kernel"] = kernel_name
    roof["avg_launch_us"] = k_sec / len(cases) * 1e6
    roof["per_layer_us_alone"] = [round(x * 1e3, 3) for x in kms]
    roof["algorithmic_bytes_per_launch"] = [c.bytes for c in cases]

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": workload_name(wl, M, g, sym, bits), "M": M,
            "layers_KxN": [[l.K, l.N] for l in wl.layers], "g": g if g else "K (per-channel)",
            "mode": "sym" if sym else "asym", "description": wl.description,
            "l2": f"{copies} rotating copies of weights+activations "
                  f"({copies * in_bytes_step / 2**20:.0f} MiB, > 2x L2 of {l2 / 2**20:.0f} MiB)",
            "parallelism": f"replicas x{world} (independent problems, no collective)",
            "plan": plans, "algorithmic_bytes_per_step": bytes_step,
            "flops_per_step": flops_step,
        },
        "roofline": roof,
        "gpu_launches": sum(launches_per_call(p) for p in plans) * args.steps,
        "clocks": clocks,
    }

    # ------------------------------------------------ end to end through the public API
    # (4-bit workloads; the 8-bit ones exist to profile the 8-bit kernels)
    if bits == 4:
        pinned = [c.X[0].cpu().pin_memory() for c in cases]
        host_y = [torch.empty(c.M, c.N, dtype=torch.bfloat16, pin_memory=True) for c in cases]
        h2d = sum(x.numel() * 2 for x in pinned)
        d2h = sum(c.M * c.N * 2 for c in cases)
        e2e_steps = min(args.steps, 2000)

        def e2e_step(i):
            # host X in, host Y out for every layer; the step waits once, for its last copy
            for c, xh, yh in zip(cases, pinned, host_y):
                j = i % copies
                w4.gemm(xh, c.P[j], c.S[j], c.Z[j], c.g, c.sym, out=yh, sync=False, static_weights=True)
            torch.cuda.current_stream().synchronize()

        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(e2e_steps):
            e2e_step(i)
        b.record()
        b.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(world, a.elapsed_time(b))
        e2e_total = sum_over_ranks(world, (bytes_step if half == "hbm" else flops_step) * e2e_steps)
        e2e_val = e2e_total / (e2e_ms / 1e3) / (1e9 if half == "hbm" else 1e12)
        line["e2e"] = {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                       "ms_per_step": e2e_ms / e2e_steps}

    # ------------------------------------------------ comparisons and the other metric half
    if not args.no_extras and bits == 4:
        line["comparisons"] = comparisons(w4, cases, copies, l2, half)
        if half == "hbm":
            ro = read_only_stream_gbs(dev)
            roof["read_only_stream_gbs"] = ro
            roof["frac_of_read_only_stream"] = roof["achieved"] / ro
            roof["frac_of_nominal"] = roof["achieved"] / NOMINAL_HBM_GBS
        else:
            roof["frac_of_nominal"] = roof["achieved"] / NOMINAL_BF16_TFLOPS
        if args.workload != "prefill":
            others = [n for n in ("decode70b", "decode70b_sym", "decode7b") if n != args.workload]
            line["decode_workloads"] = workload_extras(w4, others, peaks, peak_src, l2, dev)
            line["prefill"] = prefill_extra(w4, peaks, peak_src, l2, dev)
            pr = line["prefill"]["roofline"]
            pr["frac_of_nominal"] = pr["achieved"] / NOMINAL_BF16_TFLOPS
            line["crossover"] = crossover_rows(w4, dev, l2)
            line["quantize_dequantize"] = elementwise_extras(w4, peaks, l2, dev)
            line["per_channel"] = workload_extras(w4, ["decode7b_pc", "prefill_pc"], peaks, peak_src,
                                                  l2, dev)
            line["w8a16"] = w8a16_extras(w4, peaks, l2, dev)
            line["act_scale"] = act_scale_extras(w4, l2, dev)
            line["w8a8"] = w8a8_extras(w4, peaks, l2, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and bits == 4:
        cb = cpu_baseline(wl.layers, M, g, sym, unit_bytes=(half == "hbm")) \
            if half == "hbm" else cpu_baseline_sampled(wl.layers[0], M, g, sym, rows=16)
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del rot, singles
        torch.cuda.synchronize()
        dist.destroy_process_group()


# Nominal B200 figures (for context beside the measured denominators).
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def read_only_stream_gbs(dev, nbytes: int = 2 << 30, iters: int = 10) -> float:
    """HBM read bandwidth of a plain streaming reduction (torch.sum over a buffer
    16x the L2), the read-only counterpart of the measured copy bandwidth."""
    buf = torch.ones(nbytes // 4, dtype=torch.float32, device=dev)
    out = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(3):
        torch.sum(buf, dim=0, out=out)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        torch.sum(buf, dim=0, out=out)
    b.record()
    b.synchronize()
    gbs = nbytes * iters / (a.elapsed_time(b) / 1e3) / 1e9
    del buf
    torch.cuda.empty_cache()
    return gbs


def elementwise_extras(w4, peaks, l2, dev, iters=20):
    """Quantize/pack and standalone dequantize of a 7B-shaped weight (K=4096,
    N=11008, g=128, asym): single HBM passes, reported against the measured copy
    bandwidth.  Bytes: quantize reads W (2 B/weight) and writes codes, scales and
    zeros; dequantize reads those and writes Ŵ (2 B/weight)."""
    layer = workloads.DECODE_7B.layers[0]
    N, K, g = layer.N, layer.K, 128
    W = layer.weight().to(dev)
    packed_bytes = N * K // 2 + 4 * N * (K // g)
    copies = max(2, -(-2 * l2 // (N * K * 2)) + 1)
    Ws = [W] + [W.clone() for _ in range(copies - 1)]
    outs = [w4.quantize(w, g, False) for w in Ws]
    gs = graph_of(lambda i: w4.quantize(Ws[i % copies], g, False), copies)
    qms = time_graphs(gs, iters)
    del gs
    Wh = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    gs = graph_of(lambda i: w4.dequantize(*outs[i % copies], g, False, out=Wh), copies)
    dms = time_graphs(gs, iters)
    del gs, Ws, outs, Wh, W
    torch.cuda.empty_cache()
    pk = peaks["hbm_gbs"]
    qb, db = N * K * 2 + packed_bytes, packed_bytes + N * K * 2
    return {"shape": f"N={N},K={K},g={g},asym",
            "quantize": {"us": qms * 1e3, "GB/s": qb / (qms / 1e3) / 1e9, "frac": qb / (qms / 1e3) / 1e9 / pk},
            "dequantize": {"us": dms * 1e3, "GB/s": db / (dms / 1e3) / 1e9, "frac": db / (dms / 1e3) / 1e9 / pk}}


def workload_extras(w4, names, peaks, peak_src, l2, dev, decode_iters=400, tensor_iters=30):
    """Other workloads of WORKLOAD_DEFS measured like the headline — rotation
    graphs over copies larger than L2, CUDA events on the replay stream — each
    with its own roofline object (achieved = the workload's algorithmic bytes or
    FLOPs per step over the time per step; traffic from the committed ncu table
    when it matches the kernel's current source).  Per-channel workloads count
    one scale (and zero) per row."""
    out = {}
    for name in names:
        wl, M, g, sym, half, bits = WORKLOAD_DEFS[name]
        in_bytes = sum(input_bytes(M, l.N, l.K, group_of(g, l.K), sym, bits) for l in wl.layers)
        copies = copies_for(in_bytes, l2)
        cases = [GemmCase(w4, l, M, group_of(g, l.K), sym, copies, dev, bits) for l in wl.layers]
        rot, singles = capture_rotation_graph(w4, cases, copies)
        n = decode_iters if half == "hbm" else tensor_iters
        replay_steps(rot, singles, copies, 3)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        replay_steps(rot, singles, copies, n)
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b) / n
        kms = per_layer_ms(w4, cases, copies, reps=20 if half == "hbm" else 5)
        plans = [(w4.plan8 if bits == 8 else w4.plan)(M, c.N, c.K, c.g, sym) for c in cases]
        kernel = "gemv_decode_kernel" if plans[0]["path"] == "decode" else "gemm_tc_kernel"
        if half == "hbm":
            work = sum(c.bytes for c in cases)
            ach, pk, unit = work / (ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
        else:
            work = sum(c.flops for c in cases)
            ach, pk, unit = work / (ms / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        out[name] = {"workload": workload_name(wl, M, g, sym, bits), "ms_per_step": ms, "value": ach,
                     "unit": unit,
                     "roofline": {"bound": "hbm" if half == "hbm" else "tensor", "achieved": ach,
                                  "peak": pk, "unit": unit, "frac": ach / pk,
                                  "peak_source": peak_src + ("" if half == "hbm" else " (burst)"),
                                  "traffic": ncu_traffic(f"{kernel}:{name}"), "kernel": kernel,
                                  "avg_launch_us": ms / len(cases) * 1e3,
                                  "per_layer_us_alone": [round(x * 1e3, 3) for x in kms],
                                  "algorithmic_bytes_per_launch": [c.bytes for c in cases]},
                     "plan": plans}
        del rot, singles, cases
        torch.cuda.empty_cache()
    return out


def w8a16_extras(w4, peaks, l2, dev, iters=200):
    """W8A16 (8-bit codes, one per byte) at g=128 asym: quantize/pack and
    dequantize of a 7B-shaped weight (N=11008, K=4096), the fused M=1 decode GEMM
    over both 7B-shaped and both 70B-shaped layers, and the tensor-core kernel at
    M=2048, K=N=8192, with
    inputs rotated past L2 and graph-replayed.
    Bytes: quantize reads W and writes codes + scales + zeros; dequantize the
    reverse; the GEMV reads codes + scales + zeros + X and writes Y."""
    g, sym = 128, False
    layers = workloads.DECODE_7B.layers
    L0 = layers[0]
    N, K = L0.N, L0.K
    pk = peaks["hbm_gbs"]
    W = L0.weight().to(dev)
    meta = 4 * N * (K // g)
    copies = max(2, -(-2 * l2 // (N * K * 2)) + 1)
    Ws = [W] + [W.clone() for _ in range(copies - 1)]
    outs = [w4.quantize8(w, g, sym) for w in Ws]
    gs = graph_of(lambda i: w4.quantize8(Ws[i % copies], g, sym), copies)
    qms = time_graphs(gs, 20)
    del gs
    Wh = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    gs = graph_of(lambda i: w4.dequantize8(*outs[i % copies], g, sym, out=Wh), copies)
    dms = time_graphs(gs, 20)
    del gs, Ws, outs, Wh, W
    qb = db = N * K * 2 + N * K + meta
    # fused decode GEMM, M=1, both layers per step: the 7B- and the 70B-shaped pair
    def decode_step_ms(layers):
        per_step = sum(l.N * l.K + 4 * l.N * (l.K // g) + 2 * l.K for l in layers)
        gcopies = copies_for(per_step, l2)
        sets = []
        for l in layers:
            C, S, Z = w4.quantize8(l.weight().to(dev), g, sym)
            X = l.activation(1).to(dev)
            Y = torch.empty(1, l.N, dtype=torch.bfloat16, device=dev)
            sets.append([(C, S, Z, X, Y)] + [(C.clone(), S.clone(), Z.clone(), X.clone(), Y)
                                             for _ in range(gcopies - 1)])

        def step(i):
            for cs in sets:
                C, S, Z, X, Y = cs[i % gcopies]
                w4.gemm8(X, C, S, Z, g, sym, out=Y)

        gs = graph_of(step, gcopies)
        ms = time_graphs(gs, iters)
        del gs, sets
        torch.cuda.empty_cache()
        nbytes = sum(algorithmic_bytes(1, l.N, l.K, g, sym) + l.N * l.K // 2 for l in layers)
        return ms, nbytes

    gms, gbytes = decode_step_ms(layers)
    gbs = gbytes / (gms / 1e3) / 1e9
    gms70, gbytes70 = decode_step_ms(workloads.DECODE_70B.layers)
    gbs70 = gbytes70 / (gms70 / 1e3) / 1e9
    # tensor-core kernel with 8-bit codes: prefill M=2048, K=N=8192
    P = workloads.PREFILL.layers[0]
    M = 2048
    pin = P.N * P.K + 4 * P.N * (P.K // g) + 2 * M * P.K
    pcopies = copies_for(pin, l2)
    C, S, Z = w4.quantize8(P.weight().to(dev), g, sym)
    X = P.activation(M).to(dev)
    Y = torch.empty(M, P.N, dtype=torch.bfloat16, device=dev)
    psets = [(C, S, Z, X)] + [(C.clone(), S.clone(), Z.clone(), X.clone()) for _ in range(pcopies - 1)]
    def prefill_step(i):
        Cc, Sc, Zc, Xc = psets[i % pcopies]
        w4.gemm8(Xc, Cc, Sc, Zc, g, sym, out=Y)

    gs = graph_of(prefill_step, pcopies)
    pms = time_graphs(gs, 30)
    del gs, psets, C, S, Z, X, Y
    torch.cuda.empty_cache()
    ptf = 2 * M * P.N * P.K / (pms / 1e3) / 1e12
    return {"shape": f"N={N},K={K},g={g},asym; GEMV: both 7B-shaped layers, M=1",
            "quantize": {"us": qms * 1e3, "GB/s": qb / (qms / 1e3) / 1e9, "frac": qb / (qms / 1e3) / 1e9 / pk},
            "dequantize": {"us": dms * 1e3, "GB/s": db / (dms / 1e3) / 1e9, "frac": db / (dms / 1e3) / 1e9 / pk},
            "gemv_M1": {"us_per_step": gms * 1e3, "bytes_per_step": gbytes, "GB/s": gbs,
                        "frac": gbs / pk, "kernel": "gemv_decode_kernel (8-bit codes)"},
            "gemv_M1_70b": {"us_per_step": gms70 * 1e3, "bytes_per_step": gbytes70, "GB/s": gbs70,
                            "frac": gbs70 / pk, "kernel": "gemv_decode_kernel (8-bit codes)",
                            "layers_KxN": [[l.K, l.N] for l in workloads.DECODE_70B.layers]},
            "prefill_2048x8192x8192": {"us": pms * 1e3, "TFLOP/s": ptf,
                                       "frac": ptf / peaks["bf16_tflops"],
                                       "kernel": "gemm_tc_kernel (8-bit codes)"}}


# Dense INT8 tensor-core rate relative to bf16 (nominal 4.5 vs 2.25 PFLOP/s per
# B200): the INT8 roofline is the measured bf16 peak times this ratio.
INT8_OVER_BF16 = 2.0


def w8a8_extras(w4, peaks, l2, dev, iters=30):
    """W8A8 at the prefill shape (M=2048, K=N=8192): per-token activation
    quantization, the INT8 tensor-core GEMM, and both together, graph-replayed
    over copies past L2; TOPS against the INT8 roofline (measured bf16 burst
    peak x 2, the nominal INT8/bf16 ratio)."""
    layer = workloads.PREFILL.layers[0]
    M, N, K = 2048, layer.N, layer.K
    C, S = w4.quantize8(layer.weight().to(dev), K, True)[:2]
    X = layer.activation(M).to(dev)
    copies = copies_for(N * K + 2 * M * K, l2)
    Cs = [C] + [C.clone() for _ in range(copies - 1)]
    Xs = [X] + [X.clone() for _ in range(copies - 1)]
    qs = [w4.quantize_act8(x) for x in Xs]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    gs = graph_of(lambda i: w4.quantize_act8(Xs[i % copies], out=qs[i % copies]), copies)
    qms = time_graphs(gs, iters)
    del gs
    gs = graph_of(lambda i: w4.gemm_w8a8(*qs[i % copies], Cs[i % copies], S, out=Y), copies)
    gms = time_graphs(gs, iters)
    del gs
    gs = graph_of(lambda i: (w4.quantize_act8(Xs[i % copies], out=qs[i % copies]),
                             w4.gemm_w8a8(*qs[i % copies], Cs[i % copies], S, out=Y)), copies)
    bms = time_graphs(gs, iters)
    del gs, Cs, Xs, qs, Y
    torch.cuda.empty_cache()
    ops = 2 * M * N * K
    pk = peaks["bf16_tflops"] * INT8_OVER_BF16
    tops = ops / (gms / 1e3) / 1e12
    qbytes = 2 * M * K + M * K + 4 * M
    return {"shape": f"M={M},K={K},N={N}; weights per-channel int8, activations per-token int8",
            "quantize_activations": {"us": qms * 1e3, "GB/s": qbytes / (qms / 1e3) / 1e9,
                                     "frac": qbytes / (qms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "gemm": {"us": gms * 1e3, "TOPS": tops,
                     "roofline": {"bound": "tensor", "achieved": tops, "peak": pk, "unit": "TOPS",
                                  "frac": tops / pk,
                                  "peak_source": "measured bf16 burst x 2 (nominal INT8/bf16 ratio)",
                                  "traffic": ncu_traffic("gemm_w8a8_kernel:w8a8")},
                     "kernel": "gemm_w8a8_kernel"},
            "quantize_and_gemm": {"us": bms * 1e3, "TOPS": ops / (bms / 1e3) / 1e12}}


def act_scale_extras(w4, l2, dev, iters=100):
    """Cost of the fused per-input-channel activation scale (w4a16_gemm_act_scaled):
    the same GEMM with and without a[K], graph-replayed over weight copies past
    L2 — the first 70B-shaped layer at M=1 (decode kernel) and the M=2048,
    K=N=8192 prefill (tensor-core kernel)."""
    out = {}
    for name, layer, M in (("decode70b_layer0_M1", workloads.DECODE_70B.layers[0], 1),
                           ("prefill_2048x8192x8192", workloads.PREFILL.layers[0], 2048)):
        g, sym = 128, False
        copies = copies_for(input_bytes(M, layer.N, layer.K, g, sym), l2)
        case = GemmCase(w4, layer, M, g, sym, copies, dev)
        a = workloads.make_act_scale(layer.K, 77).to(dev)
        times = {}
        for label, act in (("plain_us", None), ("act_scaled_us", a)):
            def call(i, act=act):
                j = i % copies
                w4.gemm(case.X[j], case.P[j], case.S[j], case.Z[j], g, sym, out=case.Y[j], act_scale=act)
            gs = graph_of(call, copies)
            times[label] = time_graphs(gs, iters if M == 1 else 20) * 1e3
            del gs
        times["overhead"] = times["act_scaled_us"] / times["plain_us"] - 1.0
        out[name] = times
        del case, a
        torch.cuda.empty_cache()
    return out


def comparisons(w4, cases, copies, l2, half):
    """Dense bf16 cuBLAS GEMM and the unfused dequantize-then-GEMM at the same
    shapes, timed the same way (graphs, rotation past L2)."""
    out = {}
    dense_bytes = sum(c.N * c.K * 2 for c in cases)
    dcopies = max(2, -(-2 * l2 // dense_bytes) + 1)
    Wd = [[c.W_dense] + [c.W_dense.clone() for _ in range(dcopies - 1)] for c in cases]

    def dense(i):
        for c, ws in zip(cases, Wd):
            torch.matmul(c.X[0], ws[i % dcopies].t(), out=c.Y[0])

    gs = graph_of(dense, dcopies)
    ms = time_graphs(gs, 200)
    out["dense_bf16_cublas"] = {"ms_per_step": ms, "bytes_per_step": dense_bytes}
    del gs
    Wh = [torch.empty_like(c.W_dense) for c in cases]

    def unfused(i):
        for c, wh in zip(cases, Wh):
            j = i % copies
            w4.dequantize(c.P[j], c.S[j], c.Z[j], c.g, c.sym, out=wh)
            torch.matmul(c.X[j], wh.t(), out=c.Y[j])

    gs = graph_of(unfused, copies)
    out["unfused_dequant_then_cublas"] = {"ms_per_step": time_graphs(gs, 100)}
    del gs
    fused = graph_of(lambda i: [c.call(w4, i) for c in cases], copies)
    out["fused_w4a16"] = {"ms_per_step": time_graphs(fused, 200)}
    out["speedup_vs_dense"] = out["dense_bf16_cublas"]["ms_per_step"] / out["fused_w4a16"]["ms_per_step"]
    out["speedup_vs_unfused"] = (out["unfused_dequant_then_cublas"]["ms_per_step"] /
                                 out["fused_w4a16"]["ms_per_step"])
    del Wd
    torch.cuda.empty_cache()
    return out


def prefill_extra(w4, peaks, peak_src, l2, dev, iters=50):
    """The metric's other half: TFLOPS at M=2048, K=N=8192 (g=128, asym)."""
    layer = workloads.PREFILL.layers[0]
    M = 2048
    in_bytes = layer.N * layer.K // 2 + 4 * layer.N * (layer.K // 128) + 2 * M * layer.K
    copies = copies_for(in_bytes, l2)
    case = GemmCase(w4, layer, M, 128, False, copies, dev)
    rot, singles = capture_rotation_graph(w4, [case], copies)
    replay_steps(rot, singles, copies, 3)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    replay_steps(rot, singles, copies, iters)
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / iters
    kms = ms
    tflops = case.flops / (kms / 1e3) / 1e12
    pk = peaks["bf16_tflops"]
    res = {"workload": "prefill_2048x8192x8192_g128_asym", "ms_per_step": ms,
           "TFLOP/s": case.flops / (ms / 1e3) / 1e12,
           "roofline": {"bound": "tensor", "achieved": tflops, "peak": pk, "unit": "TFLOP/s",
                        "frac": tflops / pk, "peak_source": peak_src + " (burst)",
                        "traffic": ncu_traffic("gemm_tc_kernel:prefill"),
                        "kernel": "gemm_tc_kernel", "per_launch_us": kms * 1e3},
           "plan": w4.plan(M, layer.N, layer.K, 128, False)}
    dcopies = max(2, -(-2 * l2 // (layer.N * layer.K * 2 + 2 * M * layer.K)) + 1)
    Wd = [case.W_dense] + [case.W_dense.clone() for _ in range(dcopies - 1)]
    Xd = [case.X[0]] + [case.X[0].clone() for _ in range(dcopies - 1)]
    gs = graph_of(lambda i: torch.matmul(Xd[i % dcopies], Wd[i % dcopies].t(), out=case.Y[0]),
                  dcopies)
    dms = time_graphs(gs, iters)
    res["dense_bf16_cublas"] = {"ms_per_step": dms, "TFLOP/s": case.flops / (dms / 1e3) / 1e12}
    del gs, Wd, Xd, rot, singles, case
    torch.cuda.empty_cache()
    return res


CROSSOVER_MODES = ((128, False), (128, True), (64, False), (64, True), (32, False), (32, True))


def crossover_rows(w4, dev, l2, iters=40, iters_large=12):
    """M-dispatch evidence at K=N=8192 (the crossover workload): for every M, g
    and mode, the time of each kernel that can run it (the decode kernel for
    M <= 16, the tensor-core kernel for every M), which one the dispatch takes,
    and — for g=128 asym — a dense bf16 cuBLAS GEMM of the same shape; inputs
    rotate over copies larger than L2.  Rows: {g, mode, M, dispatch, decode_us,
    tensorcore_us, dense_bf16_cublas_us, fastest, ...}."""
    layer = workloads.CROSSOVER.layers[0]
    N, K = layer.N, layer.K
    W = layer.weight().to(dev)
    rows = []
    for g, sym in CROSSOVER_MODES:
        P, S, Z = w4.quantize(W, g, sym)
        wbytes = N * K // 2 + 2 * N * (K // g) * (1 if sym else 2)
        copies = copies_for(wbytes, l2)
        Ps = [P] + [P.clone() for _ in range(copies - 1)]
        Ss = [S] + [S.clone() for _ in range(copies - 1)]
        Zs = [Z] + [Z.clone() for _ in range(copies - 1)]
        for M in workloads.CROSSOVER.Ms:
            X = layer.activation(M).to(dev)
            Xs = [X] + [X.clone() for _ in range(copies - 1)]
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            n = iters if M <= 1024 else iters_large
            row = {"g": g, "mode": "sym" if sym else "asym", "M": M,
                   "dispatch": w4.plan(M, N, K, g, sym)["path"],
                   "algorithmic_bytes": algorithmic_bytes(M, N, K, g, sym), "flops": 2 * M * N * K}
            for path in ("decode", "tensorcore"):
                if path == "decode" and M > 16:
                    continue
                # an NVTX range per measurement, so that a profiler's launch list can
                # name each kernel launch by (g, mode, M, kernel)
                torch.cuda.nvtx.range_push(f"xover_g{g}_{row['mode']}_M{M}_{path}")
                gs = graph_of(lambda i, path=path: w4.gemm(Xs[i % copies], Ps[i % copies],
                                                           Ss[i % copies], Zs[i % copies], g, sym,
                                                           path=path, out=Y, static_weights=True),
                              copies)
                row[path + "_us"] = round(time_graphs(gs, n) * 1e3, 3)
                torch.cuda.nvtx.range_pop()
                del gs
            if g == 128 and not sym:
                dcopies = max(2, -(-2 * l2 // (N * K * 2 + 2 * M * K)) + 1)
                Wd = [W] + [W.clone() for _ in range(dcopies - 1)]
                Xd = Xs[:1] + [X.clone() for _ in range(dcopies - 1)]
                torch.cuda.nvtx.range_push(f"xover_g{g}_{row['mode']}_M{M}_dense")
                gs = graph_of(lambda i: torch.matmul(Xd[i % dcopies], Wd[i % dcopies].t(), out=Y),
                              dcopies)
                row["dense_bf16_cublas_us"] = round(time_graphs(gs, n) * 1e3, 3)
                torch.cuda.nvtx.range_pop()
                del gs, Wd, Xd
            cand = {k[:-3]: v for k, v in row.items() if k in ("decode_us", "tensorcore_us")}
            row["fastest"] = min(cand, key=cand.get)
            t = row[row["dispatch"] + "_us"] * 1e-6
            row["dispatched_GBps"] = round(row["algorithmic_bytes"] / t / 1e9, 1)
            row["dispatched_TFLOPs"] = round(row["flops"] / t / 1e12, 2)
            rows.append(row)
            del Xs, X, Y
            torch.cuda.empty_cache()
        del P, S, Z, Ps, Ss, Zs
        torch.cuda.empty_cache()
    return rows


CROSSOVER8_MS = (1, 2, 4, 8, 12, 16, 24, 32, 64)


def crossover8_rows(w4, dev, l2, iters=40):
    """The same evidence for 8-bit codes (W8A16, g=128 asym, K=N=8192): the decode
    kernel (M <= 16) and the tensor-core kernel at each M, forced through
    w8a16_gemm_ex, and which one the dispatch takes."""
    layer = workloads.CROSSOVER.layers[0]
    N, K = layer.N, layer.K
    g, sym = 128, False
    C, S, Z = w4.quantize8(layer.weight().to(dev), g, sym)
    copies = copies_for(N * K + 4 * N * (K // g), l2)
    Cs = [C] + [C.clone() for _ in range(copies - 1)]
    Ss = [S] + [S.clone() for _ in range(copies - 1)]
    Zs = [Z] + [Z.clone() for _ in range(copies - 1)]
    rows = []
    for M in CROSSOVER8_MS:
        X = layer.activation(M).to(dev)
        Xs = [X] + [X.clone() for _ in range(copies - 1)]
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        row = {"g": g, "mode": "asym", "M": M, "dispatch": w4.plan8(M, N, K, g, sym)["path"],
               "algorithmic_bytes": algorithmic_bytes(M, N, K, g, sym) + N * K // 2}
        for path in ("decode", "tensorcore"):
            if path == "decode" and M > 16:
                continue
            torch.cuda.nvtx.range_push(f"xover8_M{M}_{path}")
            gs = graph_of(lambda i, path=path: w4.gemm8(Xs[i % copies], Cs[i % copies], Ss[i % copies],
                                                        Zs[i % copies], g, sym, out=Y, path=path,
                                                        static_weights=True), copies)
            row[path + "_us"] = round(time_graphs(gs, iters) * 1e3, 3)
            torch.cuda.nvtx.range_pop()
            del gs
        cand = {k[:-3]: v for k, v in row.items() if k in ("decode_us", "tensorcore_us")}
        row["fastest"] = min(cand, key=cand.get)
        rows.append(row)
        del Xs, X, Y
        torch.cuda.empty_cache()
    return rows


def crossover_sweep(args):
    """Print the crossover rows as one JSON object {"crossover": [...]}; not a
    benchmark line."""
    import weight_only_quantization_rtn_b200 as w4
    from weight_only_quantization_rtn_b200 import build as w4build
    w4build.build()
    w4.lib()
    dev = torch.device("cuda", 0)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 0) or L2_BYTES_FALLBACK
    if args.crossover8:
        print(json.dumps({"crossover_w8a16": crossover8_rows(w4, dev, l2)}))
    else:
        print(json.dumps({"crossover": crossover_rows(w4, dev, l2)}))


# Extras that bench.py --extra NAME runs alone (their ncu captures use that command).
EXTRAS = ("w8a8", "quantize", "w8a16")


def run_extra(args):
    """One extra of the benchmark line, printed alone ({"<name>": {...}})."""
    import weight_only_quantization_rtn_b200 as w4
    from weight_only_quantization_rtn_b200 import build as w4build
    w4build.build()
    w4.lib()
    dev = torch.device("cuda", 0)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 0) or L2_BYTES_FALLBACK
    peaks, _ = load_peaks()
    if args.extra == "w8a8":
        print(json.dumps({"w8a8": w8a8_extras(w4, peaks, l2, dev)}))
    elif args.extra == "quantize":
        print(json.dumps({"quantize_dequantize": elementwise_extras(w4, peaks, l2, dev)}))
    elif args.extra == "w8a16":
        print(json.dumps({"w8a16": w8a16_extras(w4, peaks, l2, dev)}))


def run_reference(args):
    """The reference arm: the host oracle as it stands, timed on this machine's
    cores, on the same workload and metric; each step a bounded sample."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl, M, g, sym, half, bits = WORKLOAD_DEFS[args.workload]
    if bits != 4:
        raise SystemExit("the reference arm times the 4-bit workloads")
    if half == "hbm":
        import oracle
        oracle.build()
        prepared = []
        for layer in wl.layers:
            Wb = workloads.bits(layer.weight())
            Xb = workloads.bits(layer.activation(M))
            P, S, Z = oracle.quantize(Wb, group_of(g, layer.K), sym)
            prepared.append((Xb, P, S, Z, group_of(g, layer.K)))
        bytes_step = sum(algorithmic_bytes(M, l.N, l.K, group_of(g, l.K), sym) for l in wl.layers)
        for _ in range(min(args.warmup, 1)):
            for Xb, P, S, Z, gl in prepared:
                oracle.gemm_w4a16(Xb, P, S, Z, gl, sym)
        steps = max(1, min(args.steps, 20))
        t0 = time.perf_counter()
        for _ in range(steps):
            for Xb, P, S, Z, gl in prepared:
                oracle.gemm_w4a16(Xb, P, S, Z, gl, sym)
        el = time.perf_counter() - t0
        value, unit = bytes_step * steps / el / 1e9, "GB/s"
        sample = f"{steps} full step(s): both layer GEMMs, dequantize + binary64 matmul"
        cores = oracle.num_threads()
    else:
        cb = cpu_baseline_sampled(wl.layers[0], M, g, sym, rows=16)
        steps, el = 1, cb["s_per_step"]
        value, unit, sample, cores = cb["value"], cb["unit"], cb["sample"], cb["cores"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": el / steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_name(wl, M, g, sym), "M": M,
                       "layers_KxN": [[l.K, l.N] for l in wl.layers],
                       "g": g if g else "K (per-channel)",
                       "mode": "sym" if sym else "asym"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_DEFS), default="decode70b")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip comparisons and the prefill half (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--crossover", action="store_true",
                    help="print the M-dispatch sweep at K=N=8192 instead of a benchmark line")
    ap.add_argument("--crossover8", action="store_true",
                    help="the same sweep for 8-bit codes (W8A16)")
    ap.add_argument("--extra", choices=list(EXTRAS),
                    help="print one extra measurement of the benchmark line by itself (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.extra:
        run_extra(args)
    elif args.crossover or args.crossover8:
        crossover_sweep(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
