"""Benchmark of the ternary linear layer on B200: one JSON line on rank 0.

A step is one decoded token (M = 1) through a synthetic 64-layer stack of 27B-class
ternary projections: per layer qkv (5120 -> 7168), o (5120 -> 5120), fused gate/up
(5120 -> 34816) and down (17408 -> 5120), every projection with its own weights
resident in HBM (64 distinct copies per shape: 5.6 GB PQ2_0 / 4.6 GB PTQ1_0, far
larger than the 126 MB L2, so nothing is served from cache between steps).  Each
projection is one bonsai_ternary_linear call: fused block-Hadamard rotation of x,
trit decode, group scales, reduction.  The 256 calls of a step are replayed from a
CUDA graph.

  value      whole-job HBM GB/s: algorithmic bytes of all ranks' steps (trit planes +
             FP16 scales + x + y) / max-over-ranks device time.
  roofline   the dominant kernel (the gate/up GEMV), timed live with CUDA events on
             its stream, against the measured HBM copy bandwidth.
  e2e        the same metric through the C ABI with pinned host buffers: every step
             copies the step's activations host -> device and its outputs back.
  cpu_baseline  the float64 CPU checker on a bounded sample (one layer), rank 0, N=1.

Multi-GPU: one process per GPU (torchrun); each rank decodes its own token stream
through its own copy of the stack (replicas, weak scaling, no collective on the
data path).  `--impl reference` times the CPU checker itself on the same metric.
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

METRIC = "batch-1 ternary GEMV HBM GB/s (% of 8 TB/s); prefill GEMM TFLOPS (% peak)"
SHAPES = [("qkv", 5120, 7168), ("o", 5120, 5120), ("gate_up", 5120, 34816), ("down", 17408, 5120)]
LAYERS = 64
FMT_NAMES = {1: "PTQ1_0", 2: "PQ2_0", 3: "Q1_0", 4: "PQ2_0_g64"}
FMTS = {"ptq1": 1, "pq2": 2, "q1": 3, "pq2g64": 4}
# the kernel a batch-1 call runs for each packing, and its source file
DOM_KERNEL = {1: "lookup-table GEMV (gemv_split_kernel + in-order reduction)",
              2: "integer tensor-core GEMV (gemv_imma_kernel)",
              3: "lookup-table GEMV (gemv_split_kernel, 1-bit tables + in-order reduction)",
              4: "integer tensor-core GEMV (gemv_imma_kernel, 64-weight scale groups)"}
DOM_SOURCE = {1: "gemv_lut.cu", 2: "gemv_imma.cu", 3: "gemv_lut.cu", 4: "gemv_imma.cu"}
# the arithmetic of that kernel: integer MMA (u8 codes x s8 bytes of 16-bit fixed-point x',
# s32 sums, then FP32 group scaling), or FP32 table sums
DECODE_DTYPE = {1: "f32", 2: "int8", 3: "f32", 4: "int8"}


def weights(fmt, seed, N, K):
    """Seeded weights of the workload: trits, or signs for the 1-bit Q1_0 packing."""
    from ternary_weight_02_b200 import inputs
    return inputs.signs(seed, N, K) if fmt == 3 else inputs.trits(seed, N, K)


def stack_workload(fmt):
    """The decode workload both arms report: the 64-layer linear stack, one token per step."""
    return (f"64-layer 27B-class linear stack at M=1 (qkv 5120->7168, o 5120->5120, "
            f"gate/up 5120->34816, down 17408->5120), {FMT_NAMES[fmt]}, one token per step")


def scale_group(fmt):
    """Weights per FP16 scale: 64 for the g64 variant of PQ2_0, else 128."""
    return 64 if fmt == 4 else 128


def scales(fmt, seed, N, K):
    """Seeded N x K/group FP16 scale plane of the workload."""
    from ternary_weight_02_b200 import inputs
    return inputs.scales(seed, N, K, group=scale_group(fmt))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def plane_bytes(fmt, N, K):
    trit = N * (K // 128) * 26 if fmt == 1 else (N * K // 8 if fmt == 3 else N * K // 4)
    return trit + N * (K // scale_group(fmt)) * 2


def step_bytes(fmt):
    """Algorithmic bytes of one token through the stack: weights + scales + x + y."""
    per_layer = sum(plane_bytes(fmt, N, K) + 2 * K + 2 * N for _, K, N in SHAPES)
    return LAYERS * per_layer


# NVML clock-event reason bits that the timing rules name (nvmlClocksEventReason*)
CLOCK_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


def summarize_clock_samples(samples):
    """Median SM clock, max SM clock and the throttle reasons seen in a list of
    (sm_mhz, sm_max_mhz, reasons_bitmask) samples; None without a valid sample."""
    sm = [float(a) for a, b, r in samples if a is not None and a > 0]
    smax = [float(b) for a, b, r in samples if b is not None and b > 0]
    if not sm:
        return None
    reasons = sorted({name for _, _, r in samples for bit, name in CLOCK_REASONS.items() if r & bit})
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax) if smax else None,
            "reasons": reasons, "samples": len(sm)}


class Clocks:
    """Samples the GPU's SM clock and clock-event reasons through NVML in a background
    thread (every 10 ms) while a timed region runs.  The NVML device is the one whose
    UUID matches the torch device, so a CUDA_VISIBLE_DEVICES remap cannot mislead it."""

    def __init__(self, torch_device_index):
        self.index = torch_device_index
        self.samples = []
        self.thread = None
        self.stop_flag = None
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            want = str(torch.cuda.get_device_properties(self.index).uuid).lower().replace("gpu-", "")
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
                if u == want:
                    self.handle = h
                    break
            self.nvml = pynvml
        except Exception:  # no NVML or no match: the line's clocks stay null
            self.handle = None

    def _sample(self):
        n = self.nvml
        try:
            sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
            smax = n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM)
            reasons = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
            self.samples.append((sm, smax, int(reasons)))
        except Exception:
            pass

    def start(self):
        if self.handle is None:
            return
        import threading
        self.samples = []
        self.stop_flag = threading.Event()

        def loop():
            while not self.stop_flag.is_set():
                self._sample()
                self.stop_flag.wait(0.01)

        self._sample()
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self._sample()
        self.stop_flag.set()
        self.thread.join(timeout=5)
        self.thread = None
        return summarize_clock_samples(self.samples)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(ms: float, device=None) -> float:
    """Max of a per-rank time over all ranks (the job's time); identity without a group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: all ranks' bytes of one step over the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_max * 1e-3) / 1e9


def kernel_traffic(fmt):
    """DRAM bytes per gate/up launch from the committed ncu summary, if it was taken on
    the kernel source as it is now (matched by hash); else None."""
    path = os.path.join(ROOT, "profiles", "gemv_traffic.json")
    src = os.path.join(ROOT, "ternary_weight_02_b200", "csrc", DOM_SOURCE[fmt])
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    ent = d.get(FMT_NAMES[fmt])
    if not ent or ent.get("source_sha256_16") != h:
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    """The CPU checker as it stands, timed on this host's cores: each step is one layer
    (the four projections) of the stack at M = 1, a bounded sample of the workload."""
    import oracle
    from ternary_weight_02_b200 import inputs
    fmt = FMTS[args.fmt]
    probs = []
    for i, (name, K, N) in enumerate(SHAPES):
        t = weights(fmt, i, N, K)
        probs.append((inputs.activations(i, 1, K), oracle.pack(fmt, t), scales(fmt, i, N, K), N, K))
    threads = oracle.max_threads()

    def one_step():
        for x, p, s, N, K in probs:
            oracle.ternary_linear(x, p, s, N, K, fmt)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = (time.perf_counter() - t0) / args.steps
    sample_bytes = step_bytes(fmt) / LAYERS
    value = sample_bytes / dt / 1e9
    sample = f"one layer (qkv, o, gate/up, down at M=1, {FMT_NAMES[fmt]}) of the 64-layer stack per step"
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": stack_workload(fmt), "sample": sample, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ our arm

def nvtx(torch, name):
    """A named NVTX range around a bench phase (visible to profilers; no cost otherwise)."""
    import contextlib

    @contextlib.contextmanager
    def rng():
        torch.cuda.nvtx.range_push(name)
        try:
            yield
        finally:
            torch.cuda.nvtx.range_pop()
    return rng()


def base_planes(fmt, dev, bz, torch):
    """One seeded packed plane, scale plane and FP16 x (M = 1) per projection shape."""
    from ternary_weight_02_b200 import inputs
    out = []
    for i, (name, K, N) in enumerate(SHAPES):
        t = torch.from_numpy(weights(fmt, i, N, K)).to(dev)
        packed = bz.pack(fmt, t)
        del t
        s = torch.from_numpy(scales(fmt, i, N, K).view(np.int16)).to(dev).view(torch.float16)
        out.append((packed, s))
    return out


def build_stack(fmt, base, dev, torch):
    """Weights of the 64-layer stack: LAYERS distinct copies of each shape's planes (far
    more than L2 holds, so every step streams them from HBM); x and y per shape."""
    from ternary_weight_02_b200 import inputs
    stack, xs, ys = [], [], []
    for i, (name, K, N) in enumerate(SHAPES):
        packed, s = base[i]
        stack.append([(packed.clone(), s.clone()) for _ in range(LAYERS)])
        xs.append(torch.from_numpy(inputs.activations(i, 1, K).view(np.int16)).to(dev).view(torch.float16))
        ys.append(torch.empty((1, N), dtype=torch.float16, device=dev))
    return stack, xs, ys


def capture(torch, stream, fn):
    """fn() enqueued once eagerly (first-use set-up), then captured into a CUDA graph."""
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


def time_graph(torch, stream, g, reps, warmup=3):
    """Device time of one replay of g in ms: CUDA events on its stream around reps replays."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_decode(f, base, dev, bz, torch, args, world, hbm):
    """The decode stack of packing f (step time, e2e), each projection's batch-1 call
    time in a graph of LAYERS calls on distinct weight copies, and the live timing of the
    dominant (gate/up) kernel."""
    stack, xs, ys = build_stack(f, base, dev, torch)
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream

    def enqueue(only=None):
        for layer in range(LAYERS):
            for i, (name, K, N) in enumerate(SHAPES):
                if only is not None and i != only:
                    continue
                p, s = stack[i][layer]
                bz.bonsai_ternary_linear(xs[i], p, s, ys[i], 1, N, K, f, sp)

    g = capture(torch, stream, enqueue)
    # ---- device-resident timing of the whole step
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    clocks = Clocks(dev.index)
    clocks.start()
    with nvtx(torch, f"decode stack {FMT_NAMES[f]}"):
        ms = time_graph(torch, stream, g, args.steps, warmup=0)
    clk = clocks.stop()
    ms = max_over_ranks(ms, dev)
    value = whole_job_gbs(step_bytes(f), world, ms)

    # ---- each projection alone: LAYERS calls per replay, each on its own weight copy
    per = {}
    with nvtx(torch, f"per-projection {FMT_NAMES[f]}"):
        for i, (name, K, N) in enumerate(SHAPES):
            gi = capture(torch, stream, lambda i=i: enqueue(only=i))
            reps = max(3, args.steps)
            us = time_graph(torch, stream, gi, reps) * 1e3 / LAYERS
            b = plane_bytes(f, N, K) + 2 * K + 2 * N
            per[name] = {"K": K, "N": N, "us": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                         "frac": round(b / (us * 1e-6) / 1e9 / hbm, 4), "bytes": b,
                         "launches": bz.bonsai_launch_count(1, N, K, f)}
            del gi

    # ---- end to end through the C ABI with host buffers
    hx = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in xs]
    for h, x in zip(hx, xs):
        h.copy_(x.cpu())
    hy = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in ys]
    h2d = sum(h.numel() * h.element_size() for h in hx)
    d2h = sum(h.numel() * h.element_size() for h in hy)

    def e2e_step():
        for h, x in zip(hx, xs):
            x.copy_(h, non_blocking=True)
        g.replay()
        for h, y in zip(hy, ys):
            h.copy_(y, non_blocking=True)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with nvtx(torch, f"e2e {FMT_NAMES[f]}"), torch.cuda.stream(stream):
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    e2e = whole_job_gbs(step_bytes(f), world, ms_e2e)

    launches_per_layer = sum(bz.bonsai_launch_count(1, N, K, f) for _, K, N in SHAPES)
    out = {"launches_per_layer": launches_per_layer, "value": value, "ms": ms, "clocks": clk,
           "per_projection": per, "e2e": e2e, "h2d": h2d, "d2h": d2h, "traffic": kernel_traffic(f)}
    if f == 2:
        out["swiglu_decode"] = measure_swiglu_decode(stack, xs, bz, torch, stream, dev, args)
    if args.skinny and f in (1, 2):
        out["skinny_grid"] = measure_skinny_grid(f, stack, dev, bz, torch, stream, args, hbm)
    del stack, g
    torch.cuda.synchronize()
    return out


def measure_skinny_grid(f, stack, dev, bz, torch, stream, args, hbm):
    """Decode batches of M in {1, 2, 4, 8, 16} tokens on each projection: the automatic
    choice (the integer GEMV for PQ2_0 at M <= 2 where K allows, else the skinny kernel or
    the lookup-table GEMV), the skinny kernel with and without split-K, and the prefill
    GEMM, each as LAYERS calls on distinct weight copies per replay.  GB/s counts the
    weight, scale, x and y bytes."""
    from ternary_weight_02_b200 import inputs
    sp = stream.cuda_stream
    grid = {}
    variants = [("auto", bz.BONSAI_ALGO_AUTO, 0), ("skinny", bz.BONSAI_ALGO_SKINNY, 0),
                ("skinny_no_split", bz.BONSAI_ALGO_SKINNY, 1), ("gemm", bz.BONSAI_ALGO_GEMM, 0)]
    with nvtx(torch, f"skinny grid {FMT_NAMES[f]}"):
        for M in (1, 2, 4, 8, 16):
            for i, (name, K, N) in enumerate(SHAPES):
                x = torch.from_numpy(inputs.activations(100 + i, M, K).view(np.int16)).to(dev).view(torch.float16)
                y = torch.empty((M, N), dtype=torch.float16, device=dev)
                b = plane_bytes(f, N, K) + 2 * M * K + 2 * M * N
                row = {}
                for vname, algo, sk in variants:
                    try:
                        bz.bonsai_launch_count(M, N, K, f, algo, sk)
                    except bz.BonsaiError:
                        continue  # this kernel does not take the shape or packing

                    def enq(algo=algo, sk=sk):
                        for layer in range(LAYERS):
                            p, s = stack[i][layer]
                            bz.bonsai_ternary_linear_algo(x, p, s, y, M, N, K, f, algo, sk, sp)
                    gi = capture(torch, stream, enq)
                    us = time_graph(torch, stream, gi, max(3, args.steps // 4)) * 1e3 / LAYERS
                    row[vname] = {"us": round(us, 2), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                                  "frac": round(b / (us * 1e-6) / 1e9 / hbm, 4)}
                    del gi
                grid[f"M{M}_{name}"] = row
    return {"workload": (f"M in {{1,2,4,8,16}} tokens x the four 27B-class projections, {FMT_NAMES[f]}, "
                         f"{LAYERS} distinct weight copies per replay (weights re-read from HBM)"),
            "unit": "us per call", "grid": grid}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from ternary_weight_02_b200 import bonsai as bz

    world, rank, local = dist_setup()
    # bind this rank to its GPU before the process group so that NCCL uses it
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    if bz.bonsai_check_device() != bz.BONSAI_OK:
        raise RuntimeError("libbonsai: not an sm_100 device")
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    fmt = FMTS[args.fmt]
    bz.bonsai_reserve(16, 34816, 17408)

    results = {}
    prefill = None
    for f in ([fmt] + [o for o in (2, 1, 3, 4) if o != fmt]) if args.both else [fmt]:
        base = base_planes(f, dev, bz, torch)
        results[f] = measure_decode(f, base, dev, bz, torch, args, world, hbm)
        if args.prefill_m > 0 and f in (1, 2) and (args.both or f == fmt):
            pg = measure_prefill(f, base, dev, bz, torch, args, peaks, peak_kind)
            prefill = pg if prefill is None else {**prefill, "grid": {**prefill["grid"], **pg["grid"]}}
        del base
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    r = results[fmt]
    line = None
    if rank == 0:
        dom = r["per_projection"]["gate_up"]
        line = {
            "metric": METRIC, "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"], 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DECODE_DTYPE[fmt],
            "data": "synthetic (seeded SplitMix64 trits P(0)=.38, FP16 scales U[.01,.05], FP16 x N(0,1))",
            "config": {
                "workload": stack_workload(fmt),
                "packing": FMT_NAMES[fmt], "layers": LAYERS, "tokens_per_step": 1,
                "bytes_per_step": step_bytes(fmt), "l2": "inputs larger than L2 (weights re-read every step)",
                "per_token_us": round(r["ms"] * 1e3, 2), "frac_of_8TBps": round(r["value"] / 8000.0, 4),
                "frac_of_measured_hbm": round(r["value"] / hbm, 4), "parallelism": f"replicas x{world}",
            },
            "roofline": {
                "bound": "hbm", "kernel": f"{DOM_KERNEL[fmt]}, gate/up 5120->34816", "achieved": dom["gbs"],
                "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom["gbs"] / hbm, 4),
                "traffic": r["traffic"], "algorithmic_bytes_per_launch": dom["bytes"],
                "avg_launch_us": dom["us"],
            },
            "e2e": {"value": round(r["e2e"], 1), "unit": "GB/s", "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"]},
            "gpu_launches": LAYERS * r["launches_per_layer"] * args.steps,
            "clocks": r["clocks"],
            "per_projection": {FMT_NAMES[k]: v["per_projection"] for k, v in results.items()},
        }
        others = {FMT_NAMES[k]: {"value": round(v["value"], 1), "unit": "GB/s",
                                 "per_token_us": round(v["ms"] * 1e3, 2),
                                 "gate_up_gbs": v["per_projection"]["gate_up"]["gbs"], "e2e": round(v["e2e"], 1),
                                 "clocks": v["clocks"]}
                  for k, v in results.items() if k != fmt}
        if others:
            line["other_packings"] = others
        grids = {FMT_NAMES[k]: v["skinny_grid"] for k, v in results.items() if "skinny_grid" in v}
        if grids:
            line["skinny"] = grids
        sw = next((v["swiglu_decode"] for v in results.values() if "swiglu_decode" in v), None)
        if sw is not None:
            line["swiglu"] = {"decode": sw}
        if prefill is not None:
            if "swiglu_gate_up" in prefill:
                line.setdefault("swiglu", {})["prefill"] = prefill.pop("swiglu_gate_up")
            line["prefill"] = prefill
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def measure_swiglu_decode(stack, xs, bz, torch, stream, dev, args):
    """The MLP's gate/up projection at M = 1 followed by SwiGLU, 64 layers per replay:
    fused (bonsai_ternary_linear_swiglu: the integer GEMV's epilogue applies it) against
    the linear call and then bonsai_swiglu (a second kernel)."""
    _, K, N = SHAPES[2]
    F = N // 2
    h = torch.empty((1, F), dtype=torch.float16, device=dev)
    y2 = torch.empty((1, N), dtype=torch.float16, device=dev)
    sp = stream.cuda_stream
    out = {}
    for fused in (True, False):
        def enq():
            for layer in range(LAYERS):
                p, s = stack[2][layer]
                if fused:
                    bz.bonsai_ternary_linear_swiglu(xs[2], p, s, h, 1, F, K, 2, sp)
                else:
                    bz.bonsai_ternary_linear(xs[2], p, s, y2, 1, N, K, 2, sp)
                    bz.bonsai_swiglu(y2, h, 1, F, sp)
        g = capture(torch, stream, enq)
        us = time_graph(torch, stream, g, max(3, args.steps)) * 1e3 / LAYERS
        out["fused_us_per_layer" if fused else "unfused_us_per_layer"] = round(us, 3)
        del g
    out["workload"] = f"gate/up 5120 -> 2 x {F} at M=1 then SwiGLU, 64 distinct weight copies per replay, PQ2_0"
    return out


PREFILL_MS = (512, 2048, 8192)  # the prefill workload's token counts


def measure_prefill(fmt, base, dev, bz, torch, args, peaks, peak_kind):
    """Prefill: M tokens through each of the four projections (tcgen05 GEMM with the
    rotation of x), for M in PREFILL_MS.  Every call is timed on its own with CUDA events,
    after a write of twice the L2 size that evicts the previous call's data; at least 20
    calls per (M, projection)."""
    from ternary_weight_02_b200 import inputs
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    flush = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size, dtype=torch.uint8, device=dev)
    calls = max(20, args.steps)
    burst = float(peaks["bf16_tflops"])
    grid = {}
    summary = None
    for M in args.prefill_ms:
        per = {}
        total_flop, layer_us = 0, 0.0
        for i, (name, K, N) in enumerate(SHAPES):
            packed, s = base[i]
            x = torch.from_numpy(inputs.activations(200 + i, M, K).view(np.int16)).to(dev).view(torch.float16)
            y = torch.empty((M, N), dtype=torch.float16, device=dev)
            bz.bonsai_reserve(M, N, K)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
            with nvtx(torch, f"prefill M={M} {name} {FMT_NAMES[fmt]}"), torch.cuda.stream(stream):
                for _ in range(2):
                    bz.bonsai_ternary_linear(x, packed, s, y, M, N, K, fmt, sp)
                for a, b in ev:
                    flush.fill_(1)
                    a.record(stream)
                    bz.bonsai_ternary_linear(x, packed, s, y, M, N, K, fmt, sp)
                    b.record(stream)
            torch.cuda.synchronize()
            us = sum(a.elapsed_time(b) for a, b in ev) * 1e3 / calls
            flop = 2 * M * N * K
            total_flop += flop
            layer_us += us
            per[name] = {"us": round(us, 1), "tflops": round(flop / us / 1e6, 1),
                         "frac": round(flop / us / 1e6 / burst, 4), "calls": calls,
                         "launches": bz.bonsai_launch_count(M, N, K, fmt)}
            del x, y
        grid[f"{FMT_NAMES[fmt]}_M{M}"] = {"per_projection": per, "us_per_layer": round(layer_us, 1),
                                          "tflops": round(total_flop / layer_us / 1e6, 1)}
        if M == args.prefill_m:
            dom = per["gate_up"]
            summary = {
                "metric": "prefill GEMM TFLOP/s", "value": round(total_flop / layer_us / 1e6, 1), "unit": "TFLOP/s",
                "workload": f"M={M} tokens x the four 27B-class projections, {FMT_NAMES[fmt]}, "
                            f"FP16 x FP16 -> FP32 (tcgen05)",
                "us_per_layer": round(layer_us, 1), "per_projection": per,
                "roofline": {"bound": "tensor", "kernel": "gemm gate/up 5120->34816 (incl. the rotation of x)",
                             "achieved": dom["tflops"], "peak": burst,
                             "peak_kind": f"{peak_kind} bf16 burst (fp16 same dense rate)",
                             "unit": "TFLOP/s", "frac": round(dom["tflops"] / burst, 4),
                             "frac_of_sustained": round(dom["tflops"] / float(peaks["bf16_tflops_sustained"]), 4),
                             "traffic": None},
            }
    out = {"grid": grid, "l2": "every call after a write of 2x the L2 size", "calls_per_entry": calls}
    if summary is not None:
        out.update(summary)
    if fmt == 2 and args.prefill_m in args.prefill_ms:
        out["swiglu_gate_up"] = measure_swiglu_prefill(fmt, base, dev, bz, torch, args.prefill_m, calls, flush)
    return out


def measure_swiglu_prefill(fmt, base, dev, bz, torch, M, calls, flush):
    """gate/up then SwiGLU at M tokens: fused in the GEMM's epilogue against the GEMM and
    bonsai_swiglu."""
    from ternary_weight_02_b200 import inputs
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    name, K, N = SHAPES[2]
    packed, s = base[2]
    F = N // 2
    x = torch.from_numpy(inputs.activations(202, M, K).view(np.int16)).to(dev).view(torch.float16)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    h = torch.empty((M, F), dtype=torch.float16, device=dev)
    sw = {}
    for fused in (True, False):
        def call():
            if fused:
                bz.bonsai_ternary_linear_swiglu(x, packed, s, h, M, F, K, fmt, sp)
            else:
                bz.bonsai_ternary_linear(x, packed, s, y, M, N, K, fmt, sp)
                bz.bonsai_swiglu(y, h, M, F, sp)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
        with torch.cuda.stream(stream):
            call()
            for a, b in ev:
                flush.fill_(1)
                a.record(stream)
                call()
                b.record(stream)
        torch.cuda.synchronize()
        sw["fused_us" if fused else "unfused_us"] = round(sum(a.elapsed_time(b) for a, b in ev) * 1e3 / calls, 1)
    sw["workload"] = f"M={M} x gate/up 5120 -> 2 x {F} then SwiGLU, {FMT_NAMES[fmt]}"
    return sw


def cpu_baseline(fmt):
    """The checker on one layer of the stack (rank 0, N = 1): a bounded CPU sample, timed
    on all host cores and on one."""
    import oracle
    from ternary_weight_02_b200 import inputs
    probs = []
    for i, (name, K, N) in enumerate(SHAPES):
        probs.append((inputs.activations(i, 1, K), oracle.pack(fmt, weights(fmt, i, N, K)),
                      scales(fmt, i, N, K), N, K))

    def timed(threads):
        t0 = time.perf_counter()
        for x, p, s, N, K in probs:
            oracle.ternary_linear(x, p, s, N, K, fmt, nthreads=threads)
        return time.perf_counter() - t0

    cores = oracle.max_threads()
    dt_all, dt_one = timed(cores), timed(1)
    layer = step_bytes(fmt) / LAYERS
    sample = f"one layer (4 projections, M=1, {FMT_NAMES[fmt]}) of the 64-layer stack, float64"
    return {"value": round(layer / dt_all / 1e9, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": sample,
            "single_thread": {"value": round(layer / dt_one / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "kind": "oracle", "sample": sample}}


def run_case(args):
    """One projection, `reps` calls (a small case for profilers: python bench.py --case ...)."""
    import torch
    from ternary_weight_02_b200 import bonsai as bz
    from ternary_weight_02_b200 import inputs
    fmt = FMTS[args.fmt]
    i = [n for n, _, _ in SHAPES].index(args.shape)
    _, K, N = SHAPES[i]
    # the integer GEMV takes batches of up to 3 tokens (--m); the lookup-table GEMV one
    M = 1 if args.case == "gemv" or (args.case == "imma" and args.m > 3) else args.m
    dev = torch.device("cuda")
    t = torch.from_numpy(weights(fmt, i, N, K)).to(dev)
    packed = bz.pack(fmt, t)
    del t
    s = torch.from_numpy(scales(fmt, i, N, K).view(np.int16)).to(dev).view(torch.float16)
    x = torch.from_numpy(inputs.activations(i, M, K).view(np.int16)).to(dev).view(torch.float16)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    algo = {"gemv": bz.BONSAI_ALGO_GEMV, "imma": bz.BONSAI_ALGO_IMMA, "gemm": bz.BONSAI_ALGO_GEMM,
            "skinny": bz.BONSAI_ALGO_SKINNY}[args.case]
    bz.bonsai_reserve(M, N, K)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.reps):
        bz.bonsai_ternary_linear_algo(x, packed, s, y, M, N, K, fmt, algo, args.tile)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.reps
    print(json.dumps({"case": args.case, "shape": args.shape, "fmt": FMT_NAMES[fmt], "M": M, "K": K, "N": N,
                      "tile": args.tile, "reps": args.reps, "us_per_call": round(us, 2)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--fmt", choices=list(FMTS), default="pq2")
    ap.add_argument("--both", type=int, default=1, help="also measure the other packing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-m", type=int, default=2048,
                    help="tokens of the prefill summary line, one of 512, 2048, 8192 (0: skip the prefill grid)")
    ap.add_argument("--prefill-ms", default=",".join(str(m) for m in PREFILL_MS),
                    help="token counts of the prefill grid (comma-separated)")
    ap.add_argument("--skinny", type=int, default=1, help="measure the M = 1..16 decode grid (PQ2_0, PTQ1_0)")
    ap.add_argument("--case", choices=["gemv", "imma", "gemm", "skinny"], help="run one projection only (profiler case)")
    ap.add_argument("--shape", choices=[n for n, _, _ in SHAPES], default="gate_up")
    ap.add_argument("--m", type=int, default=2048,
                    help="tokens for --case gemm / skinny / imma (skinny: at most 16; imma: 1 to 3, else 1)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--tile", type=int, default=0,
                    help="--case: the kernel's split/tile argument (GEMM: 1, 2 or 3 = CTA pairs; 0 automatic)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.prefill_ms = tuple(int(m) for m in args.prefill_ms.split(",") if m)

    world, rank, _ = dist_setup()
    if args.case:
        run_case(args)
        return
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    line = run_ours(args)
    if rank == 0 and line is not None:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(FMTS[args.fmt])
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
