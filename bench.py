"""Benchmark of the OWQ mixed-precision weight-only matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl owq|reference]
                    [--workload opt-6.7b-decode|llama-7b-decode|opt-66b-decode] [--M m]

Default workload (the decode configuration the metric is quoted on): OPT-6.7B-shaped decoder
layer sets (q, k, v, out 4096x4096; fc1 16384x4096; fc2 4096x16384), 3-bit per-output-channel
codes, k = K/128 fp16 weak columns, one token (M = 1).  A step is one token through a stack of
32 such layer sets with distinct resident weights (2.5 GB, 20x the L2), i.e. 192 products;
q/k/v share one launch (owq_gemv_multi).  Each step is a CUDA graph; the timed region replays
exactly K of them between a barrier + synchronize on both sides.

value = effective weight GB/s of the whole job (algorithmic bytes of all products / time),
with inputs resident in HBM.  e2e = the same metric with each step's activations copied in
from pinned host memory and its outputs read back inside the timed region.  With N > 1 every
rank streams its own stack (independent replicas, weak scaling, no collective on the path);
time is the max over ranks.  --impl reference times the CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
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

import owq_synth  # noqa: E402

METRIC = "decode GEMV µs/layer & effective weight GB/s (frac. of HBM peak); prefill TFLOP/s"
UNIT = "GB/s"
DEPTH = {"opt-6.7b-decode": 32, "llama-7b-decode": 32, "opt-66b-decode": 64}
WID = {"opt-6.7b-decode": 1, "llama-7b-decode": 2, "opt-66b-decode": 3}
# launches of one layer set: layers sharing an input (q/k/v, gate/up) are one multi launch
GROUPS = {
    "opt-6.7b-decode": [["q", "k", "v"], ["out"], ["fc1"], ["fc2"]],
    "llama-7b-decode": [["q", "k", "v"], ["o"], ["gate", "up"], ["down"]],
    "opt-66b-decode": [["q", "k", "v"], ["out"], ["fc1"], ["fc2"]],
}


# ---------------------------------------------------------------------------------- ranks
def dist_setup():
    """(rank, world, local_rank); initialises torch.distributed when WORLD_SIZE > 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        # a short timeout: a rank that dies or never joins ends the others' next collective
        # with an error instead of a wait
        secs = float(os.environ.get("OWQ_PG_TIMEOUT_S", "120"))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=secs))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------- helpers
def layer_bytes(N, K, bits, group, k, M):
    """Algorithmic bytes of one product: packed codes (weak slots included: the latency layout
    stores them), fp16 scale+zero per (row, group), fp16 weak block, int32 indices, x, y."""
    G = K // group
    return N * K * bits // 8 + N * G * 4 + N * k * 2 + 4 * k + 2 * M * K + 2 * M * N


def weight_bytes(N, K, bits, group, k):
    G = K // group
    return N * K * bits // 8 + N * G * 4 + N * k * 2 + 4 * k


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            self.max_mhz = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        self._t.start()
        return self

    def __exit__(self, *a):
        self._sample()
        self._stop.set()
        self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def ncu_traffic(kernel_tag: str):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, or None when the
    kernel's source changed after the capture (the summary stores the source digest)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    src = os.path.join(ROOT, "weight_only_mixed_owq_b200", "csrc", vals.get("source", ""))
    if not os.path.exists(src):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if digest != vals.get("sha256_16"):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------------- owq arm
def build_stack(owq, torch, spec, depth, M, dev):
    """Quantise one layer set on the GPU and pack `depth` resident copies of it."""
    sets, info = [], {}
    inputs = {}
    for li, L in enumerate(spec.layers):
        short = L.name.split(".")[-1]
        d = owq_synth.draw_layer(L, spec, M, owq_synth.seed_for(spec.wid, li))
        W = torch.from_numpy(d["W"]).to(dev)
        X = torch.from_numpy(d["X"]).to(dev)
        q = owq.quantize(W, X, L.bits, L.group, L.k)
        del W, X
        inputs[short] = {"q": q, "x": torch.from_numpy(d["x"]).to(dev), "L": L}
        info[short] = L
    for c in range(depth):
        layers = {}
        for short, v in inputs.items():
            q, L = v["q"], v["L"]
            layers[short] = owq.OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"] if L.k else None,
                                         q["w_weak"] if L.k else None, L.bits, L.group)
        sets.append(layers)
    for v in inputs.values():
        del v["q"]
    torch.cuda.synchronize()
    return sets, inputs, info


class Stack:
    """`depth` resident copies of one quantised layer set of a decode workload, and the timed
    step over them: one token batch through every layer set, each launch group (layers that
    share an input: q/k/v, gate/up) one launch, captured as CUDA graphs."""

    def __init__(self, owq, torch, wl, depth, Mmax, dev):
        self.owq, self.torch, self.wl, self.depth, self.dev = owq, torch, wl, depth, dev
        self.spec = owq_synth.WORKLOADS[WID[wl]]
        self.groups = GROUPS[wl]
        self.sets, self.inputs, self.info = build_stack(owq, torch, self.spec, depth, Mmax, dev)

    def launch_bytes(self, names, M):
        info = self.info
        return sum(layer_bytes(info[n].N, info[n].K, info[n].bits, info[n].group, info[n].k, M) for n in names)

    def close(self):
        for c in self.sets:
            for L in c.values():
                L.close()
        self.sets = []

    def measure(self, M, steps, warmup, world, local, e2e=True):
        """Times `steps` replays of the step graph (after `warmup`); returns the figures of one
        bench line (GB/s of the algorithmic bytes, per-launch diagnostics, e2e)."""
        import torch

        from cuda.bindings import runtime as rt
        owq, dev, depth, groups, info = self.owq, self.dev, self.depth, self.groups, self.info
        xs = {n: v["x"][:M].contiguous() for n, v in self.inputs.items()}
        ys = {s: torch.empty((M, info[s].N), dtype=torch.float16, device=dev) for s in info}
        step_bytes = depth * sum(self.launch_bytes(g, M) for g in groups)
        step_wbytes = depth * sum(weight_bytes(info[n].N, info[n].K, info[n].bits, info[n].group, info[n].k)
                                  for g in groups for n in g)
        launches_per_step = depth * len(groups)
        sets = self.sets

        def issue(c, stream_ptr, ev=None):
            """Enqueue one layer set (copy c); optional external event pairs around each launch."""
            for gi, g in enumerate(groups):
                if ev is not None:
                    rt.cudaEventRecordWithFlags(ev[gi][0], stream_ptr, rt.cudaEventRecordExternal)
                if len(g) == 1:
                    st = owq.owq_gemv(sets[c][g[0]].handle, xs[g[0]], ys[g[0]], M, stream_ptr)
                else:
                    st = owq.owq_gemv_multi([sets[c][n].handle for n in g], [xs[n] for n in g],
                                            [ys[n] for n in g], M, stream_ptr)
                if st != 0:
                    raise RuntimeError(f"launch failed: {owq.owq_status_string(st)}")
                if ev is not None:
                    rt.cudaEventRecordWithFlags(ev[gi][1], stream_ptr, rt.cudaEventRecordExternal)

        stream = torch.cuda.Stream(device=dev)
        sp = stream.cuda_stream
        # eager warm-up of every copy (loads modules, sets kernel attributes)
        for c in range(depth):
            issue(c, sp)
        torch.cuda.synchronize()

        # the timed step: one CUDA graph of every launch, back to back, so that each kernel's
        # prologue overlaps the previous kernel's tail (programmatic dependent launch)
        NG = 2
        graphs = []
        for _ in range(NG):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                cs = torch.cuda.current_stream().cuda_stream
                for c in range(depth):
                    issue(c, cs)
            graphs.append(g)
        # diagnostic copy with an event pair around every launch (the events serialise the
        # launches, so these per-launch times exclude the overlap the timed step gets)
        ev_diag = [[[rt.cudaEventCreate()[1], rt.cudaEventCreate()[1]] for _ in groups] for _ in range(depth)]
        g_diag = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_diag, stream=stream):
            cs = torch.cuda.current_stream().cuda_stream
            for c in range(depth):
                issue(c, cs, ev_diag[c])

        for i in range(warmup):
            graphs[i % NG].replay()
        torch.cuda.synchronize()

        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            with torch.cuda.stream(stream):
                t0.record(stream)
                for i in range(steps):
                    graphs[i % NG].replay()
                t1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        ms_max = max_over_ranks(t0.elapsed_time(t1), world)

        # per-launch diagnostics from the instrumented copy (after the timed region)
        for _ in range(2):
            g_diag.replay()
        torch.cuda.synchronize()
        durs = []
        for c in range(depth):
            for gi, g in enumerate(groups):
                err, t = rt.cudaEventElapsedTime(ev_diag[c][gi][0], ev_diag[c][gi][1])
                durs.append(t if err == rt.cudaError_t.cudaSuccess else float("nan"))
        per_group = {}
        for j, g in enumerate(groups):
            sel = durs[j::len(groups)]
            if sel:
                us = 1e3 * sum(sel) / len(sel)
                per_group["+".join(g)] = {"us": round(us, 3), "GBps": round(self.launch_bytes(g, M) / (us * 1e-6) / 1e9, 1)}
        for pair in ev_diag:
            for a, b in pair:
                rt.cudaEventDestroy(a)
                rt.cudaEventDestroy(b)
        del g_diag

        out = {"M": M, "ms_per_step": ms_max / steps, "ms_max": ms_max, "step_bytes": step_bytes,
               "step_wbytes": step_wbytes, "launches_per_step": launches_per_step,
               "per_group": per_group, "clocks": clk.summary()}
        if e2e:
            # e2e graph: pinned host activations in, outputs out, around the same step
            host_x = {n: torch.empty_like(xs[n], device="cpu").pin_memory() for n in xs}
            for n in xs:
                host_x[n].copy_(xs[n].cpu())
            host_y = {n: torch.empty_like(ys[n], device="cpu").pin_memory() for n in ys}
            g_e2e = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_e2e, stream=stream):
                for n in xs:
                    xs[n].copy_(host_x[n], non_blocking=True)
                cs = torch.cuda.current_stream().cuda_stream
                for c in range(depth):
                    issue(c, cs)
                for n in ys:
                    host_y[n].copy_(ys[n], non_blocking=True)
            out["h2d"] = sum(v.numel() * v.element_size() for v in host_x.values())
            out["d2h"] = sum(v.numel() * v.element_size() for v in host_y.values())
            for _ in range(max(1, warmup)):
                g_e2e.replay()
            torch.cuda.synchronize()
            barrier(world)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for i in range(steps):
                    g_e2e.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            out["e2e_ms_max"] = max_over_ranks(e0.elapsed_time(e1), world)
            del g_e2e
        del graphs
        torch.cuda.synchronize()
        return out


def run_owq(args, rank, world, local):
    import torch

    import weight_only_mixed_owq_b200 as owq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = args.workload
    M = args.M
    depth = args.depth or DEPTH[wl]
    stack = Stack(owq, torch, wl, depth, M, dev)
    spec, groups, info = stack.spec, stack.groups, stack.info
    r = stack.measure(M, args.steps, args.warmup, world, local)
    ms_max, step_bytes, step_wbytes = r["ms_max"], r["step_bytes"], r["step_wbytes"]
    launches_per_step = r["launches_per_step"]

    # every launch of the timed region is the decode kernel: its average launch duration is
    # the timed region (CUDA events on the launching stream) over the launches in it
    launch_us = ms_max * 1e3 / (args.steps * launches_per_step)
    achieved = step_bytes * args.steps / (ms_max * 1e-3) / 1e9

    total_bytes = sum_over_ranks(step_bytes * args.steps, world)
    value = total_bytes / (ms_max * 1e-3) / 1e9
    e2e_value = total_bytes / (r["e2e_ms_max"] * 1e-3) / 1e9
    peaks, peak_kind = measured_peaks()
    per_layer_us = ms_max * 1e3 / args.steps / (depth * sum(len(g) for g in groups))

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": f"{wl}: {depth} resident OPT/LLaMA-shaped decoder layer sets per token, M={M}",
            "layers": {n: [info[n].N, info[n].K] for n in info},
            "bits": spec.layers[0].bits, "group": "per-channel" if spec.layers[0].group == spec.layers[0].K else spec.layers[0].group,
            "weak_cols": "K/128", "M": M, "products_per_step": depth * sum(len(g) for g in groups),
            "launches_per_step": launches_per_step, "step_bytes": step_bytes, "step_weight_bytes": step_wbytes,
            "l2": "inputs larger than L2 (distinct resident weights, no reuse within a step)",
            "per_layer_us": round(per_layer_us, 3),
            "weight_GBps": round(sum_over_ranks(step_wbytes * args.steps, world) / (ms_max * 1e-3) / 1e9, 2),
            "parallelism": f"replicas x{world}",
        },
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {
            "bound": "hbm",
            "kernel": "k_gemv (decode GEMV)",
            "achieved": round(achieved, 2) if achieved else None,
            "peak": peaks["hbm_gbs"],
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4) if achieved else None,
            "frac_of_8TBps_spec": round(achieved / 8000.0, 4) if achieved else None,
            "traffic": ncu_traffic("k_gemv"),
            "launch_us": round(launch_us, 3),
            "basis": "algorithmic bytes of the timed launches / timed region (CUDA events); all launches are k_gemv",
            "per_launch_group_serialised": r["per_group"],
        },
        "clocks": r["clocks"],
    }
    stack.close()
    return line


def decode_sweep(args, wl, Ms, depth, steps, warmup, local):
    """Further decode workloads measured in the same run (one GPU): the same step and timing as
    the default line, for each token count in Ms.  Returns a dict keyed by M."""
    import torch

    import weight_only_mixed_owq_b200 as owq
    dev = torch.device("cuda", local)
    peaks, kind = measured_peaks()
    stack = Stack(owq, torch, wl, depth, max(Ms), dev)
    out = {}
    for M in Ms:
        r = stack.measure(M, steps, warmup, 1, local, e2e=False)
        gbs = r["step_bytes"] * steps / (r["ms_max"] * 1e-3) / 1e9
        out[str(M)] = {"GBps": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                       "frac_of_8TBps_spec": round(gbs / 8000.0, 4),
                       "ms_per_step": round(r["ms_per_step"], 4),
                       "us_per_layer": round(r["ms_per_step"] * 1e3 / (depth * sum(len(g) for g in stack.groups)), 3),
                       "per_launch_group_serialised": r["per_group"], "clocks": r["clocks"]}
    layers = {n: [stack.info[n].N, stack.info[n].K] for n in stack.info}
    stack.close()
    torch.cuda.synchronize()
    return {"workload": f"{wl}: {depth} resident layer sets per step", "layers": layers,
            "bits": stack.spec.layers[0].bits,
            "group": "per-channel" if stack.spec.layers[0].group == stack.spec.layers[0].K else stack.spec.layers[0].group,
            "steps": steps, "warmup": warmup, "peak_hbm_gbs": peaks["hbm_gbs"], "peak_kind": kind,
            "timing": "CUDA graph of the whole step, CUDA events on the launching stream", "per_M": out}


def graph_time(calls, replays=5):
    """Device seconds per call: one CUDA graph of `calls` (zero-argument callables, one library
    call each, over distinct operand sets), 3 warm-up replays, median of `replays` timed ones."""
    import torch
    for c in calls:   # grows the handles' scratch outside the capture
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(replays):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    del g
    return statistics.median(times) * 1e-3 / len(calls)


def cold_copies(per_call_bytes, cap=64):
    """Operand sets needed so that one pass over them holds more than twice the 126 MB L2."""
    return int(max(2, min(cap, -(-2 * 126 * 2**20 // max(1, per_call_bytes)))))


def prefill_measure(args, dev, Ms=None, reps=5):
    """TFLOP/s of owq_gemm on the LLaMA-13B-shaped prefill layers (13824x5120, 5120x13824,
    3-bit, g = 128, k = 40 / 108) for the token counts of that workload (or `Ms`): one CUDA
    graph over R packed copies of the pair (more than twice the L2 in all), device time / R."""
    import torch

    import weight_only_mixed_owq_b200 as owq
    spec = owq_synth.WORKLOADS[4]
    out = {}
    peaks, kind = measured_peaks()
    pair, xs = [], []
    for li, L in enumerate(spec.layers):
        d = owq_synth.draw_layer(L, spec, max(spec.Ms), owq_synth.seed_for(4, li))
        W, X = torch.from_numpy(d["W"]).to(dev), torch.from_numpy(d["X"]).to(dev)
        pair.append((L, owq.quantize(W, X, L.bits, L.group, L.k)))
        xs.append(torch.from_numpy(d["x"]).to(dev))
        del W, X
    pair_bytes = sum(L.N * L.K * L.bits // 8 for L, _ in pair)
    R = cold_copies(pair_bytes, cap=8)
    layers = [(L, owq.OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"], q["w_weak"], L.bits, L.group), li)
              for _ in range(R) for li, (L, q) in enumerate(pair)]
    for M in (Ms or spec.Ms):
        ys = [torch.empty((M, L.N), dtype=torch.float16, device=dev) for L, _ in pair]
        xm = [x[:M].contiguous() for x in xs]
        t = graph_time([lambda lay=lay, li=li: lay.gemm(xm[li], ys[li]) for L, lay, li in layers], replays=reps)
        t_pair = t * 2   # seconds per call x two layers
        flop = sum(2.0 * M * L.N * L.K for L, _ in pair)
        tf = flop / t_pair / 1e12
        out[str(M)] = {"tflops": round(tf, 2), "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                       "us_per_pair": round(t_pair * 1e6, 2)}
    for _, lay, _ in layers:
        lay.close()
    return {"layers": "13824x5120 + 5120x13824, 3-bit g128, k=40/108", "per_M": out,
            "peak_tflops": peaks["bf16_tflops"], "peak_kind": kind, "copies": R,
            "timing": "CUDA graph over R copies of the layer pair (> 2x L2), device time per pair"}


def wct_measure(args, dev, layers=(0, 4, 5), Ms=(1, 16, 256, 2048), weak=True):
    """Weak column tuning kernels on the OPT-6.7B-shaped layers (3-bit per channel, k = K/128):
    owq_input_grad (dX = dY W_eff from the packed layout; GB/s of its algorithmic bytes: packed +
    scales/zeros + weak block + idx + dY + dX, against the HBM roofline at 1 and 16 tokens, and
    TFLOP/s of 2 M N K against the bf16 tensor roofline at 256 and 2048) and owq_weak_grad
    (dW_weak = dY^T x[:, idx]; bytes dY + the gathered x columns + fp32 dW_weak).

    Timing: one CUDA graph of R calls over R distinct operand sets (R packed copies of the layer
    for the input gradient, R (x, dY) pairs for the weak-block gradient) that together hold more
    than twice the L2, so every call reads its operands from HBM; device time of the replay / R,
    median of 5 replays after 3."""
    import torch

    import weight_only_mixed_owq_b200 as owq
    spec = owq_synth.WORKLOADS[1]
    peaks, kind = measured_peaks()

    out = {}
    for li in layers:   # 0: q (4096 x 4096), 4: fc1 (16384 x 4096), 5: fc2 (4096 x 16384)
        L = spec.layers[li]
        d = owq_synth.draw_layer(L, spec, 16, owq_synth.seed_for(1, li))
        W, X = torch.from_numpy(d["W"]).to(dev), torch.from_numpy(d["X"]).to(dev)
        q = owq.quantize(W, X, L.bits, L.group, L.k)
        del W, X
        wbytes = L.N * L.K * L.bits // 8 + L.N * (L.K // L.group) * 4 + L.N * L.k * 2 + 4 * L.k
        R = cold_copies(wbytes)
        lays = [owq.OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"], q["w_weak"], L.bits, L.group)
                for _ in range(R)]
        row = {}
        for M in Ms:
            dy = torch.randn((M, L.N), device=dev).half()
            dx = torch.empty((M, L.K), dtype=torch.float16, device=dev)
            t = graph_time([lambda lay=lay: lay.input_grad(dy, dx) for lay in lays])
            B = wbytes + 2 * M * L.N + 2 * M * L.K
            F = 2.0 * M * L.N * L.K
            row[f"input_grad_M{M}"] = {"us": round(t * 1e6, 2), "GBps": round(B / t / 1e9, 1),
                                       "frac_hbm": round(B / t / 1e9 / peaks["hbm_gbs"], 4),
                                       "TFLOPs": round(F / t / 1e12, 1),
                                       "frac_bf16": round(F / t / 1e12 / peaks["bf16_tflops"], 4), "copies": R}
        for lay in lays[1:]:
            lay.close()
        lay = lays[0]
        for M in ((16, 2048) if weak else ()):
            B = 2 * M * L.N + 2 * M * L.k + 4 * L.N * L.k
            Rw = cold_copies(2 * M * (L.N + L.K), cap=16)
            xs = [torch.randn((M, L.K), device=dev).half() for _ in range(Rw)]
            dys = [torch.randn((M, L.N), device=dev).half() for _ in range(Rw)]
            dw = torch.empty((L.N, L.k), dtype=torch.float32, device=dev)
            t = graph_time([lambda x=x, dy=dy: lay.weak_grad(x, dy, dw) for x, dy in zip(xs, dys)])
            row[f"weak_grad_M{M}"] = {"us": round(t * 1e6, 2), "GBps": round(B / t / 1e9, 1),
                                      "TFLOPs": round(2.0 * M * L.N * L.k / t / 1e12, 2), "copies": Rw}
            del xs, dys
        out[f"{L.name} {L.N}x{L.K} k={L.k}"] = row
        lay.close()
    return {"layers": out, "peak_hbm_gbs": peaks["hbm_gbs"], "peak_kind": kind,
            "timing": "CUDA graph of R calls over R operand sets holding > 2x L2; device time / R"}


# ---------------------------------------------------------------------------------- oracle arm
def oracle_sample(wl: str, rows: int):
    """Quantise (oracle) one layer set and keep the first `rows` rows of each layer."""
    import oracle
    spec = owq_synth.WORKLOADS[WID[wl]]
    out = []
    for li, L in enumerate(spec.layers):
        d = owq_synth.draw_layer(L, spec, 1, owq_synth.seed_for(spec.wid, li))
        r = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
        n = min(rows, L.N)
        packed = oracle.pack(r["codes"][:n], L.bits)
        out.append({"L": L, "n": n, "packed": packed, "scales": r["scales"][:n], "zeros": r["zeros"][:n],
                    "w_weak": r["w_weak"][:n], "idx": r["idx"], "x": d["x"]})
    return out


def oracle_step(sample) -> int:
    """One pass of the oracle's product over the sample; returns its algorithmic bytes."""
    import oracle
    b = 0
    for s in sample:
        L = s["L"]
        codes = oracle.unpack(s["packed"], L.K, L.bits)
        W_hat = oracle.dequant(codes, s["scales"], s["zeros"])
        oracle.matmul(W_hat, s["w_weak"], s["idx"], s["x"])
        b += layer_bytes(s["n"], L.K, L.bits, L.group, L.k, 1)
    return b


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl: str, budget_s: float = 12.0):
    rows = 1024
    sample = oracle_sample(wl, rows)
    t0 = time.perf_counter()
    b, n = 0, 0
    while True:
        b += oracle_step(sample)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(b / dt / 1e9, 4), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"first {rows} rows of each layer of one {wl} layer set, M=1, {n} passes, {dt:.1f} s "
                      "(unpack, dequant, fp64 product)"}


def run_reference(args):
    """The oracle (numpy, fp64) on the host cores: each step one pass over a bounded sample."""
    rows = 256
    sample = oracle_sample(args.workload, rows)
    for _ in range(args.warmup):
        oracle_step(sample)
    t0 = time.perf_counter()
    b = 0
    for _ in range(args.steps):
        b += oracle_step(sample)
    dt = time.perf_counter() - t0
    v = b / dt / 1e9
    sdesc = f"first {rows} rows of each layer of one {args.workload} layer set, M=1 (unpack, dequant, fp64 product)"
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload} (oracle sample)", "M": 1},
        "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle", "sample": sdesc},
        "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="owq", choices=["owq", "reference"])
    ap.add_argument("--workload", default="opt-6.7b-decode", choices=sorted(DEPTH))
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--depth", type=int, default=0, help="resident layer sets per step (default: model depth)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-wct", action="store_true", help="skip the weak column tuning kernels")
    ap.add_argument("--no-sweeps", action="store_true", help="skip the LLaMA-7B and OPT-66B decode lines")
    ap.add_argument("--prefill-only", default="", help="comma-separated token counts: time only owq_gemm on "
                    "the LLaMA-13B-shaped layers at those counts (3 launches each) and print that line")
    ap.add_argument("--input-grad-only", default="", help="comma-separated token counts: time only "
                    "owq_input_grad on the OPT-6.7B-shaped q layer (4096x4096, 3-bit) and print that line")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)

    rank, world, local = dist_setup()
    if args.prefill_only:
        import torch
        if rank == 0:
            Ms = [int(v) for v in args.prefill_only.split(",")]
            print(json.dumps({"prefill": prefill_measure(args, torch.device("cuda", local), Ms, reps=3)}), flush=True)
        teardown(world)
        return 0
    if args.input_grad_only:
        import torch
        if rank == 0:
            Ms = [int(v) for v in args.input_grad_only.split(",")]
            print(json.dumps({"wct": wct_measure(args, torch.device("cuda", local), layers=(0,), Ms=Ms, weak=False)}),
                  flush=True)
        teardown(world)
        return 0
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        teardown(world)
        return 0

    line = run_owq(args, rank, world, local)
    if rank == 0 and world == 1:
        import torch
        if not args.no_sweeps and args.workload == "opt-6.7b-decode":
            # the LLaMA-7B token sweep and the whole 64-layer OPT-66B set (25.5 GB resident),
            # each in the same step form as the default line
            line["llama7b"] = decode_sweep(args, "llama-7b-decode", (1, 2, 4, 8, 16), DEPTH["llama-7b-decode"],
                                           max(5, args.steps // 2), 3, local)
            line["opt66b"] = decode_sweep(args, "opt-66b-decode", (1,), DEPTH["opt-66b-decode"], 3, 3, local)
        if not args.no_prefill:
            line["prefill"] = prefill_measure(args, torch.device("cuda", local))
        if not args.no_wct:
            line["wct"] = wct_measure(args, torch.device("cuda", local))
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    teardown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
