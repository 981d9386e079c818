#!/usr/bin/env python
"""Benchmark of the MoE feed-forward layer forward pass on B200.

One step = one full forward of the layer (router scores, softmax + top-k,
histogram/scan/permutation, grouped gate/up + SiLU GEMM, grouped down GEMM,
shared SwiGLU, weighted combine) over one batch of T synthetic tokens, with
every input already resident in HBM. Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle, rank 0 only

Multi-GPU (torchrun): every rank runs an independent replica of the workload
on its own GPU (the layer has no exchange step on one node); the timed region
is bracketed by a barrier and a device synchronise, its device time is the
max over ranks, and `value` counts the tokens of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "dsv3_prefill_t4096_d7168_f2048_e256k8_s1"
METRIC = "MoE-layer tokens/s at 1 B200; TFLOP/s vs bf16 peak (HBM GB/s when weight-bound)"
L2_FLUSH_BYTES = 256 << 20          # twice the 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling runs)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override N_r (profiling runs: a small case of the same kernels)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain stream launches instead of CUDA-graph replays")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU seconds of the oracle sample")
    ap.add_argument("--per-workload", choices=["all", "none"], default="all",
                    help="also measure the other four workloads (per_workload in the line)")
    ap.add_argument("--min-seconds", type=float, default=0.25,
                    help="least device time of each per-workload timed region")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- peaks, profiles
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            m = json.load(fh)
        return {k: float(m[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the GEMM kernel's code (comments and blank lines removed, so that
    a comment-only edit keeps the committed counters valid)."""
    h = hashlib.sha256()
    for name in ("gemm_sm100.cuh", "ptx_sm100.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_ffn_expert_b200", "csrc", name),
                  encoding="utf-8") as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode("utf-8") + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, or None when there is
    none or the kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.txt")
    if not os.path.exists(path):
        return None
    text = open(path, encoding="utf-8").read()
    m_t = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    m_h = re.search(r"^kernel_source_sha256_16:\s*([0-9a-f]+)", text, re.M)
    if not m_t or not m_h or m_h.group(1) != kernel_source_hash():
        return None
    return float(m_t.group(1))


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02, probe: bool = False):
        self.idx, self.period = device_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        if probe:          # a sampler that samples nothing (untimed probe runs)
            return
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:     # CUDA and NVML number devices differently under CUDA_VISIBLE_DEVICES
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for b, name in self.REASONS.items():
            if bits & b and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml" if self.ok else "unavailable"}


# ----------------------------------------------------------------- oracle (CPU)
def oracle_experts(inp_host, shape, budget_bytes=16 << 30):
    """Expert e -> its fp64 (W1, W3, W2) for the oracle. The bf16 -> fp64 widening is
    input preparation, not the oracle's work: done once, outside any timed region,
    when all experts fit in budget_bytes (the coarse layer: 11.3 GB); otherwise per
    call, and then it is part of the timed oracle run. Returns (fn, converted_once)."""
    import torch
    keys = ("W1", "W3", "W2")
    if 8 * 3 * shape.d * shape.f * shape.n_routed <= budget_bytes:
        conv = [tuple(inp_host[k][e].to(torch.float64).numpy() for k in keys)
                for e in range(shape.n_routed)]
        return (lambda e: conv[e]), True
    return (lambda e: tuple(inp_host[k][e].to(torch.float64).numpy() for k in keys)), False


def oracle_sample_run(inp, shape, tokens, expert):
    """Run the fp64 oracle on the rows `tokens` of x; returns seconds."""
    import numpy as np
    import torch
    from oracle import moe_layer

    x = inp["x"][torch.as_tensor(tokens)].to(torch.float64).numpy()
    wg = inp["W_g"].to(torch.float64).numpy()
    bias = None if inp["bias"] is None else inp["bias"].to(torch.float64).numpy()
    shared = None
    if shape.n_shared > 0:
        shared = tuple(inp[k].to(torch.float64).numpy() for k in ("W1s", "W3s", "W2s"))
    t0 = time.perf_counter()
    r = moe_layer(x, wg, bias, expert, shared, shape.top_k, shape.renorm)
    dt = time.perf_counter() - t0
    assert np.all(np.isfinite(r["out"]))
    return dt


def host_copy_of_inputs(inp_dev):
    """bf16 host copies (D2H once, outside any timing)."""
    return {k: (None if v is None else v.cpu()) for k, v in inp_dev.items()}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def timed_oracle(inp_host, shape, target_s, expert, max_tokens=None):
    """Grow a seeded token sample until one oracle run costs about target_s."""
    import numpy as np
    rng = np.random.default_rng(0)
    T = shape.T if max_tokens is None else max_tokens
    order = rng.permutation(T)
    n = 1
    while True:
        dt = oracle_sample_run(inp_host, shape, np.sort(order[:n]), expert)
        if dt >= 0.6 * target_s or n >= T:
            return n, dt
        n = min(T, max(n + 1, int(n * min(8.0, max(2.0, target_s / max(dt, 1e-3))))))


# ----------------------------------------------------------------- arms
def run_reference(args, info):
    """The fp64 oracle as it stands, timed on this machine's host cores (rank 0 only)."""
    import torch
    from mixture_experts_ffn_expert_b200.inputs import WORKLOADS, make_layer_inputs

    if info.rank != 0:
        return None
    shape = WORKLOADS[args.workload]
    if args.tokens:
        shape = shape.with_tokens(args.tokens)
    if args.experts:
        shape = shape.with_experts(args.experts)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = host_copy_of_inputs(make_layer_inputs(shape, seed=0, device=dev))
    expert, once = oracle_experts(inp, shape)
    # size one step to about (two minutes) / (steps + warmup)
    per_step = max(0.25, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    n_tok, _ = timed_oracle(inp, shape, per_step, expert)
    import numpy as np
    rng = np.random.default_rng(1)
    for _ in range(args.warmup):
        oracle_sample_run(inp, shape, np.sort(rng.choice(shape.T, n_tok, replace=False)), expert)
    times = []
    for _ in range(args.steps):
        times.append(oracle_sample_run(inp, shape,
                                       np.sort(rng.choice(shape.T, n_tok, replace=False)), expert))
    total = sum(times)
    value = n_tok * args.steps / total
    cores = cpu_threads()
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_tok} seeded tokens of T={shape.T} per step (routing and "
                                   f"experts for those tokens only; expert weights widened to "
                                   f"fp64 {'once, outside the timing' if once else 'inside each run'}"
                                   f")"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def workload_config(shape, args):
    return {"workload": shape.name, "T": shape.T, "d": shape.d, "f": shape.f,
            "n_routed": shape.n_routed, "top_k": shape.top_k, "n_shared": shape.n_shared,
            "renorm": shape.renorm, "logit_bias": shape.bias, "seed": 0,
            "parallelism": f"replicas x{args.gpus}",
            "l2": "flushed between timed steps outside the step events (256 MiB write, "
                  "then 256 MiB read so the write's dirty lines leave L2 before the step); "
                  "weights also exceed L2"}


class L2Flush:
    """Between timed steps: a 256 MiB write, which evicts everything the step
    left in the 126 MB L2, then a 256 MiB read, so that the dirty lines of that
    write go back to HBM here, before the next step, and not during it (with the
    write alone the next step starts with ~126 MB of someone else's dirty data
    to write back: measured +6 us on the 512-expert decode step)."""

    def __init__(self, dev):
        import torch
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.sweep = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.sink = torch.empty(1, dtype=torch.int64, device=dev)

    def __call__(self):
        import torch
        self.buf.fill_(1)
        torch.sum(self.sweep, dim=0, keepdim=True, out=self.sink)


def timed_steps(step, flush, stream, steps, info, clocks):
    """Device time (ms, max over ranks) of `steps` calls of step(), L2 flushed
    between them outside the per-step events; clocks sampled meanwhile."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    from mixture_experts_ffn_expert_b200 import replicas
    replicas.barrier(info)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
        flush()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    replicas.barrier(info)
    return sum(a.elapsed_time(b) for a, b in ev), clock_info


def roofline_of(flops, nbytes, seconds, peaks, peak_src):
    """Achieved rate against the bound that limits (flops, bytes) at the measured
    peaks. A tensor fraction uses the burst bf16 peak (each timed region here is
    far shorter than the seconds-long loop the sustained figure comes from)."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    if flops and t_tensor >= t_hbm:
        ach, peak = flops / seconds / 1e12, peaks["bf16_tflops"]
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "peak_source": f"{peak_src} (bf16 burst)",
                "frac_of_sustained_peak": round(ach / peaks["bf16_tflops_sustained"], 4)}
    ach, peak = nbytes / seconds / 1e9, peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(ach, 2), "peak": peak, "unit": "GB/s",
            "frac": round(ach / peak, 4), "peak_source": f"{peak_src} (HBM copy)"}


def measure_workload(shape, args, info, dev, steps, headline):
    """One workload: warm-up, CUDA-graph capture, `steps` timed replays (None: at
    least --steps and at least --min-seconds of device time, estimated from a
    3-step run), a pass of plain launches with per-kernel events, and (headline
    only) the end-to-end leg and the oracle baseline. Returns a dict."""
    import torch
    from mixture_experts_ffn_expert_b200 import replicas
    from mixture_experts_ffn_expert_b200.inputs import make_layer_inputs
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    from mixture_experts_ffn_expert_b200.metrics import kernel_work, layer_bytes, layer_flops

    T = shape.T
    inp = make_layer_inputs(shape, seed=0, device=dev)
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device=dev)
    x = inp["x"]
    out = torch.empty_like(x)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    warm = max(args.warmup, 3)
    for _ in range(warm):
        layer(x, out)
        flush()
    torch.cuda.synchronize(dev)
    routing = layer.routing()
    counts = routing["counts"].cpu()
    touched = int((counts > 0).sum())
    launches_per_step = layer.plan.last_launch_count()

    # ---- the step: one forward, replayed from a CUDA graph (default) or launched
    graph = None
    if not args.no_graph:
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            layer(x, out)
        stream.wait_stream(cap)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            layer(x, out)
        torch.cuda.synchronize(dev)
        for _ in range(3):
            graph.replay()
            flush()
        torch.cuda.synchronize(dev)

    def step():
        if graph is not None:
            graph.replay()
        else:
            layer(x, out)

    if steps is None:
        # all ranks take the same count (the largest estimate)
        probe_ms, _ = timed_steps(step, flush, stream, 3, info, ClockSampler(-1, probe=True))
        est = replicas.max_over_ranks(probe_ms, info, device=dev) / 3 / 1e3
        steps = int(min(5000, max(args.steps, -(-args.min_seconds // max(est, 1e-6)))))

    # ---- timed region: device time of `steps` steps, max over ranks
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    local_ms, clock_info = timed_steps(step, flush, stream, steps, info, clocks)
    total_ms = replicas.max_over_ranks(local_ms, info, device=dev)
    ms_per_step = total_ms / steps
    value = info.world_size * T * steps / (total_ms / 1e3)

    # ---- per-kernel times: plain launches with events recorded around every
    #      kernel on the stream it runs on (the events between kernels break the
    #      programmatic-launch overlap, so these are shares, not absolutes)
    layer.plan.enable_timing(True)
    ktimes = {}
    names = None
    n_k = max(3, min(steps, 50))
    for i in range(n_k):
        layer(x, out)
        flush()
        if names is None:
            names = layer.plan.kernel_names()
        if i > 0:     # read the previous step while this one is queued
            for name, t in zip(names, layer.plan.kernel_times(back=1)):
                ktimes.setdefault(name, []).append(t)
    for name, t in zip(names, layer.plan.kernel_times(back=0)):
        ktimes.setdefault(name, []).append(t)
    torch.cuda.synchronize(dev)
    layer.plan.enable_timing(False)
    assert layer.device_status() == 0, "a kernel reported a bounded-wait timeout"

    # ---- rooflines: the layer as a whole, and its dominant kernel
    peaks, peak_src = load_peaks()
    kavg = {k: sum(v) / len(v) for k, v in ktimes.items()}
    ksum = sum(kavg.values())
    dominant = max(kavg, key=kavg.get)
    flops, nbytes = kernel_work(dominant, shape, T, touched)
    kroof = roofline_of(flops, nbytes, kavg[dominant] / 1e3, peaks, peak_src)
    kroof.update({"kernel": dominant, "algorithmic_flops_per_launch": flops,
                  "algorithmic_bytes_per_launch": nbytes,
                  "avg_launch_ms": round(kavg[dominant], 4),
                  "traffic": profiled_traffic(dominant.split("[")[0], shape.name)})
    lflops, lbytes = layer_flops(shape), layer_bytes(shape, touched)
    lroof = roofline_of(lflops, lbytes, ms_per_step / 1e3, peaks, peak_src)
    lroof.update({"algorithmic_flops_per_step": lflops, "algorithmic_bytes_per_step": lbytes})
    mhz = clock_info.get("sm_mhz")
    res = {
        "value": value, "ms_per_step": ms_per_step, "steps": steps,
        "tflops": lflops / (ms_per_step / 1e3) / 1e12 * info.world_size,
        "layer_roofline": lroof, "roofline": kroof, "clocks": clock_info,
        "sm_kcycles_per_step": round(ms_per_step * mhz, 1) if mhz else None,
        "gpu_launches_per_step": launches_per_step,
        "kernels_ms": {k: round(v, 4) for k, v in kavg.items()},
        "kernel_shares": {k: round(v / ksum, 4) for k, v in kavg.items()},
        "routing": {"touched_experts": touched, "max_rows": int(counts.max()),
                    "p99_rows": float(counts.float().quantile(0.99)),
                    "median_rows": float(counts.float().median()),
                    "min_rows": int(counts.min())},
        "step_launch": "cuda graph replay" if graph is not None else "stream launches",
    }

    # ---- end to end through the public API with pinned host buffers: every
    #      step copies its x in from pinned host memory and its output back out;
    #      the copies run on their own streams, double-buffered, so the copy-in
    #      of step i+1 and the copy-out of step i-1 overlap the forward of step i
    if headline and not args.no_e2e:
        n_e2e = max(3, min(steps, 50))
        x_host = [x.cpu().pin_memory() for _ in range(2)]
        out_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(x) for _ in range(2)]
        out_dev = [torch.empty_like(x) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def run_pipeline(n):
            ready = [torch.cuda.Event() for _ in range(n)]
            done = [torch.cuda.Event() for _ in range(n)]
            copied = [torch.cuda.Event() for _ in range(n)]
            with torch.cuda.stream(h2d):
                x_dev[0].copy_(x_host[0], non_blocking=True)
                ready[0].record(h2d)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    with torch.cuda.stream(h2d):
                        if i >= 1:
                            h2d.wait_event(done[i - 1])      # x_dev[(i+1)%2] free again
                        x_dev[(i + 1) % 2].copy_(x_host[(i + 1) % 2], non_blocking=True)
                        ready[i + 1].record(h2d)
                stream.wait_event(ready[i])
                if i >= 2:
                    stream.wait_event(copied[i - 2])         # out_dev[b] read out already
                layer(x_dev[b], out_dev[b])
                done[i].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(done[i])
                    out_host[b].copy_(out_dev[b], non_blocking=True)
                    copied[i].record(d2h)
            return copied[n - 1]

        run_pipeline(3)
        torch.cuda.synchronize(dev)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        replicas.barrier(info)
        torch.cuda.synchronize(dev)
        start.record(h2d)            # before the first copy-in
        stream.wait_event(start)
        last = run_pipeline(n_e2e)
        stream.wait_event(last)
        stop.record(stream)          # after the last copy-out
        torch.cuda.synchronize(dev)
        e_ms = replicas.max_over_ranks(start.elapsed_time(stop), info, device=dev)
        res["e2e"] = {"value": info.world_size * T * n_e2e / (e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": x_host[0].numel() * x_host[0].element_size(),
                      "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size(),
                      "steps": n_e2e,
                      "path": "pinned host x -> device (copy stream), moe_forward, device -> "
                              "pinned host out (copy stream); double-buffered so copies overlap "
                              "forwards; plain stream launches, no L2 flush (each step's x "
                              "arrives by copy, so it is partly L2-resident when the forward "
                              "starts, as in use)"}

    # ---- CPU baseline: the oracle on a bounded sample, rank 0 at N=1 only
    if headline and not args.no_cpu_baseline and info.rank == 0 and info.world_size == 1:
        inp_host = host_copy_of_inputs(inp)
        del inp
        expert, once = oracle_experts(inp_host, shape)
        n_tok, dt = timed_oracle(inp_host, shape, args.cpu_seconds, expert)
        res["cpu_baseline"] = {
            "value": n_tok / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n_tok} seeded tokens of T={T} (routing and experts for those "
                      f"tokens; expert weights widened to fp64 "
                      f"{'once, outside the timing' if once else 'inside the run'}), "
                      f"one run of {dt:.1f} s"}
        del inp_host
    return res


PER_WORKLOAD_KEYS = ("value", "ms_per_step", "steps", "tflops", "layer_roofline", "roofline",
                     "sm_kcycles_per_step", "gpu_launches_per_step", "kernel_shares", "routing")


def run_ours(args, info):
    import gc
    import torch
    from mixture_experts_ffn_expert_b200.inputs import WORKLOADS

    dev = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(dev)
    shape = WORKLOADS[args.workload]
    if args.tokens:
        shape = shape.with_tokens(args.tokens)
    if args.experts:
        shape = shape.with_experts(args.experts)

    head = measure_workload(shape, args, info, dev, args.steps, headline=True)
    per = {}
    if args.per_workload == "all":
        per[shape.name] = {k: head[k] for k in PER_WORKLOAD_KEYS}
        per[shape.name]["clocks"] = head["clocks"]
        for name, other in WORKLOADS.items():
            if name == shape.name:
                continue
            gc.collect()
            torch.cuda.empty_cache()
            r = measure_workload(other, args, info, dev, None, headline=False)
            per[name] = {k: r[k] for k in PER_WORKLOAD_KEYS}
            per[name]["clocks"] = r["clocks"]
            per[name]["config"] = workload_config(other, args)
            del r
    gc.collect()
    torch.cuda.empty_cache()

    out = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s",
        "n_gpus": info.world_size, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init weights scaled 1/sqrt(fan_in))",
        "config": workload_config(shape, args),
        "tflops": head["tflops"], "roofline": head["roofline"],
        "layer_roofline": head["layer_roofline"],
        "cpu_baseline": head.get("cpu_baseline"), "e2e": head.get("e2e"),
        "gpu_launches": head["gpu_launches_per_step"] * args.steps,
        "step_launch": head["step_launch"],
        "clocks": head["clocks"], "sm_kcycles_per_step": head["sm_kcycles_per_step"],
        "kernels_ms": head["kernels_ms"],
        "kernels_ms_basis": "plain stream launches with CUDA events around each kernel on its "
                            "own stream, after the timed region; the events break the "
                            "programmatic-launch overlap, so use them as shares only",
        "kernel_shares": head["kernel_shares"],
        "routing": head["routing"],
    }
    if per:
        out["per_workload"] = per
        out["per_workload_basis"] = (
            "every workload of the layer's five configurations, measured the same way as the "
            "headline (CUDA-graph replays, L2 flushed between steps, device time); steps per "
            "workload >= --steps and >= --min-seconds of device time; layer_roofline = the "
            "layer's algorithmic FLOPs or bytes per step / ms_per_step against the measured "
            "bf16 burst peak or HBM copy bandwidth, whichever bounds the layer; "
            "sm_kcycles_per_step = ms_per_step x median SM MHz (compare across clock states)")
    return out


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    from mixture_experts_ffn_expert_b200 import replicas
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        info = replicas.RankInfo(0, 1, 0, False)
        res = run_reference(args, info)
    else:
        info = replicas.init_from_env("nccl")
        try:
            res = run_ours(args, info)
        finally:
            replicas.shutdown(info)
    if res is not None and info.rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
