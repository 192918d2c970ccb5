"""Benchmark: causal long convolution (FFT conv) throughput on B200.

One step = one forward call of the whole hot path (gating prologue, forward
transform, product with the precomputed filter spectrum, inverse transform,
gating epilogue) over one batch of the gated bf16 workload B=64, H=768,
N=4096 (FFT size 8192); the filter transform is precomputed once, off the
per-call path, and timed separately.  Metric: B*H*N output elements per second
(higher is better), with the achieved fraction of the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): every rank convolves its own shard of
channels of the same size (weak scaling, no collective on the data path);
timing is the max over ranks of the device-timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "FFT-conv B*H*N elems/s and achieved % of roofline (1xB200)"
UNIT = "elems/s"


TC_PATHS = ("tc_fused", "tc_staged")


def kf_bytes_per_bin(path: str) -> int:
    """Stored width of one filter-spectrum bin: complex fp16 (4 B) on the
    tensor-core paths, complex fp32 (8 B) on the fp32-lane paths."""
    return 4 if path in TC_PATHS else 8


def algorithmic_bytes(w: W.Workload, path: str = "simt_fused") -> int:
    """Compulsory HBM bytes of one forward call: read u (and w, v), write y,
    read the filter spectrum once at its stored width (N+1 bins per channel;
    L+1 for a partial filter; the kept bins for a block-sparse one)."""
    esz = 4 if w.dtype == "f32" else 2
    per_elem = 2 * esz + (2 * esz if w.gated else 0)
    bins = (w.L + 1) if w.L < w.N else (w.N + 1)
    if w.monarch_keep:
        bins = int(round(W.monarch_kept_fraction(w) * (w.N + 1)))
    elif w.sparsity > 0:
        bins = int(round((1 - w.sparsity) * (w.N + 1)))
    return w.elems * per_elem + w.H * bins * kf_bytes_per_bin(path)


def backward_bytes(w: W.Workload, path: str) -> int:
    """Compulsory HBM bytes of one backward call (fftconv_backward): read u,
    dy (and w, v), write du (and dw, dv), read the filter spectrum once at
    its stored width and write the fp32 filter gradient dk [H, L]."""
    esz = 4 if w.dtype == "f32" else 2
    per_elem = 3 * esz + (4 * esz if w.gated else 0)
    bins = (w.L + 1) if w.L < w.N else (w.N + 1)
    return w.elems * per_elem + w.H * bins * kf_bytes_per_bin(path) + w.H * w.L * 4


def mma_flops_per_elem(w: W.Workload, path: str):
    """(schedule, flops per output element) of the tensor-core contractions the
    path issues, counted from the instruction shapes (complex values as real
    pairs: 2 flops per real multiply-add).  The 8192-point engine is
    32 x 32 x 8.  A zero-padded transform of 4096 inputs whose first 4096
    outputs are kept (N = 4096, each overlap-save window, and a row of
    4096/N packed shorter sequences, each in a zero-padded slot of 2N points)
    issues 8*32 + 16*(32 + 8) = 896 per point of its window (also each block
    of 4096 of the N = 8192 two-block mode); a transform of all 8192 inputs
    and outputs (the N = 8192 parity split of masked calls, the staged row
    pass) 16*(32 + 32 + 8) = 1152 per point.  fp32-lane paths issue none."""
    if path == "tc_fused":
        if w.N == 4096 and w.monarch_keep:
            return "32x32x8, Monarch-masked c2 skipped", monarch_mma_flops_per_elem(w.monarch_keep)
        if w.N == 4096:
            return "32x32x8", 896.0
        if w.N < 4096:
            return "32x32x8 (%d packed per row)" % (4096 // w.N), 896.0
        if w.N == 8192:
            if w.sparsity > 0:
                return "32x32x8 (x2 parity halves)", 1152.0
            return "32x32x8 (two blocks of 4096)", 896.0
        if w.N == 16384:
            return "32x32x8 (four blocks of 4096)", 896.0
        nwin = w.N // 2048 - 1
        return "32x32x8 windows", 896.0 * nwin * 4096 / w.N
    if path == "tc_staged":
        return "columns on fp32 lanes x rows 32x32x8", 1152.0
    return "fp32 lanes", 0.0


def monarch_mma_flops_per_elem(keep: int) -> float:
    """Issued MMA flops per output of the N = 4096 kernel with a
    Monarch-aligned mask, from the instructions it issues per tile (M = 128,
    2 flops per multiply-add; a tile is 32768 outputs): S1 16 of 128x64x16,
    S2 32 of 128x64x16, S3 and S3' one 128x16x16 per kept c2 and j3 pair
    (8 each per c2 over the tile), S2' 8 per K step of eight c2 with any kept,
    S1' 32 of 128x32x16.  keep = all ones gives 896."""
    big, small, s1i = 2 * 128 * 64 * 16, 2 * 128 * 16 * 16, 2 * 128 * 32 * 16
    kept = bin(keep & 0xFFFFFFFF).count("1")
    ksteps = sum(1 for s in range(4) if (keep >> (8 * s)) & 0xFF)
    per_tile = (16 + 32) * big + 2 * kept * small + 8 * ksteps * big + 32 * s1i
    return per_tile / 32768.0


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1607.7)), "measured"
    return 6650.0, 1590.0, "fallback"


def read_traffic(kernel_key: str):
    """DRAM bytes per launch of the workload's dominant kernel from a committed
    ncu capture, or None.  The entry names the kernel's source file and its
    SHA-256 at capture time; a kernel changed since then reads as None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent:
        return None
    import hashlib
    src = os.path.join(ROOT, ent.get("source", ""))
    if not os.path.isfile(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != ent.get("source_sha256"):
            return None
    return ent


class ClockSampler:
    """SM clock, power and clock-event reasons of the benchmark's GPU, sampled
    through NVML every `interval` seconds on a background thread while the
    timed region runs (the timed work runs in ctypes calls and CUDA
    synchronisation, which release the interpreter lock)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, torch_device: int, interval: float = 0.001):
        self.dev = torch_device
        self.interval = interval
        self.samples = []
        self.max_mhz = None
        self.thread = None
        self.error = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        try:
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self, h, stop):
        import pynvml
        while not stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((sm, rs, pw))
            except Exception as e:  # pragma: no cover - driver-side failure
                self.error = repr(e)
                return
            stop.wait(self.interval)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._run, args=(h, self.stop), daemon=True)
            self.thread.start()
        except Exception as e:
            self.error = repr(e)
            self.thread = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        return False

    def summary(self):
        if not self.samples:
            return None if self.error is None else {"error": self.error}
        reasons = set()
        for _, rs, _ in self.samples:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[0] for x in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "power_w_max": max(x[2] for x in self.samples), "source": "nvml"}


# --------------------------------------------------------------- oracle ---

def time_oracle(w: W.Workload, target_s: float = 10.0, cores: int = 0, H: int = 64):
    """The fp64 oracle on a bounded sample of the workload: a block of whole
    sequences (b, h) of the workload's shape, convolved repeatedly on `cores`
    host threads (0: all) until about `target_s` seconds have passed.  Returns
    (elems/s, threads, description)."""
    import oracle
    cores = cores or (os.cpu_count() or 1)
    sub = w.with_shape(B=min(w.B, 16), H=min(w.H, H))
    inp = W.make_all(sub)
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"], mask=inp["mask"], nthreads=cores)
        done += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    elems = done * sub.elems
    return elems / dt, cores, (f"{done} passes over {sub.B * sub.H} whole sequences (B={sub.B}, H={sub.H}) of "
                               f"N={w.N}: {done * sub.B * sub.H} sequences in {dt:.1f} s on {cores} threads")


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.WORKLOADS[W.BENCH_WORKLOAD]
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    # each step: a bounded sample of the workload (whole sequences)
    sub = w.with_shape(B=1, H=32)
    inp = W.make_all(sub)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"], mask=inp["mask"], nthreads=cores)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    tstep = statistics.median(times)
    value = sub.elems / tstep
    sample = f"{sub.B * sub.H} whole sequences of N={w.N} per step (fp64 oracle, {cores} threads)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tstep * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "gated": w.gated, "io_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- main ---

# Workloads timed beside the headline (one GPU): every other configuration
# of the hot path, each for at least about a second of steps.
# backward passes timed beside the forward workloads (the workload's shape)
BACKWARD_WORKLOADS = ("gated_bf16_n4k", "partial_bf16_n8k")
SIDE_WORKLOADS = ("fp32_n1k", "fp16_n16k", "fp16_n32k", "dna_bf16_n1m", "partial_bf16_n8k", "sparse_bf16_n8k",
                  "monarch_bf16_n4k", "gated_bf16_n1k", "bf16_n1k", "dna_bf16_n4m_l1m")


def roofline_entry(w: W.Workload, path: str, ms_per_step: float, hbm_peak: float, tc_peak: float):
    """Roofline of one workload: T_roof = max(compulsory bytes at the measured
    HBM bandwidth, issued MMA flops at the measured dense bf16/fp16 peak);
    frac = T_roof / T_measured, and the HBM-only fraction beside it."""
    abytes = algorithmic_bytes(w, path)
    sched, fpe = mma_flops_per_elem(w, path)
    t_hbm = abytes / (hbm_peak * 1e9)
    t_mma = fpe * w.elems / (tc_peak * 1e12)
    t = ms_per_step * 1e-3
    return {"algorithmic_bytes": abytes, "achieved_gbs": abytes / t / 1e9, "hbm_frac": t_hbm / t,
            "mma_schedule": sched, "mma_flops_per_elem": fpe, "t_hbm_us": t_hbm * 1e6, "t_mma_us": t_mma * 1e6,
            "frac": max(t_hbm, t_mma) / t, "bound": "hbm" if t_hbm >= t_mma else "tensor"}


def time_in_graph(call, stream, calls: int = 100, replays: int = 50):
    """Per-call device time of `call` replayed from a CUDA graph of `calls`
    captured calls (after one warm-up replay); {"error": ...} when capture
    fails, so the eager number stands alone."""
    import torch
    try:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            call()                              # warm-up on the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(calls):
                call()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / (calls * replays)
        del graph
        return {"ms_per_call": ms, "calls_per_graph": calls, "replays": replays}
    except Exception as exc:                    # capture is an extra view, never fatal
        torch.cuda.synchronize()
        return {"error": f"{type(exc).__name__}: {exc}"[:200]}


def time_side_workload(name: str, hbm_peak: float, tc_peak: float, min_seconds: float = 1.0):
    """One configuration end to end on the device: seeded inputs copied to HBM,
    plan, filter precompute, 3 warm-up calls, then enough calls for about
    `min_seconds`, timed with CUDA events on the launching stream while NVML
    samples the clocks."""
    import torch
    import long_sequence_fft_b200 as lsf
    w = W.WORKLOADS[name]
    inp = W.make_all(w)
    dt = W.torch_dtype(w.dtype)
    dev = lambda a: None if a is None else torch.from_numpy(a).to(dt).cuda()
    u, k, g, v = dev(inp["u"]), dev(inp["k"]), dev(inp["w"]), dev(inp["v"])
    del inp["u"], inp["w"], inp["v"]
    mask = torch.from_numpy(inp["mask"]).cuda() if inp["mask"] is not None else None
    plan = lsf.Plan(w.N, w.H, w.dtype, L=w.L)
    Kf = plan.precompute(k)
    y = torch.empty_like(u)
    stream = torch.cuda.current_stream()
    if w.monarch_keep:
        fwd = lambda: plan.forward_monarch(u, Kf, w.monarch_keep, w=g, v=v, out=y)
    else:
        fwd = lambda: plan.forward(u, Kf, w=g, v=v, mask=mask, out=y)
    for _ in range(3):
        fwd()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    fwd()
    e1.record(stream)
    torch.cuda.synchronize()
    steps = int(min(20000, max(10, min_seconds / max(e0.elapsed_time(e1) * 1e-3, 1e-6))))
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(steps):
            fwd()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    graph = None
    if ms < 0.05:
        graph = time_in_graph(fwd, stream)
    status = plan.device_status()
    entry = {"B": w.B, "H": w.H, "N": w.N, "L": w.L, "gated": w.gated, "io_dtype": w.dtype,
             "sparsity": (1.0 - W.monarch_kept_fraction(w)) if w.monarch_keep else w.sparsity,
             "monarch_keep_c2": ("0x%08X" % w.monarch_keep) if w.monarch_keep else None,
             "path": plan.path_name, "steps": steps, "ms_per_step": ms,
             "value": w.elems / (ms * 1e-3), "unit": UNIT, "device_status": status,
             "clocks": clk.summary()}
    entry.update(roofline_entry(w, plan.path_name, ms, hbm_peak, tc_peak))
    if graph is not None:
        # launch-bound calls: the same calls replayed from a CUDA graph, which
        # removes the per-call host work (argument checks, ctypes, launch)
        if "ms_per_call" in graph:
            graph["value"] = w.elems / (graph["ms_per_call"] * 1e-3)
            graph["unit"] = UNIT
        entry["graph"] = graph
    del u, k, g, v, y, Kf, plan
    torch.cuda.empty_cache()
    return entry


def time_backward(name: str, hbm_peak: float, tc_peak: float, min_seconds: float = 1.0):
    """fftconv_backward on a workload's shape and seeded inputs (dy from its
    own stream): du, dw, dv on the tensor cores (the forward kernel with dy as
    output gate, then one correlation launch) and dk on fp32 lanes.  Timed
    like the forward workloads: 3 warm-up calls, then about `min_seconds` of
    calls into preallocated gradients, CUDA events on the launching stream."""
    import torch
    import long_sequence_fft_b200 as lsf
    w = W.WORKLOADS[name]
    inp = W.make_all(w)
    dt = W.torch_dtype(w.dtype)
    dev = lambda a: None if a is None else torch.from_numpy(a).to(dt).cuda()
    u, k, g, v = dev(inp["u"]), dev(inp["k"]), dev(inp["w"]), dev(inp["v"])
    dy = dev(W.make_grad_output(w))
    del inp
    plan = lsf.Plan(w.N, w.H, w.dtype, L=w.L)
    Kf = plan.precompute(k)
    out = plan.backward(u, Kf, dy, w=g, v=v)
    bwd = lambda: plan.backward(u, Kf, dy, w=g, v=v, out=out)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        bwd()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    bwd()
    e1.record(stream)
    torch.cuda.synchronize()
    steps = int(min(20000, max(10, min_seconds / max(e0.elapsed_time(e1) * 1e-3, 1e-6))))
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(steps):
            bwd()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    path = plan.path_name
    abytes = backward_bytes(w, path)
    fpe = 2 * mma_flops_per_elem(w, path)[1]          # the dv forward and the du/dw correlation
    t_hbm = abytes / (hbm_peak * 1e9)
    t_mma = fpe * w.elems / (tc_peak * 1e12)
    t = ms * 1e-3
    entry = {"pass": "backward (du, dw, dv, dk)", "B": w.B, "H": w.H, "N": w.N, "L": w.L, "gated": w.gated,
             "io_dtype": w.dtype, "path": path, "steps": steps, "ms_per_step": ms,
             "value": w.elems / t, "unit": UNIT, "device_status": plan.device_status(), "clocks": clk.summary(),
             "algorithmic_bytes": abytes, "achieved_gbs": abytes / t / 1e9, "hbm_frac": t_hbm / t,
             "mma_flops_per_elem": fpe, "t_hbm_us": t_hbm * 1e6, "t_mma_us": t_mma * 1e6,
             "frac": max(t_hbm, t_mma) / t, "bound": "hbm" if t_hbm >= t_mma else "tensor"}
    del u, k, g, v, dy, out, Kf, plan
    torch.cuda.empty_cache()
    return entry


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=W.BENCH_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--order", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip timing the other configurations beside the headline")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--B", type=int, default=None,
                    help="override the batch size (small cases for profiling; not a bench number)")
    ap.add_argument("--profile", action="store_true",
                    help="profiling run: skip the host-buffer, CPU-baseline and side-workload legs")
    ap.add_argument("--backward", action="store_true",
                    help="with --profile: run the backward pass (fftconv_backward) instead of the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import long_sequence_fft_b200 as lsf

    from long_sequence_fft_b200 import multigpu as mg
    ctx = mg.init_from_env()
    world, rank = ctx.world, ctx.rank
    w = W.WORKLOADS[args.workload]
    if args.B is not None:
        w = w.with_shape(B=args.B)
    w = W.shard_of(w, rank)                  # this rank's channel shard
    if w.B * w.H * w.N == 0:
        raise SystemExit("empty workload")

    # inputs: seeded host generation, copied to HBM once (each rank convolves
    # its own channel shard, drawn from its own seeded streams; all shards
    # have the workload's shape)
    inp = W.make_all(w)
    dt = W.torch_dtype(w.dtype)
    dev = lambda a: None if a is None else torch.from_numpy(a).to(dt).cuda()
    u, k, g, v = dev(inp["u"]), dev(inp["k"]), dev(inp["w"]), dev(inp["v"])
    mask = torch.from_numpy(inp["mask"]).cuda() if inp["mask"] is not None else None
    plan = lsf.Plan(w.N, w.H, w.dtype, order=args.order, L=w.L)
    stream = torch.cuda.current_stream()
    Kf = plan.new_filter()

    # filter precompute (once per filter), timed on its own
    for _ in range(2):
        plan.precompute(k, out=Kf)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    plan.precompute(k, out=Kf)
    e1.record(stream)
    torch.cuda.synchronize()
    precompute_ms = e0.elapsed_time(e1)

    if args.backward:
        # profiling run of the backward pass alone (the bench line times it in
        # its workloads object)
        if not args.profile:
            raise SystemExit("--backward is a profiling run: add --profile")
        dy = dev(W.make_grad_output(w))
        grads = plan.backward(u, Kf, dy, w=g, v=v)
        for _ in range(args.warmup):
            plan.backward(u, Kf, dy, w=g, v=v, out=grads)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            plan.backward(u, Kf, dy, w=g, v=v, out=grads)
        e1.record(stream)
        torch.cuda.synchronize()
        if plan.device_status() != 0:
            raise SystemExit("device status after the backward passes")
        if rank == 0:
            print(json.dumps({"profile_run": True, "pass": "backward", "workload": w.name, "B": w.B,
                              "ms_per_step": e0.elapsed_time(e1) / args.steps, "path": plan.path_name}), flush=True)
        mg.shutdown(ctx)
        return 0

    y = torch.empty_like(u)
    if w.monarch_keep:
        fwd = lambda: plan.forward_monarch(u, Kf, w.monarch_keep, w=g, v=v, out=y)
    else:
        fwd = lambda: plan.forward(u, Kf, w=g, v=v, mask=mask, out=y)
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    assert plan.device_status() == 0

    # timed region: K forward calls, barrier + synchronize on both sides
    mg.barrier(ctx)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for _ in range(args.steps):
            fwd()
        stop.record(stream)
        torch.cuda.synchronize()
    mg.barrier(ctx)
    ms_local = start.elapsed_time(stop)
    ms = mg.max_over_ranks(ctx, ms_local)
    status = plan.device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the timed region")
    ms_per_step = ms / args.steps
    value = mg.job_throughput(w.elems, ctx, ms_per_step)

    launches_per_step = 1
    if plan.path in (lsf.PATH_SIMT_STAGED, lsf.PATH_TC_STAGED):
        # column pass, row pass, inverse column pass per workspace chunk
        # (fp32 workspace: 2N x 8 bytes per pair; fp16 on the tensor-core path)
        per_pair = 2 * w.N * (8 if plan.path == lsf.PATH_SIMT_STAGED else 4)
        chunk = max(1, plan.workspace_bytes // per_pair)
        pairs = w.H * ((w.B + 1) // 2)
        launches_per_step = 3 * ((pairs + chunk - 1) // chunk)

    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": ms_per_step, "workload": w.name, "B": w.B,
                              "path": plan.path_name}), flush=True)
        mg.shutdown(ctx)
        return 0

    # end to end through the host-buffer entry point (pinned memory, copies in
    # the timed region); that entry point takes block masks, not Monarch keep
    # sets, so a Monarch-masked headline has no end-to-end leg
    if w.monarch_keep:
        raise SystemExit("monarch_bf16_n4k is timed beside the headline (the host-buffer entry point "
                         "has no Monarch-mask form); use --profile to time it alone")
    pin = lambda a: None if a is None else torch.from_numpy(a).to(dt).pin_memory()
    uh, gh, vh = pin(inp["u"]), pin(inp["w"]), pin(inp["v"])
    mh = torch.from_numpy(inp["mask"]).pin_memory() if inp["mask"] is not None else None
    yh = torch.empty(u.shape, dtype=dt).pin_memory()
    staging = torch.empty(plan.staging_bytes(w.B, g is not None, v is not None, 0 if mh is None else mh.shape[0]),
                          dtype=torch.uint8, device="cuda")
    plan.forward_host(uh, Kf, yh, staging, w_host=gh, v_host=vh, mask_host=mh)
    torch.cuda.synchronize()
    mg.barrier(ctx)
    s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for _ in range(args.e2e_steps):
        plan.forward_host(uh, Kf, yh, staging, w_host=gh, v_host=vh, mask_host=mh)
    t2.record(stream)
    torch.cuda.synchronize()
    e2e_ms = mg.max_over_ranks(ctx, s2.elapsed_time(t2)) / args.e2e_steps
    esz = uh.element_size()
    h2d = w.elems * esz * (1 + (gh is not None) + (vh is not None)) + (0 if mh is None else mh.numel())
    d2h = w.elems * esz
    del staging, uh, gh, vh, yh, inp

    hbm_peak, tc_peak, peak_kind = read_peaks()
    roof = roofline_entry(w, plan.path_name, ms_per_step, hbm_peak, tc_peak)
    kernel_key = f"{w.name}:{plan.path_name}"
    traffic = read_traffic(kernel_key)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        # arithmetic of the path: fp16 tensor-core operands (fp32 accumulate);
        # the tensor-core staged path runs its column passes in fp32
        "dtype": "f16" if plan.path in (lsf.PATH_TC_FUSED, lsf.PATH_TC_STAGED) else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "L": w.L, "gated": w.gated,
                   "io_dtype": w.dtype, "path": plan.path_name, "parallelism": f"channel shards x{world}",
                   "l2": "inputs exceed L2 (1.2 GB resident), no flush"},
        "roofline": {"bound": "hbm", "achieved": roof["achieved_gbs"], "peak": hbm_peak, "unit": "GB/s",
                     "frac": roof["hbm_frac"], "peak_kind": peak_kind,
                     "traffic": None if traffic is None else traffic.get("bytes_per_launch"),
                     "algorithmic_bytes": roof["algorithmic_bytes"], "kernel": kernel_key,
                     "mma_schedule": roof["mma_schedule"], "mma_flops_per_elem": roof["mma_flops_per_elem"],
                     "mma_peak_tflops": tc_peak, "t_hbm_us": roof["t_hbm_us"], "t_mma_us": roof["t_mma_us"],
                     "frac_max_of_hbm_and_mma": roof["frac"]},
        "e2e": {"value": mg.job_throughput(w.elems, ctx, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "filter_precompute_ms": precompute_ms,
        "clocks": clk.summary(),
    }
    del u, k, g, v, y, Kf, plan, mask
    torch.cuda.empty_cache()
    if world == 1 and not args.no_workloads:
        line["workloads"] = {name: time_side_workload(name, hbm_peak, tc_peak) for name in SIDE_WORKLOADS
                             if name != w.name}
        for name in BACKWARD_WORKLOADS:
            line["workloads"]["backward_" + name] = time_backward(name, hbm_peak, tc_peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, cores, sample = time_oracle(w)
        v_one, _, sample_one = time_oracle(w, target_s=8.0, cores=1, H=4)
        line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                                "single_core": {"value": v_one, "unit": UNIT, "cores": 1, "sample": sample_one}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    mg.shutdown(ctx)
    return 0


if __name__ == "__main__":
    sys.exit(main())
