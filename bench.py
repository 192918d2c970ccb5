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
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "FFT-conv B*H*N elems/s and achieved % of roofline (1xB200)"
UNIT = "elems/s"


def algorithmic_bytes(w: W.Workload) -> int:
    """Compulsory HBM bytes of one forward call: read u (and w, v), write y,
    read the filter spectrum once (N+1 complex fp32 bins per channel)."""
    esz = 4 if w.dtype == "f32" else 2
    per_elem = 2 * esz + (2 * esz if w.gated else 0)
    bins = (w.L + 1) if w.L < w.N else (w.N + 1)
    if w.sparsity > 0:
        bins = int(round((1 - w.sparsity) * (w.N + 1)))
    return w.elems * per_elem + w.H * bins * 8


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
    """nvidia-smi clocks/throttle reasons sampled every 20 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()
        return False

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, smmax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smmax = max(smmax, float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() in ("active", "1"):
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smmax, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- oracle ---

def time_oracle(w: W.Workload, target_s: float = 10.0):
    """The fp64 oracle on a bounded sample of the workload: a block of whole
    sequences (b, h) of the workload's shape, convolved repeatedly on all host
    cores until about `target_s` seconds have passed.  Returns (elems/s,
    cores, description)."""
    import oracle
    cores = os.cpu_count() or 1
    sub = w.with_shape(B=min(w.B, 16), H=min(w.H, 64))
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

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=W.BENCH_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--order", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--B", type=int, default=None,
                    help="override the batch size (small cases for profiling; not a bench number)")
    ap.add_argument("--profile", action="store_true",
                    help="profiling run: skip the host-buffer and CPU-baseline legs")
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

    y = torch.empty_like(u)
    for _ in range(args.warmup):
        plan.forward(u, Kf, w=g, v=v, mask=mask, out=y)
    torch.cuda.synchronize()
    assert plan.device_status() == 0

    # timed region: K forward calls, barrier + synchronize on both sides
    mg.barrier(ctx)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for _ in range(args.steps):
            plan.forward(u, Kf, w=g, v=v, mask=mask, out=y)
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
    # the timed region)
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
    del staging, uh, gh, vh, yh

    hbm_peak, tc_peak, peak_kind = read_peaks()
    abytes = algorithmic_bytes(w)
    achieved = abytes / (ms_per_step * 1e-3) / 1e9          # per launch-group (one forward)
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
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "traffic": None if traffic is None else traffic.get("bytes_per_launch"),
                     "algorithmic_bytes": abytes,
                     "kernel": kernel_key},
        "e2e": {"value": mg.job_throughput(w.elems, ctx, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "filter_precompute_ms": precompute_ms,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, cores, sample = time_oracle(w)
        line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    mg.shutdown(ctx)
    return 0


if __name__ == "__main__":
    sys.exit(main())
