"""One rank of the CPU multi-rank tests (launched by torchrun, gloo backend).

Modes:
  shard      each rank convolves its own channel shard with the oracle; rank 0
             checks the gathered result against the oracle on the whole
             problem and checks the host plumbing (max over ranks, throughput).
  peer_exit  rank 1 leaves before the barrier; rank 0's barrier must end with
             an error within the group timeout instead of waiting for good.

Each rank writes <outdir>/rank<r>.json with what it saw."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
import workloads as W  # noqa: E402
from long_sequence_fft_b200 import multigpu as mg  # noqa: E402


def _gather_np(ctx, a):
    out = [None] * ctx.world
    dist.all_gather_object(out, a)
    return out


def run_shard(ctx, outdir):
    base = W.WORKLOADS["gated_bf16_n4k"].with_shape(B=2, H=3, N=256)
    w = W.shard_of(base, ctx.rank)
    inp = W.make_all(w)
    y = oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"])
    yg = mg.gather_channels(ctx, torch.from_numpy(y)).numpy()
    parts = {t: _gather_np(ctx, inp[t]) for t in ("u", "k", "w", "v")}
    tmax = mg.max_over_ranks(ctx, 1.5 + ctx.rank)
    h0, h1 = mg.channel_range(w.H, ctx)
    mg.barrier(ctx)
    res = {"rank": ctx.rank, "world": ctx.world, "tmax": tmax, "channels": [h0, h1],
           "throughput": mg.job_throughput(w.elems, ctx, 2.0)}
    if ctx.rank == 0:
        u = np.concatenate(parts["u"], axis=1)
        k = np.concatenate(parts["k"], axis=0)
        g = np.concatenate(parts["w"], axis=1)
        v = np.concatenate(parts["v"], axis=1)
        ref = oracle.fftconv(u, k, w=g, v=v)
        res["max_err"] = float(np.max(np.abs(ref - yg)))
        res["scale"] = float(np.max(np.abs(ref)))
        res["shards_differ"] = bool(not np.array_equal(parts["u"][0], parts["u"][1]))
        res["shard0_is_workload"] = bool(np.array_equal(parts["u"][0], W.make_all(base)["u"]))
    with open(os.path.join(outdir, f"rank{ctx.rank}.json"), "w") as f:
        json.dump(res, f)
    mg.shutdown(ctx)


def run_peer_exit(ctx, outdir):
    mg.barrier(ctx)                       # both ranks are up
    res = {"rank": ctx.rank}
    if ctx.rank == 1:
        with open(os.path.join(outdir, "rank1.json"), "w") as f:
            json.dump(res, f)
        os._exit(0)                       # leaves between steps, nothing in flight
    try:
        mg.barrier(ctx)
        res["error"] = None
    except Exception as e:  # the missing peer must surface as an error
        res["error"] = type(e).__name__
    with open(os.path.join(outdir, "rank0.json"), "w") as f:
        json.dump(res, f)
    os._exit(0)


def main():
    mode, outdir = sys.argv[1], sys.argv[2]
    ctx = mg.init_from_env(backend="gloo", timeout_s=20.0)
    {"shard": run_shard, "peer_exit": run_peer_exit}[mode](ctx, outdir)


if __name__ == "__main__":
    main()
