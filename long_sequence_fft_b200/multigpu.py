"""One process per GPU, channels sharded across ranks.

Every (batch row, channel) sequence of the convolution is independent: each
output row depends only on its own input row and its channel's filter (the
definition of the long convolution in "FlashFFTConv: Efficient Convolutions
for Long Sequences with Tensor Cores", summary paragraph), so a job of R ranks
splits the channel axis: rank r owns channels [r*H, (r+1)*H), holds
only their filter spectra, and convolves its own inputs with no exchange on the
data path.  The only collectives are the host plumbing around a timed region
(a barrier and a max over ranks of the elapsed time) and an optional all-gather
of the output for callers that want the whole tensor on every rank.

Launch: ``torchrun --nproc-per-node R --master-addr 127.0.0.1 ...``; each
process reads RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the environment.
NCCL runs on GPUs; gloo serves the same calls on CPU (the multi-rank tests).
"""
from __future__ import annotations

import dataclasses
import datetime
import os
from typing import Optional


@dataclasses.dataclass(frozen=True)
class RankContext:
    world: int
    rank: int
    local_rank: int
    backend: Optional[str]      # None for a single process without a group
    device: str                 # where collective buffers live: "cuda" or "cpu"


def init_from_env(backend: Optional[str] = None, timeout_s: float = 120.0) -> RankContext:
    """Join the process group described by the torchrun environment.

    With WORLD_SIZE unset or 1 no group is created.  `backend` defaults to
    "nccl" when CUDA is available, else "gloo".  A short timeout makes ranks
    that wait on a missing peer fail with an error instead of hanging."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    device = "cuda" if backend == "nccl" else "cpu"
    if device == "cuda":
        torch.cuda.set_device(local)
    if world == 1:
        return RankContext(1, 0, local, None, device)
    import torch.distributed as dist
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return RankContext(world, rank, local, backend, device)


def shutdown(ctx: RankContext) -> None:
    if ctx.backend is not None:
        import torch.distributed as dist
        dist.destroy_process_group()


def barrier(ctx: RankContext) -> None:
    if ctx.backend is not None:
        import torch.distributed as dist
        if ctx.backend == "nccl":
            dist.barrier(device_ids=[ctx.local_rank])
        else:
            dist.barrier()


def max_over_ranks(ctx: RankContext, x: float) -> float:
    """The largest `x` over all ranks (the job's time is its slowest rank's)."""
    if ctx.backend is None:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=ctx.device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def channel_range(H_shard: int, ctx: RankContext) -> tuple:
    """Global channel ids [h0, h1) that this rank owns."""
    return ctx.rank * H_shard, (ctx.rank + 1) * H_shard


def job_throughput(elems_per_rank: int, ctx: RankContext, ms_per_step: float) -> float:
    """Whole-job elements per second: every rank's elements over the slowest
    rank's time per step (weak scaling: the per-rank work is fixed)."""
    if ms_per_step <= 0:
        raise ValueError(ms_per_step)
    return ctx.world * elems_per_rank / (ms_per_step * 1e-3)


def gather_channels(ctx: RankContext, y):
    """All-gather the per-rank outputs [B, H, N] into [B, R*H, N] on every rank
    (channel order = rank order).  Not on the hot path: for callers that want
    the whole output in one place."""
    if ctx.backend is None:
        return y
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(y) for _ in range(ctx.world)]
    dist.all_gather(parts, y.contiguous())
    return torch.cat(parts, dim=1)
