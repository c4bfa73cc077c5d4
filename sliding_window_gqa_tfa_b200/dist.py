"""Process plumbing for running the attention on several GPUs of one node.

The work shards without any exchange (independent (batch, KV group) units;
each rank computes its own slice and writes its own output), so there is no
data-path collective: torch.distributed carries only the start barrier and
the max over ranks of the measured device time.  One process per GPU; NCCL
between GPUs, gloo when the ranks run on the CPU (the multi-process tests).
"""
from __future__ import annotations

import datetime
import os

import torch


def env_ranks():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup(backend: str | None = None, timeout_s: int = 120):
    """Join the process group when there is more than one rank.  NCCL binds this
    rank to its GPU (LOCAL_RANK); a short timeout makes ranks that wait for a
    missing peer end with an error instead of hanging."""
    world, rank, local = env_ranks()
    if world > 1:
        import torch.distributed as dist

        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def _device():
    import torch.distributed as dist

    return torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (every rank calls it, in the same order)."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def teardown(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
