"""Running one attention call on several GPUs of one node.

The call shards without any exchange.  Its units are the (batch b, KV group g)
pairs: under the grouped-query mapping of tiny-llm "Week 2 Day 5: Tiled Dense
Prefill Attention", Task 1 (query head h reads KV head floor(h / G)), unit
(b, g) is the G query heads g G .. g G + G - 1 of element b with KV head g,
and nothing outside it.  Units are numbered b-major (u = b Hkv + g); rank r
takes the contiguous range [r U / N, (r + 1) U / N) of the U = B Hkv units.  In
the [B, H, len, D] layouts a contiguous unit range is a contiguous range of
query planes and of KV planes, so a rank's share splits into at most three
runs that are each one ordinary call on slices of the tensors (a tail of
groups of one element, whole elements, a head of groups of one element).
Each rank writes only its own rows of O; all_gather_output assembles the
whole O on every rank when a caller wants it (the one collective, optional).
torch.distributed otherwise carries only the start barrier and the max over
ranks of the measured device time.  One process per GPU; NCCL between GPUs,
gloo when the ranks run on the CPU (the multi-process tests).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

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


# ------------------------------------------------------------- sharding a call
@dataclass(frozen=True)
class Run:
    """Units [b0 Hkv + g0, ...) of one rank that are one call: elements b0 ..
    b0 + nb - 1, KV groups g0 .. g0 + ng - 1 of each (ng < Hkv only when nb = 1)."""
    b0: int
    nb: int
    g0: int
    ng: int


def unit_range(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """Rank `rank`'s contiguous share [u0, u1) of n_units, sizes differing by one at most."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    return (n_units * rank) // world, (n_units * (rank + 1)) // world


def unit_runs(u0: int, u1: int, Hkv: int) -> list[Run]:
    """Split units [u0, u1) (u = b Hkv + g) into runs that are each a contiguous
    block of the [B, H, len, D] tensors and one call of the library."""
    runs = []
    u = u0
    while u < u1:
        b, g = divmod(u, Hkv)
        if g > 0 or u1 - u < Hkv:  # part of one element
            ng = min(Hkv - g, u1 - u)
            runs.append(Run(b, 1, g, ng))
            u += ng
        else:  # whole elements
            nb = (u1 - u) // Hkv
            runs.append(Run(b, nb, 0, Hkv))
            u += nb * Hkv
    return runs


def rank_runs(B: int, Hkv: int, world: int, rank: int) -> list[Run]:
    """The runs rank `rank` computes when a call's B Hkv units are shared by `world` ranks."""
    return unit_runs(*unit_range(B * Hkv, world, rank), Hkv)


def run_slices(run: Run, G: int):
    """(query-plane slice over [B, Hq], KV-plane slice over [B, Hkv]) of a run, as
    (element slice, head slice) pairs."""
    return ((slice(run.b0, run.b0 + run.nb), slice(run.g0 * G, (run.g0 + run.ng) * G)),
            (slice(run.b0, run.b0 + run.nb), slice(run.g0, run.g0 + run.ng)))


def sharded_prefill(q, k, v, out, world: int, rank: int, *, key_mask=None, sinks=None, **kw):
    """This rank's share of one attention call: for each of its runs, the
    library's ordinary call on the slices (q, out: [B, Hq, L, D]; k, v:
    [B, Hkv, S, D]; key_mask [B, S]; sinks [Hq]).  Writes only this rank's rows
    of `out`.  Other keyword arguments go to binding.prefill (scale, causal,
    window, softcap, stream, ...)."""
    from . import binding

    B, Hq = q.shape[0], q.shape[1]
    Hkv = k.shape[1]
    G = Hq // Hkv
    for run in rank_runs(B, Hkv, world, rank):
        (qb, qh), (kb, kh) = run_slices(run, G)
        binding.prefill(q[qb, qh], k[kb, kh], v[kb, kh], out=out[qb, qh],
                        key_mask=key_mask[qb] if key_mask is not None else None,
                        sinks=sinks[qh] if sinks is not None else None, **kw)
    return out


def rank_planes(B: int, Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """The query planes [p0, p1) of the flat [B Hq] plane index that rank `rank` writes."""
    G = Hq // Hkv
    u0, u1 = unit_range(B * Hkv, world, rank)
    return u0 * G, u1 * G


def all_gather_output(out, world: int, rank: int, Hkv: int):
    """Every rank's rows of out [B, Hq, L, D] (each rank holding its own, from
    sharded_prefill) gathered into `out` on every rank: the rank's contiguous
    plane range, padded to the longest range, through one all_gather."""
    if world == 1:
        return out
    import torch.distributed as dist

    B, Hq = out.shape[0], out.shape[1]
    plane = out[0, 0].numel()
    flat = out.reshape(B * Hq, plane)
    ranges = [rank_planes(B, Hq, Hkv, world, r) for r in range(world)]
    longest = max(p1 - p0 for p0, p1 in ranges)
    p0, p1 = ranges[rank]
    mine = torch.zeros(longest, plane, dtype=out.dtype, device=out.device)
    mine[: p1 - p0] = flat[p0:p1]
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine)
    for r, (a, b) in enumerate(ranges):
        if r != rank:
            flat[a:b] = parts[r][: b - a]
    return out
