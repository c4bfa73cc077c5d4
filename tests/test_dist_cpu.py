"""The multi-rank path of the benchmark on the CPU: two gloo ranks on
127.0.0.1 run the plumbing bench.py uses on GPUs (join, barrier, max over
ranks, the weak-scaling aggregate, teardown), each with its own seeded inputs.
No GPU and no data-path collective is involved: the units are independent."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from sliding_window_gqa_tfa_b200 import dist as tdist
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w_, r_, l_ = tdist.setup("gloo", timeout_s=60)
    assert (w_, r_, l_) == (world, rank, rank)
    q, k, _, _ = make_inputs(WORKLOADS["witness_33x47"], seed=rank)  # each rank its own units
    tdist.barrier(world)
    my_ms = 10.0 + 5.0 * rank  # a per-rank device time
    mx = tdist.max_over_ranks(my_ms, world)
    rate = tdist.weak_scaling_rate(1000.0, world, mx * 1e-3)
    out[rank] = (mx, rate, float(q.float().sum()), float(k.float().sum()))
    tdist.teardown(world)


def test_two_gloo_ranks_take_the_max_and_aggregate():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    res = [out[r] for r in range(world)]
    for mx, rate, _, _ in res:
        assert mx == 15.0                     # the slowest rank's time, on every rank
        assert rate == pytest.approx(1000.0 * world / 15e-3)  # all ranks' units / max time
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]  # distinct per-rank inputs
    q0, k0, _, _ = make_inputs(WORKLOADS["witness_33x47"], seed=0)
    assert res[0][2] == float(q0.float().sum()) and res[0][3] == float(k0.float().sum())


def _rank_lost_peer(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    tdist.setup("gloo", timeout_s=5)
    if rank == 1:
        return  # leaves between steps, before the collective
    try:
        tdist.max_over_ranks(1.0, world)
        out[rank] = "completed"
    except Exception as e:  # the short process-group timeout ends the wait with an error
        out[rank] = type(e).__name__


def test_a_lost_rank_ends_the_others_wait_with_an_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank_lost_peer, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=60)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert out.get(0) not in (None, "completed")
