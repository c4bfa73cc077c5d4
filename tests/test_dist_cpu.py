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
from sliding_window_gqa_tfa_b200.inputs import WORKLOADS, make_inputs, shaped


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


# ---------------------------------------------------- one call sharded by KV group
@pytest.mark.parametrize("world", [1, 2, 3, 4, 5, 8, 9])
def test_partition_covers_every_unit_exactly_once(world):
    for B in range(1, 5):
        for Hkv in range(1, 9):
            seen = []
            for r in range(world):
                u0, u1 = tdist.unit_range(B * Hkv, world, r)
                assert 0 <= u1 - u0 - (B * Hkv) // world <= 1  # balanced to within one unit
                covered = []
                for run in tdist.rank_runs(B, Hkv, world, r):
                    assert run.nb >= 1 and run.ng >= 1 and run.g0 + run.ng <= Hkv
                    assert run.nb == 1 or (run.g0 == 0 and run.ng == Hkv)  # one contiguous block
                    covered += [(run.b0 + i) * Hkv + run.g0 + j for i in range(run.nb)
                                for j in range(run.ng)]
                assert covered == list(range(u0, u1))  # the rank's own range, in order
                seen += covered
            assert seen == list(range(B * Hkv))


def _rank_sharded_oracle(rank, world, port, out, case):
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    tdist.setup("gloo", timeout_s=60)
    w = shaped(*case["shape"], window=case["window"], key_mask_keep=case["keep"])
    q, k, v, km = make_inputs(w, seed=7)  # every rank holds the whole call's inputs
    G = w.Hq // w.Hkv
    o = torch.zeros(w.B, w.Hq, w.L, w.D, dtype=torch.float64)
    # this rank's runs, each computed by the oracle on its slices only
    for run in tdist.rank_runs(w.B, w.Hkv, world, rank):
        (qb, qh), (kb, kh) = tdist.run_slices(run, G)
        part = oracle.attention(q[qb, qh].contiguous(), k[kb, kh].contiguous(), v[kb, kh].contiguous(),
                                scale=w.softmax_scale, causal=w.causal, window=w.window,
                                key_mask=km[qb].contiguous() if km is not None else None)
        o[qb, qh] = torch.from_numpy(part)
    p0, p1 = tdist.rank_planes(w.B, w.Hq, w.Hkv, world, rank)
    written = o.reshape(w.B * w.Hq, -1)
    outside = torch.cat([written[:p0], written[p1:]])
    own_only = bool((outside == 0).all())
    tdist.all_gather_output(o, world, rank, w.Hkv)
    whole = oracle.attention(q, k, v, scale=w.softmax_scale, causal=w.causal, window=w.window,
                             key_mask=km)
    out[rank] = (own_only, float((o - torch.from_numpy(whole)).abs().max()))
    tdist.teardown(world)


@pytest.mark.parametrize("world,case", [
    (2, {"shape": (1, 8, 4, 33, 47, 128), "window": 0, "keep": None}),
    (3, {"shape": (2, 6, 3, 20, 50, 64), "window": 9, "keep": 0.7}),
], ids=["b1_hkv4_2ranks", "b2_hkv3_3ranks_window_mask"])
def test_sharded_call_all_gathered_equals_the_whole_call(world, case):
    # each rank computes only its (b, KV group) units, by the oracle; after the
    # all-gather every rank holds exactly the whole call's result
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_sharded_oracle, args=(world, port, out, case), nprocs=world, join=True)
    for r in range(world):
        own_only, err = out[r]
        assert own_only  # before the gather a rank wrote its own planes and nothing else
        assert err == 0.0  # rows are independent: the slices give the whole result bit for bit


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_bench_runs_weak_and_strong(world):
    import bench

    for w in (WORKLOADS["llama_gqa_chunk_2048x8192"], WORKLOADS["qwen3_prefill_b4_2048"]):
        G = w.Hq // w.Hkv
        strong_units = []
        for rank in range(world):
            # weak: every rank runs exactly its own copy of the workload
            weak = bench.bench_runs(w, world, rank, strong=False)
            units = [(r_.b0 + i, r_.g0 + j) for r_ in weak for i in range(r_.nb) for j in range(r_.ng)]
            assert units == [(b, g) for b in range(w.B) for g in range(w.Hkv)]
            # strong: the ranks share the workload's own units
            for r_ in bench.bench_runs(w, world, rank, strong=True):
                (qb, qh), (kb, kh) = tdist.run_slices(r_, G)
                assert qh.stop - qh.start == G * (kh.stop - kh.start)
                strong_units += [(r_.b0 + i, r_.g0 + j) for i in range(r_.nb) for j in range(r_.ng)]
        assert strong_units == [(b, g) for b in range(w.B) for g in range(w.Hkv)]
