"""The benchmark's multi-rank host logic on CPU: two gloo ranks (127.0.0.1), no GPU.

Each rank is an independent replica of the layer (tokens shard with no exchange
step), so the only cross-rank operations are the barrier and the maximum of the
per-rank device time; the reference arm runs on rank 0 alone.  The untimed
steps under the clock sampler are sized from each rank's own step time, and
every rank must run the same number (an expert-parallel step has collectives).
"""
import os
import socket

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.dist_barrier(world)
        mine = 10.0 + 5.0 * rank          # per-rank elapsed ms
        got = bench.dist_max(mine, world, torch.device("cpu"))
        # the reference arm: only rank 0 does any work or prints
        ref = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), None, rank, world) if rank else "rank0"
        soak = bench.soak_count(0.3 if rank == 0 else 0.5, lambda v: bench.dist_max(v, world, torch.device("cpu")))
        out.put((rank, got, ref, soak))
        bench.dist_barrier(world)
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_only_rank0_reports():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict((r, (g, ref, soak)) for r, g, ref, soak in [q.get(timeout=5) for _ in range(2)])
    assert res[0][0] == res[1][0] == 15.0
    assert res[1][1] is None and res[0][1] == "rank0"
    # about 1 s of the faster rank's 0.3 ms steps, on both ranks
    assert res[0][2] == res[1][2] == int(bench_soak_s() * 1e3 / 0.3)


def bench_soak_s():
    import bench
    return bench.SOAK_S


def test_soak_count_is_bounded():
    import bench
    same = lambda v: v  # noqa: E731  (one rank)
    assert bench.soak_count(1.0, same) == int(bench.SOAK_S * 1e3)
    assert bench.soak_count(0.0, same) == 100000  # a step time of 0 is clamped, not divided by
    assert bench.soak_count(1e9, same) == 1
