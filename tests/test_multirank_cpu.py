"""The benchmark's multi-rank host logic on CPU: two gloo ranks (127.0.0.1), no GPU.

Each rank is an independent replica of the layer (tokens shard with no exchange
step), so the only cross-rank operations are the barrier and the maximum of the
per-rank device time; the reference arm runs on rank 0 alone.  The clock
record's summary of NVML samples is checked against a fake NVML here.
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
        out.put((rank, got, ref))
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
    res = dict((r, (g, ref)) for r, g, ref in [q.get(timeout=5) for _ in range(2)])
    assert res[0][0] == res[1][0] == 15.0
    assert res[1][1] is None and res[0][1] == "rank0"


class _FakeNvml:
    """The NVML reason constants the clock record decodes (their values in NVML's header)."""
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40


def test_clock_record_from_samples():
    import bench
    idle_bit = 0x1  # GPU idle: not a reason the record reports
    samples = [(1965.0, 0), (1830.0, 0x4), (1965.0, idle_bit), (1890.0, 0x4)]
    rec = bench.clock_summary(samples, 1965.0, _FakeNvml)
    assert rec == {"sm_mhz": 1927.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 4}
    rec = bench.clock_summary([(1500.0, 0x8 | 0x40)], 1965.0, _FakeNvml)
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.clock_summary([], None, _FakeNvml)["sm_mhz"] is None
