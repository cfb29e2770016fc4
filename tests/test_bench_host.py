"""Host-side logic of bench.py that needs no GPU: the clock record's summary and the
multi-rank timing (barrier, maximum over ranks) on world_size-2 gloo process groups.

The forward shards as independent replicas (one whole problem per GPU, no collective on
the data path); the only cross-rank steps are the timing barrier and the max-reduction of
the per-rank device time, which these tests exercise on CPU.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_clock_summary_reads_reasons_and_median():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbled",
    ]
    s = c.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_thermal_slowdown():
    c = bench.ClockSampler(0)
    c.lines = ["0, 1200, 1965, 0, 0x40, Not Active, Active, Not Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_thermal_slowdown"]


def test_clock_summary_without_samples():
    assert bench.ClockSampler(0).summary()["samples"] == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times_ms, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        total = bench.allreduce_max(times_ms[rank], world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, total))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("times_ms", [(120.0, 95.5), (10.0, 10.0)])
def test_max_over_ranks_on_two_gloo_ranks(times_ms):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = dict(q.get(timeout=5) for _ in range(world))
    assert got == {r: max(times_ms) for r in range(world)}


def test_single_rank_needs_no_process_group():
    bench.barrier(1)
    assert bench.allreduce_max(3.25, 1, torch.device("cpu")) == 3.25
