"""bench.py's host logic, on the CPU.

Multi-rank plumbing as two gloo ranks on 127.0.0.1: with N > 1 every rank
trains its own replica; the job's time is the slowest rank's (an all-reduce
MAX that every rank joins), the value counts the tokens of all ranks, and the
reference arm runs on rank 0 only.  And the clock record the bench line
carries, from nvidia-smi's rows.
"""
import argparse
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")  # rank 1 is the slower one
    e2e_ms = bench.max_over_ranks(3.0 - rank, world, "cpu")  # rank 0 is the slower one
    value = bench.job_tokens_per_s(world, 5, 524288, ms)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, e2e_ms, value))


def test_two_ranks_take_the_slowest_rank_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        out = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r for r, *_ in out] == [0, 1]
    for _, ms, e2e_ms, value in out:
        assert ms == 15.0
        assert e2e_ms == 3.0
        assert value == pytest.approx(2 * 5 * 524288 / 0.015)


def test_one_rank_keeps_its_own_time():
    import bench

    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_tokens_per_s(1, 4, 1000, 2000.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="t1024", warmup=1, steps=1, gpus=2)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_clock_summary_takes_busy_samples_and_active_reasons():
    """The clock record of the bench line, from nvidia-smi's CSV rows
    (index, sm, max sm, power, active mask, hw, hw thermal, sw thermal, sw power cap)."""
    import bench

    rows = [
        "0, 1980, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle sample at start
        "0, 1590, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1560, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1605, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 300, 1965, 80.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # below half the maximum
    ]
    rec = bench.ClockSampler.summarize("\n".join(rows))
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["sm_mhz"] == 1597.5  # median of 1980, 1590, 1560, 1605
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] == 5
    hot = rows[1].replace("Not Active, Not Active, Not Active, Active", "Active, Not Active, Active, Active")
    assert bench.ClockSampler.summarize(hot)["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarize("") is None
