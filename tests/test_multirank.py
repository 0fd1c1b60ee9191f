"""The N > 1 host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

The layer shards by tokens with no exchange, so multi-GPU runs are independent
replicas; what the ranks share is the timing protocol: a barrier on both sides
of the timed region, the step time taken as the maximum over ranks, rank 0
alone printing, and the reference arm running on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        # each rank "measured" a different time; every rank must see the slowest
        out[rank] = bench._max_over_ranks(1.5 + rank, world)
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup = 1, 3

    # rank 1 returns at once: no oracle work, nothing printed
    assert bench.run_reference(Args, bench.WORKLOAD.layers[0]) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(3.25, 1) == 3.25
    bench._barrier(1)


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """Rank 0 of the reference arm (the oracle on the host cores) prints one JSON
    line with the bench contract's keys, its own cpu_baseline and an e2e entry
    with no host-device traffic."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")

    class Args:
        steps, warmup = 1, 3

    assert bench.run_reference(Args, bench.WORKLOAD.layers[0]) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == bench.WORKLOAD.name
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_clock_sampler_summary_parses_nvidia_smi_lines():
    """The clocks record of the bench line: median SM clock under load, the
    largest max clock, and every throttle reason seen Active in any sample."""
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler("GPU-00000000-0000-0000-0000-000000000000")
    assert cs.uuid.startswith("GPU-")
    cs.out = "\n".join([
        "1965, 1965, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1800, 1965, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1900, 1965, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
    ])
    s = cs.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4
    cs.out = ""
    assert cs.summary()["reasons"] == ["unavailable"]
