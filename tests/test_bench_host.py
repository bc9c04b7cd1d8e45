"""Host logic of bench.py: work accounting and the multi-rank aggregation.

The replica path has no data-path collective; the only cross-rank steps are
the max over ranks of the device time and the sum of the work.  They are
checked here with world-size-2 gloo process groups on the CPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from oracle import area_oracle as ora
from workloads import CONFIGS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [120.5, 97.25][rank]
        work = [3.0e12, 5.0e12][rank]
        mx = bench.reduce_max(dist, ms)
        tot = bench.reduce_sum(dist, work)
        bench.barrier(dist)
        out[rank] = (mx, tot)
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        mx, tot = out[r]
        assert mx == 120.5 and tot == 8.0e12


def test_reduce_identity_without_process_group():
    assert bench.reduce_max(None, 3.5) == 3.5
    assert bench.reduce_sum(None, 2.0) == 2.0


def test_dist_env_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "2")
    monkeypatch.setenv("LOCAL_RANK", "2")
    assert bench.dist_env() == (2, 4, 2)


def test_phase_flop_counts_match_closed_forms():
    cfg = CONFIGS["flux4096"]
    assert bench.phase1_flops(cfg) == 4.0 * 24 * 65536 * 4096 * 128      # 3.30 TFLOP
    assert abs(bench.phase1_flops(cfg) / 1e12 - 3.298) < 1e-3
    assert abs(bench.full_flops(CONFIGS["flux6144"]) / 1e12 - 267.2) < 0.1
    # Phase I is 1/f^2 of full attention
    assert bench.phase1_flops(cfg) * cfg.f ** 2 == bench.full_flops(cfg)


def test_window_flops_from_plan_dict():
    rng = np.random.default_rng(0)
    E = rng.random((8, 8)).astype(np.float32)
    plan = ora.window_plan(E, 16, 16, 6, 1, 5, 0.4)
    d = {"B": 1, "nwin": np.array([plan.windows.shape[0]]), "win": plan.windows[None],
         "ext": plan.ext[None], "gcount": plan.gcount[None]}
    want = 0
    for i, (y0, x0, hy, wx) in enumerate(plan.windows):
        want += hy * wx * (len(ora.window_kv_tokens(plan, i)))
    assert bench.window_flops(d, H=3, D=128) == 4.0 * 128 * 3 * want


def test_plan_launch_count():
    assert bench.plan_launches(1) == 18
    assert bench.plan_launches(2) == 31


def test_head_range_partitions_the_heads():
    for H in (1, 2, 5, 24, 25):
        for world in range(1, 9):
            ranges = [bench.head_range(r, world, H) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0                                   # contiguous, no overlap
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1                   # balanced


def _shard_worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        h0, h1 = bench.head_range(rank, world, 24)
        work = 1.0e12 * (h1 - h0)                      # per-rank share of one problem
        ms = 100.0 + rank                              # slowest rank sets the time
        out[rank] = (bench.reduce_sum(dist, work), bench.reduce_max(dist, ms))
    finally:
        dist.destroy_process_group()


def test_head_sharded_job_value_over_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 3, port, out)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(3):
        total, ms = out[r]
        assert total == 24.0e12 and ms == 102.0           # whole problem over the slowest rank


def test_reference_arm_line(capsys, monkeypatch):
    # the reference arm (the oracle on the host cores) prints the contract's
    # keys with the same config object as the device arm
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import json
    assert bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0",
                       "--ref-budget", "0.5"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["config"] == bench.workload_config(CONFIGS["tiny"], CONFIGS["tiny"].H, 1, False)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_clock_summary_reads_the_sampled_csv(tmp_path):
    # nvidia-smi rows: index, sm, max sm, power, active, hw, hw_thermal, sw_thermal, sw_power_cap
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join([
        "0, 1965, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1750, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 300, 1965, 80.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle sample
        "garbage line",
    ]) + "\n")
    cs = bench.ClockSampler(0)
    cs.path = str(path)
    cs.proc = object()                               # as if nvidia-smi had run
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965.0 and s["samples"] == 4
    assert s["sm_mhz"] == 1800.0                     # median of the samples under load
    assert s["reasons"] == ["sw_power_cap"]
    path.write_text("0, 1500, 1965, 700.0, 0x8, Not Active, Active, Not Active, Not Active\n")
    assert bench.ClockSampler.summary(cs)["reasons"] == ["hw_thermal_slowdown"]


def test_clock_summary_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None,
                            "reasons": ["nvidia-smi unavailable"]}


def test_traffic_is_null_for_another_kernel_revision(monkeypatch, tmp_path):
    # roofline.traffic comes from the committed DRAM capture only while it was
    # taken from the same build of the kernel
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"flux6144": {"window_attn": {"kernel_revision": bench.KERNEL_REVISION,
                                      "bytes_per_call": 123.0}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("flux6144", "window_attn") == 123.0
    monkeypatch.setattr(bench, "KERNEL_REVISION", "some later build")
    assert bench.load_traffic("flux6144", "window_attn") is None
    assert bench.load_traffic("no-such-workload", "window_attn") is None


def _error_worker(rank, world, port, out):
    # a failure seen by one rank reaches every rank through the same
    # collective, so all of them take the same exit
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_error = 1.0 if rank == 1 else 0.0
        out[rank] = bench.reduce_max(dist, local_error)
    finally:
        dist.destroy_process_group()


def test_one_ranks_error_reaches_all_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_error_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 1.0 and out[1] == 1.0
