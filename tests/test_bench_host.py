"""Host-side logic of bench.py: multi-rank timing (world size 2 over gloo on
CPU) and the sizing of the oracle arm. No GPU needed."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own_ms = [2.0, 3.5][rank]                 # rank 1 is the slow one
        ms = bench.max_over_ranks(own_ms, world, dist, torch.device("cpu"))
        rate = bench.whole_job_rate(1000.0, ms, world)
        results[rank] = (ms, rate)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        got = dict(results)
    assert got[0] == got[1]                       # every rank reports the same figure
    ms, rate = got[0]
    assert ms == 3.5                              # the slowest rank sets the time
    assert rate == pytest.approx(2 * 1000.0 / 3.5e-3)  # units of both ranks / that time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.whole_job_rate(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_reference_rows_fit_the_budget():
    Ns = [5120, 17408, 5120]
    per_row = [1e-5, 1e-5, 3.4e-5]
    full = sum(p * n for p, n in zip(per_row, Ns))
    assert bench.reference_rows(per_row, Ns, 10 * full) == Ns     # whole matrices when they fit
    rows = bench.reference_rows(per_row, Ns, full / 4)
    assert all(8 <= r <= n for r, n in zip(rows, Ns))
    assert sum(p * r for p, r in zip(per_row, rows)) <= full / 4 * 1.001
    assert bench.reference_rows(per_row, Ns, 0.0) == [8, 8, 8]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3", "--ref-seconds", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "GB/s" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle"
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0


def test_clock_summary_reads_median_and_active_reasons():
    # index, clocks.sm, clocks.max.sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = cs.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_thermal_and_handles_no_samples():
    cs = bench.ClockSampler(0)
    cs.lines = ["0, 1500, 1965, 1000.0, 0x48, Active, Not Active, Active, Not Active"]
    s = cs.summary()
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    empty = bench.ClockSampler(0)
    assert empty.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
