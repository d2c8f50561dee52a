"""Host logic of bench.py, without a GPU: the FLOP and byte accounting, the clock
summary, per-rank seeding, the max-over-ranks reductions on world_size 2 (gloo), and
the reference arm's JSON line."""

from __future__ import annotations

import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from workloads import get  # noqa: E402


def test_ring_plan_accounts_for_the_nominal_flops():
    w = get("ring_32k")
    fracs, merges = bench.ring_step_plan(w.n_chunks, w.causal)
    assert len(fracs) == 36 and fracs.count(0.5) == 8
    assert merges == [2, 3, 4, 5, 6, 7, 8]          # query chunk 0 has one part: no merge
    C = w.N // w.n_chunks
    assert sum(fracs) * 4.0 * w.B * w.Hq * C * C * w.d == pytest.approx(w.flops)
    assert w.flops == pytest.approx(8.796e12, rel=1e-3)


def test_merge_bytes():
    assert bench.merge_bytes(3, 10, 128) == 4 * 10 * 129 * 4


def test_parse_clocks_filters_this_gpu_and_reports_reasons():
    hdr = ("pci.bus_id, clocks.current.sm [MHz], clocks.max.sm [MHz], power.draw [W], "
           "clocks_event_reasons.active, clocks_event_reasons.hw_slowdown, "
           "clocks_event_reasons.hw_thermal_slowdown, clocks_event_reasons.sw_thermal_slowdown, "
           "clocks_event_reasons.sw_power_cap")
    rows = [
        "00000000:1B:00.0, 1800 MHz, 1965 MHz, 900.0 W, 0x4, Not Active, Not Active, Not Active, Active",
        "00000000:1B:00.0, 1700 MHz, 1965 MHz, 950.0 W, 0x4, Not Active, Not Active, Not Active, Active",
        "00000000:1B:00.0, 120 MHz, 1965 MHz, 140.0 W, 0x0, Not Active, Not Active, Not Active, Not Active",
        "00000000:2C:00.0, 900 MHz, 1965 MHz, 990.0 W, 0x40, Not Active, Active, Not Active, Not Active",
    ]
    s = bench.parse_clocks("\n".join([hdr] + rows), "00000000:1B:00")
    assert s["sm_mhz"] == 1750 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    all_gpus = bench.parse_clocks("\n".join([hdr] + rows), None)
    assert "hw_thermal_slowdown" in all_gpus["reasons"]
    assert bench.parse_clocks("", None)["samples"] == 0


def test_rank_seeds_differ_and_are_stable():
    seeds = [bench.rank_seed(2, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == 2


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        t = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
        n = bench.sum_over_ranks(36 + rank, torch.device("cpu"))
        Path(out_dir, f"r{rank}.json").write_text(json.dumps(
            {"rank": r, "world": w, "local": local, "max": t, "sum": n,
             "seed": bench.rank_seed(2, r)}))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_reductions_with_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.loads((tmp_path / f"r{r}.json").read_text()) for r in range(world)]
    for r, x in enumerate(res):
        assert x["rank"] == r and x["world"] == world and x["local"] == r
        assert x["max"] == 11.0            # max over ranks of 10 + rank
        assert x["sum"] == 36 + 37
    assert res[0]["seed"] != res[1]["seed"]


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.3"],
                       capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["metric"] == bench.METRIC


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       env=env, timeout=120, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_event_timer_busy_time_is_the_union_of_intervals():
    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    t = bench.EventTimer(None)
    t.records = [("partial", Ev(0), Ev(2)), ("partial", Ev(1), Ev(3)),
                 ("partial", Ev(5), Ev(6)), ("merge", Ev(3), Ev(4))]
    tot = t.totals(Ev(0))
    assert tot["partial"] == (4.0, 3, 5.0)      # [0,3] and [5,6]
    assert tot["merge"] == (1.0, 1, 1.0)


def test_traffic_is_reported_only_for_the_captured_kernel_source(monkeypatch):
    digest = bench.kernel_source_digest()
    assert len(digest) == 64
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {digest: {"batched": 7.0e9}})
    assert bench.measured_traffic(True) == 7.0e9
    assert bench.measured_traffic(False) is None
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {"0" * 64: {"batched": 7.0e9}})
    assert bench.measured_traffic(True) is None
