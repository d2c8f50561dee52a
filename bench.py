"""Benchmark of exact blockwise attention forward + (O, LSE) merge on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ring_32k]

One step is one pass of the whole path over one batch of synthetic input: for the
default workload (B=1, H=32, N=32768, d=128, causal, Ring Attention's schedule of 8
query/key-value chunks emulated on one GPU) that is 36 partial attentions and 7
merges. The line printed by rank 0 reports:

  value      device-timed TFLOP/s of the whole job (nominal causal FLOPs
             4*B*H*N^2*d/2 per step, summed over ranks, over the max-over-ranks time),
             inputs resident in HBM; inputs (768 MiB) exceed L2, so no flush is needed;
  roofline   the attention kernel's achieved TFLOP/s (algorithmic FLOPs per launch over
             its CUDA-event duration, on its stream) against the measured burst bf16
             peak (each launch is milliseconds long and the timed region about a
             second, so the burst figure applies; the fraction of the sustained peak,
             measured under the power cap at a lower clock, is reported beside it);
  merge      the merge kernel's achieved GB/s against the measured HBM copy bandwidth;
  e2e        the same metric through the C ABI call with host buffers
             (attn_ring_fwd_host, page-locked): the host->device copies of Q, K, V and
             the device->host copies of O, LSE are inside the timed region, pipelined
             with the compute chunk by chunk;
  cpu_baseline  the fp64 oracle on the host cores, on a bounded row sample of the
             same workload (rank 0, N=1 only);
  per_workload  the other workloads at full size (tiny_chunks4 single pass and as 4
             partials plus a merge; causal_4k, gqa_128k single passes; grid2d_64k_stress
             as its 4 x 4 grid plus merges and as a single pass), a few device-timed
             steps each, with the attention kernel's fraction of the burst peak, the
             merges' GB/s and the oracle's time: in full for tiny_chunks4 and causal_4k,
             on sampled rows (full-size time extrapolated) for the others.

With --gpus N > 1 (launched by torchrun), every rank runs its own independent
problem of the same size (different seed): weak scaling, no data-path collective.
``--impl reference`` times the fp64 oracle on the host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------------------
# host-side helpers (no GPU needed; covered by tests/test_bench_host.py)
# --------------------------------------------------------------------------------------
def dist_env() -> tuple[int, int, int]:
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Independent problem per rank: same shapes, different seeded inputs."""
    return base_seed + 7919 * rank


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(n: int, device) -> int:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return int(n)
    t = torch.tensor([n], dtype=torch.int64, device=device)
    dist.all_reduce(t)
    return int(t.item())


def load_peaks() -> tuple[dict, str]:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return d, "measured"
        except Exception:
            pass
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of ONE attention launch of
# the default step, from one ncu capture of `bench.py --steps 3 --warmup 3
# --no-cpu-baseline` (summarised with its command under profiles/). Keyed by the
# digest of the code (comments excluded) of the kernel sources the capture ran, and by
# launch mode; any other code gives null.
MEASURED_TRAFFIC: dict[str, dict[str, float]] = {
    "3769c3ed194c8c71d93a93eb29b7ab2243cf8d152e4fb47c597a16e7dc31f76b":
        {"batched": 4_207_384_320 + 2_407_732_736},
}


def _code_only(text: str) -> str:
    """C++ source with comments removed and whitespace collapsed: edits to comments or
    layout leave the compiled kernel, and so a traffic capture, unchanged."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_digest() -> str:
    """SHA-256 over the code of the attention kernel's device sources (the files whose
    change invalidates a DRAM-traffic capture), comments and layout excluded."""
    h = hashlib.sha256()
    for name in ("attn_fwd_kernel.cuh", "sm100_ptx.cuh"):
        src = (ROOT / "online_softmax_exact_b200" / "csrc" / name).read_text()
        h.update(_code_only(src).encode())
    return h.hexdigest()


def measured_traffic(batched: bool) -> float | None:
    return MEASURED_TRAFFIC.get(kernel_source_digest(), {}).get(
        "batched" if batched else "per_pair")


def ring_step_plan(n_chunks: int, causal: bool):
    """(partial launches with their nominal FLOP fraction of a full chunk pair, merges
    with their part counts) of one ring step."""
    from online_softmax_exact_b200.schedules import ring_order

    order = ring_order(n_chunks, causal)
    partial_fracs, merge_parts = [], []
    for qi, visit in enumerate(order):
        for kv in visit:
            partial_fracs.append(0.5 if (causal and kv == qi) else 1.0)
        if len(visit) > 1:
            merge_parts.append(len(visit))
    return partial_fracs, merge_parts


def merge_bytes(n_parts: int, rows: int, d: int) -> int:
    """Algorithmic HBM bytes of one merge: each part's O and LSE read once, the result
    written once (fp32)."""
    return (n_parts + 1) * rows * (d + 1) * 4


def parse_clocks(csv_text: str, bus_id: str | None = None) -> dict:
    """Summarise nvidia-smi samples: median SM clock under load and active reasons."""
    lines = [ln.strip() for ln in csv_text.strip().splitlines() if ln.strip()]
    if len(lines) < 2:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    header = [h.strip() for h in lines[0].split(",")]
    rows = [[c.strip() for c in ln.split(",")] for ln in lines[1:] if not ln.startswith(header[0])]

    def col(name):
        for i, h in enumerate(header):
            if h.startswith(name):
                return i
        return None

    i_bus, i_sm, i_max = col("pci.bus_id"), col("clocks.current.sm"), col("clocks.max.sm")
    i_pw = col("power.draw")
    flags = {"hw_slowdown": col("clocks_event_reasons.hw_slowdown"),
             "hw_thermal_slowdown": col("clocks_event_reasons.hw_thermal_slowdown"),
             "sw_thermal_slowdown": col("clocks_event_reasons.sw_thermal_slowdown"),
             "sw_power_cap": col("clocks_event_reasons.sw_power_cap")}
    sel = []
    for r in rows:
        if len(r) != len(header):
            continue
        if bus_id and i_bus is not None and not r[i_bus].upper().startswith(bus_id.upper()):
            continue
        sel.append(r)

    def num(s):
        try:
            return float(s.split()[0])
        except Exception:
            return None

    sm = [num(r[i_sm]) for r in sel if i_sm is not None and num(r[i_sm]) is not None]
    mx = [num(r[i_max]) for r in sel if i_max is not None and num(r[i_max]) is not None]
    pw = [num(r[i_pw]) for r in sel if i_pw is not None and num(r[i_pw]) is not None]
    # "under load": samples drawing well above idle power, else all samples
    load = [s for s, p in zip(sm, pw) if p is not None and p > 300.0] if pw else []
    use = load or sm
    reasons = sorted({name for r in sel for name, i in flags.items()
                      if i is not None and r[i].lower().startswith("active")})
    return {"sm_mhz": statistics.median(use) if use else None,
            "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(sel),
            "samples_under_load": len(load)}


class ClockSampler:
    """nvidia-smi sampling of clocks and throttle reasons while the timed region runs."""

    QUERY = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.tmp = None

    def __enter__(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv", "-lms", "100"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self) -> dict:
        if self.proc is None or self.tmp is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.tmp.flush()
        text = Path(self.tmp.name).read_text()
        try:
            os.unlink(self.tmp.name)
        except OSError:
            pass
        return parse_clocks(text, self.bus_id)


# --------------------------------------------------------------------------------------
# oracle baseline (rank 0 only)
# --------------------------------------------------------------------------------------
def oracle_sample_throughput(w, seconds: float, seed: int = 0) -> dict:
    """Time the fp64 oracle on rows of the workload until ~``seconds`` of CPU work:
    returns nominal TFLOP/s (4 * visible keys * d per row), rows and threads used."""
    import numpy as np

    import oracle
    from workloads import attention_inputs

    q, k, v = attention_inputs(w)
    rng = np.random.default_rng(seed)
    threads = oracle.default_threads()
    flops = 0.0
    rows_done = 0
    t_total = 0.0
    batch = 16
    while t_total < seconds:
        rows = np.sort(rng.choice(w.N, size=batch, replace=False)).astype(np.int64)
        b = int(rng.integers(0, w.B))
        h = int(rng.integers(0, w.Hq))
        g = h // (w.Hq // w.Hkv)
        qh = q[b:b + 1, h:h + 1]
        kh, vh = k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1]
        t0 = time.perf_counter()
        oracle.attention_rows(qh, kh, vh, causal=w.causal, scale=w.scale, rows=rows)
        t_total += time.perf_counter() - t0
        vis = (rows + 1) if w.causal else np.full(batch, w.N)
        flops += float(4.0 * vis.sum() * w.d)
        rows_done += batch
        batch = min(batch * 2, 512)
    return {"tflops": flops / t_total / 1e12, "rows": rows_done, "seconds": t_total,
            "threads": threads, "flops": flops}


def run_reference(args, w) -> int:
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    per_step = args.cpu_seconds if args.cpu_seconds_set else \
        max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_throughput(w, per_step / 4)
    vals, rows, secs, threads = [], 0, 0.0, 1
    flops = 0.0
    for s in range(args.steps):
        r = oracle_sample_throughput(w, per_step, seed=s + 1)
        vals.append(r["tflops"])
        rows += r["rows"]
        secs += r["seconds"]
        flops += r["flops"]
        threads = r["threads"]
    value = flops / secs / 1e12
    sample = (f"{rows} query rows of {w.name} drawn uniformly over (batch, head, row), "
              f"each row's full softmax materialised; {per_step:.1f} s of CPU work per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.flops / (value * 1e12) if value > 0 else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "note": "fp64 CPU oracle (plain materialised softmax, OpenMP over rows); "
                "ms_per_step is extrapolated from the sampled rows' throughput",
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------
METRIC = "attention fwd TFLOP/s and % of bf16 tensor peak on 1 B200; merge HBM GB/s"


def workload_config(w, world: int, streams: int | None = None, batched=None) -> dict:
    return {"workload": f"{w.name}: {w.description}", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
            "N": w.N, "d": w.d, "causal": w.causal, "schedule": w.schedule,
            "n_chunks": w.n_chunks, "global_batch": w.B * world, "seq_len": w.N,
            "parallelism": "single GPU" if world == 1 else f"{world} independent replicas",
            "streams": streams,
            "launch": None if batched is None else (
                "one attn_fwd_partial_batch launch for the 36 ring partials, then 7 merges"
                if batched else "one attn_fwd_partial launch per ring partial, then 7 merges"),
            "l2": "inputs larger than L2 (Q, K, V = 768 MiB per step); no flush"}


class EventTimer:
    """Brackets launches with CUDA events on the stream each launch is issued on."""

    def __init__(self, stream):
        self.stream = stream
        self.records = []  # (kind, start, end)
        self.enabled = False
        self._kind = None
        self._stream = stream

    def __call__(self, kind: str, stream=None):
        self._kind = kind
        self._stream = stream if stream is not None else self.stream
        return self

    def __enter__(self):
        if self.enabled:
            import torch

            self._s = torch.cuda.Event(enable_timing=True)
            self._s.record(self._stream)
        return self

    def __exit__(self, *exc):
        if self.enabled:
            import torch

            e = torch.cuda.Event(enable_timing=True)
            e.record(self._stream)
            self.records.append((self._kind, self._s, e))
        return False

    def totals(self, t0) -> dict:
        """Per kind: (busy ms = union of its launch intervals, launches, summed ms).

        With several streams, launches of one kind can overlap; the union counts the
        device time during which at least one of them was in flight."""
        spans = {}
        for kind, s, e in self.records:
            spans.setdefault(kind, []).append((t0.elapsed_time(s), t0.elapsed_time(e)))
        out = {}
        for kind, iv in spans.items():
            iv.sort()
            busy, cur_a, cur_b = 0.0, None, None
            for a, b in iv:
                if cur_b is None or a > cur_b:
                    if cur_b is not None:
                        busy += cur_b - cur_a
                    cur_a, cur_b = a, b
                else:
                    cur_b = max(cur_b, b)
            if cur_b is not None:
                busy += cur_b - cur_a
            out[kind] = (busy, len(iv), sum(b - a for a, b in iv))
        return out


def run_ours(args, w) -> int:
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())

    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.schedules import Workspace, ring_attention, ring_slots
    from workloads import attention_inputs
    from workloads.configs import Workload

    wr = Workload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})
    q_h, k_h, v_h = attention_inputs(wr)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    B, Hq, N, d = q.shape
    P, C = w.n_chunks, w.N // w.n_chunks
    out = (torch.empty((P, B, Hq, C, d), dtype=torch.float32, device=dev),
           torch.empty((P, B, Hq, C), dtype=torch.float32, device=dev))
    ws = Workspace.for_shape(ring_slots(P, w.causal, args.batched, args.streams), B, Hq, C, d,
                             dev)
    stream = torch.cuda.current_stream(dev)
    timer = EventTimer(stream)

    def step():
        ring_attention(q, k, v, n_chunks=P, causal=w.causal, scale=w.scale, out=out,
                       workspace=ws, stream=stream, timer=timer, n_streams=args.streams,
                       batched=args.batched)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if osx.attn_device_status(reset=True) != osx.ATTN_OK:
        raise RuntimeError("device-side wait ran out of time during warm-up")

    try:
        pr = torch.cuda.get_device_properties(dev)
        bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}"
    except Exception:
        bus = None
    n0 = osx.attn_launch_count()
    timer.enabled = True
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(bus) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    timer.enabled = False
    launches = osx.attn_launch_count() - n0
    ms = t0.elapsed_time(t1)
    if osx.attn_device_status() != osx.ATTN_OK:
        raise RuntimeError("device-side wait ran out of time in the timed region")
    tot = timer.totals(t0)
    clk = clocks.summary()

    ms_max = max_over_ranks(ms, dev)
    launches = sum_over_ranks(launches, dev)

    # ---- per-kernel roofline (this rank's events)
    peaks, peak_src = load_peaks()
    fracs, merges = ring_step_plan(P, w.causal)
    full_pair_flops = 4.0 * B * Hq * C * C * d
    partial_flops_per_step = full_pair_flops * sum(fracs)
    t_part, n_part, sum_part = tot.get("partial", (0.0, 0, 0.0))
    attn_achieved = partial_flops_per_step * args.steps / (t_part * 1e-3) / 1e12
    rows = B * Hq * C
    peak_t = peaks.get("bf16_tflops")
    peak_sus = peaks.get("bf16_tflops_sustained") or peak_t
    peak_h = peaks.get("hbm_gbs")

    # ---- the merge kernel in isolation: the same step on one stream, so that merges do
    # not share the device with attention launches of another stream
    iso = EventTimer(stream)
    n_iso = max(3, min(args.steps, 10))

    def step1():
        ring_attention(q, k, v, n_chunks=P, causal=w.causal, scale=w.scale, out=out,
                       workspace=ws, stream=stream, timer=iso, n_streams=1,
                       batched=args.batched)

    step1()
    torch.cuda.synchronize()
    iso.enabled = True
    t2 = torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    for _ in range(n_iso):
        step1()
    torch.cuda.synchronize()
    iso.enabled = False
    tot1 = iso.totals(t2)
    t_merge, n_merge, sum_merge = tot1.get("merge", (0.0, 0, 0.0))
    t_part1, _, _ = tot1.get("partial", (0.0, 0, 0.0))
    mbytes = sum(merge_bytes(n, rows, d) for n in merges) * n_iso
    merge_gbs = mbytes / (t_merge * 1e-3) / 1e9 if t_merge > 0 else None
    attn_single = partial_flops_per_step * n_iso / (t_part1 * 1e-3) / 1e12 if t_part1 else None

    # ---- the same ring step with the fused running merge (attn_fwd_partial_acc): no
    # partial buffers, no merge launches
    def step_fused():
        ring_attention(q, k, v, n_chunks=P, causal=w.causal, scale=w.scale, out=out,
                       stream=stream, n_streams=args.streams, fused_merge=True,
                       batched=args.batched)

    for _ in range(3):
        step_fused()
    torch.cuda.synchronize()
    n_fused = max(3, min(args.steps, 30))
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(n_fused):
        step_fused()
    f1.record(stream)
    torch.cuda.synchronize()
    ms_fused = max_over_ranks(f0.elapsed_time(f1), dev) / n_fused
    if osx.attn_device_status() != osx.ATTN_OK:
        raise RuntimeError("device-side wait ran out of time in the fused ring step")

    # ---- end to end through the public API with pinned host buffers
    e2e = run_e2e(args, w, q_h, k_h, v_h, dev, world)

    # ---- the other workloads at full size (rank 0 of a one-GPU run reports them)
    per_workload = None
    if world == 1 and args.per_workload:
        del q, k, v, out, ws
        torch.cuda.empty_cache()
        per_workload = run_per_workload(args, dev, peaks, peak_src,
                                        ["tiny_chunks4", "causal_4k", "gqa_128k",
                                         "grid2d_64k_stress"])

    total_flops = w.flops * args.steps * world
    value = total_flops / (ms_max * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: bf16 N(0,1) from a seeded torch CPU generator",
        "config": workload_config(w, world, None if args.batched else args.streams,
                                  bool(args.batched)),
        "pct_of_bf16_peak": 100.0 * (value / world) / peak_t,
        "roofline": {"bound": "tensor",
                     "kernel": "attn_fwd_kernel<128> (" + ("attn_fwd_partial_batch"
                                                           if args.batched else
                                                           "attn_fwd_partial") + ")",
                     "achieved": attn_achieved, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": attn_achieved / peak_t,
                     "peak_source": f"{peak_src} bf16_tflops (burst: the timed region is "
                                    f"{ms / 1e3:.2f} s of launches of ~{t_part / max(1, n_part):.1f}"
                                    " ms each)",
                     "frac_of_sustained": attn_achieved / peak_sus,
                     "sustained_note": f"{peak_src} bf16_tflops_sustained ({peak_sus}) was "
                                       "measured under the power cap at a lower clock; this "
                                       "run's median SM clock is in `clocks`",
                     "traffic": measured_traffic(bool(args.batched)),
                     "traffic_note": "DRAM bytes per attention launch from one ncu capture "
                                     "of this kernel source; null if the source changed",
                     "launches": n_part, "busy_ms": t_part, "summed_launch_ms": sum_part,
                     "timing": "achieved = algorithmic FLOPs of all attention launches in the "
                               "timed region / the device time during which at least one was "
                               "in flight (union of CUDA-event intervals on the launching "
                               "streams)",
                     "achieved_single_stream": attn_single},
        "merge": {"bound": "hbm", "kernel": "attn_merge_kernel<128>", "achieved": merge_gbs,
                  "peak": peak_h, "unit": "GB/s",
                  "frac": (merge_gbs / peak_h) if merge_gbs else None,
                  "peak_source": f"{peak_src} hbm_gbs", "launches": n_merge,
                  "busy_ms": t_merge, "summed_launch_ms": sum_merge,
                  "timing": f"the same ring step on one stream, {n_iso} steps after the timed "
                            "region; algorithmic bytes / CUDA-event time of the merge launches"},
        "fused_running_merge": {
            "value": w.flops * world / (ms_fused * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms_fused, "steps": n_fused,
            "what": "the same ring step with each query chunk's partials folded into one "
                    "running (O, LSE) accumulator (attn_fwd_partial_acc semantics; batched: "
                    "one launch per ring step), no merge launches, no partial buffers"},
        "e2e": e2e,
        "per_workload": per_workload,
        "gpu_launches": launches,
        "clocks": {"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                   "reasons": clk.get("reasons", []), "samples": clk.get("samples", 0)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_sample_throughput(w, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": r["tflops"], "unit": "TFLOP/s", "cores": r["threads"], "kind": "oracle",
            "sample": f"{r['rows']} query rows of {w.name} drawn uniformly over (batch, head, "
                      f"row), full softmax row materialised in fp64; {r['seconds']:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


class L2Flush:
    """Writes a buffer larger than L2 (126 MB on B200) between timed iterations whose
    inputs fit in L2."""

    def __init__(self, dev, nbytes: int = 512 << 20):
        import torch

        self.buf = torch.empty(nbytes // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)


def time_reps(fn, reps: int, stream, flush=None) -> list[float]:
    """CUDA-event times (ms) of ``reps`` calls of ``fn`` on ``stream``, each bracketed
    on its own (an optional L2 flush runs between them, outside the brackets)."""
    import torch

    out = []
    for _ in range(reps):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        out.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def run_per_workload(args, dev, peaks: dict, peak_src: str, names: list[str]) -> dict:
    """Device-timed full-size runs of the other workloads (a few steps each)."""
    import torch

    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.schedules import grid2d_attention
    from workloads import attention_inputs, get, grid_merge_orders

    peak_b = peaks.get("bf16_tflops")
    peak_h = peaks.get("hbm_gbs")
    stream = torch.cuda.current_stream(dev)
    out = {}
    for name in names:
        w = get(name)
        q_h, k_h, v_h = attention_inputs(w)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        del q_h, k_h, v_h
        in_bytes = (q.numel() + k.numel() + v.numel()) * 2
        flush = L2Flush(dev) if in_bytes < (256 << 20) else None
        B, Hq, N, d = q.shape
        o = torch.empty((B, Hq, N, d), dtype=torch.float32, device=dev)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        reps = args.workload_steps

        def single():
            osx.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, o=o, lse=lse, stream=stream)

        for _ in range(3):
            single()
        t_single = time_reps(single, reps, stream, flush)
        ms_single = statistics.median(t_single)
        tf_single = w.flops / (ms_single * 1e-3) / 1e12
        rec = {"workload": f"{w.name}: {w.description}", "flops_per_step": w.flops,
               "steps": reps, "warmup": 3,
               "l2": "flushed (512 MB write) before each timed call" if flush else
                     "inputs larger than L2; no flush",
               "single_pass": {"ms": ms_single, "tflops": tf_single,
                               "frac_of_burst_bf16": tf_single / peak_b}}
        if w.schedule == "chunks":
            # KV in n_chunks pieces as partials, then one merge (launch-bound at this size)
            P, C = w.n_chunks, w.N // w.n_chunks
            parts = [(torch.empty((B, Hq, N, d), dtype=torch.float32, device=dev),
                      torch.empty((B, Hq, N), dtype=torch.float32, device=dev))
                     for _ in range(P)]

            def chunked():
                for i in range(P):
                    osx.attn_fwd_partial(q, k, v, q_start=0, q_len=N, kv_start=i * C, kv_len=C,
                                         causal=w.causal, scale=w.scale, o=parts[i][0],
                                         lse=parts[i][1], stream=stream)
                osx.attn_merge([x[0] for x in parts], [x[1] for x in parts], o=o, lse=lse,
                               stream=stream)

            for _ in range(3):
                chunked()
            t_ch = time_reps(chunked, reps, stream, flush)
            ms_ch = statistics.median(t_ch)
            rec["chunks_with_merge"] = {
                "ms": ms_ch, "tflops": w.flops / (ms_ch * 1e-3) / 1e12,
                "launches": f"{P} attn_fwd_partial + 1 attn_merge per step (launch-bound)"}
        if w.schedule == "grid2d":
            P, C = w.n_chunks, w.N // w.n_chunks
            orders = grid_merge_orders(P, w.seed)
            out_c = (torch.empty((P, B, Hq, C, d), dtype=torch.float32, device=dev),
                     torch.empty((P, B, Hq, C), dtype=torch.float32, device=dev))
            from online_softmax_exact_b200.schedules import Workspace

            ws = Workspace.for_shape(P * P, B, Hq, C, d, dev)
            timer = EventTimer(stream)

            def grid():
                grid2d_attention(q, k, v, n_chunks=P, merge_orders=orders, causal=w.causal,
                                 scale=w.scale, out=out_c, workspace=ws, stream=stream,
                                 timer=timer, batched=True)

            for _ in range(3):
                grid()
            torch.cuda.synchronize()
            timer.enabled = True
            t0 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            t_grid = time_reps(grid, reps, stream, flush)
            timer.enabled = False
            tot = timer.totals(t0)
            ms_grid = statistics.median(t_grid)
            t_part = tot.get("partial", (0.0, 0, 0.0))[0]
            t_merge = tot.get("merge", (0.0, 0, 0.0))[0]
            attn_tf = w.flops * reps / (t_part * 1e-3) / 1e12 if t_part else None
            rows = B * Hq * C
            mbytes = merge_bytes(P, rows, d) * P * reps
            merge_gbs = mbytes / (t_merge * 1e-3) / 1e9 if t_merge else None
            rec["grid_with_merges"] = {
                "ms": ms_grid, "tflops": w.flops / (ms_grid * 1e-3) / 1e12,
                "attention_tflops": attn_tf,
                "attention_frac_of_burst_bf16": attn_tf / peak_b if attn_tf else None,
                "merge_gbs": merge_gbs,
                "merge_frac_of_hbm": merge_gbs / peak_h if merge_gbs else None,
                "launches": f"one attn_fwd_partial_batch launch of the {P * P} cells, then "
                            f"{P} attn_merge ({P} parts each, seeded order) per step"}
            del ws, out_c
        if osx.attn_device_status() != osx.ATTN_OK:
            raise RuntimeError(f"device-side wait ran out of time in {name}")
        if not args.no_cpu_baseline and w.flops <= 2e11:
            # small enough to time the oracle on the whole workload
            import oracle

            q_c, k_c, v_c = attention_inputs(w)
            t0c = time.perf_counter()
            oracle.attention(q_c, k_c, v_c, causal=w.causal, scale=w.scale)
            secs = time.perf_counter() - t0c
            rec["oracle"] = {
                "tflops": w.flops / secs / 1e12, "full_size_s": secs,
                "cores": oracle.default_threads(), "rows": B * Hq * N,
                "note": "fp64 oracle on the whole workload (every row)"}
        elif not args.no_cpu_baseline:
            r = oracle_sample_throughput(w, args.cpu_seconds_per_workload)
            rec["oracle"] = {
                "tflops": r["tflops"], "rows_per_s": r["rows"] / r["seconds"],
                "cores": r["threads"], "rows": r["rows"],
                "full_size_s_extrapolated": w.flops / (r["tflops"] * 1e12),
                "note": "fp64 oracle on uniformly sampled rows; the full-size time is "
                        "extrapolated from the sampled rows' rate"}
        rec["peak_source"] = f"{peak_src} bf16_tflops (burst) / hbm_gbs"
        out[name] = rec
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    return out


def run_e2e(args, w, q_h, k_h, v_h, dev, world) -> dict:
    """The step through the C ABI with HOST buffers (attn_ring_fwd_host): page-locked
    q, k, v in, chunk-major O, LSE out, the copies inside the timed region and
    pipelined with the compute by the library."""
    import torch

    import online_softmax_exact_b200 as osx

    qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    B, Hq, N, d = qp.shape
    C = N // w.n_chunks
    o_h = torch.empty((w.n_chunks, B, Hq, C, d), dtype=torch.float32).pin_memory()
    l_h = torch.empty((w.n_chunks, B, Hq, C), dtype=torch.float32).pin_memory()
    bufs = osx.RingHostBuffers(B, Hq, kp.shape[1], N, d, w.n_chunks, dev)
    stream = torch.cuda.current_stream(dev)
    steps = max(1, min(args.steps, 5))

    def step():
        osx.attn_ring_fwd_host(qp, kp, vp, n_chunks=w.n_chunks, causal=w.causal, scale=w.scale,
                               o_h=o_h, lse_h=l_h, buffers=bufs, device=dev, stream=stream)

    step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    if osx.attn_device_status() != osx.ATTN_OK:
        raise RuntimeError("device-side wait ran out of time in the end-to-end step")
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    h2d = qp.numel() * 2 + kp.numel() * 2 + vp.numel() * 2
    d2h = o_h.numel() * 4 + l_h.numel() * 4

    # the copies alone, same bytes, same page-locked buffers: what bounds this path
    def copies(direction):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if direction == "h2d":
            for src, dst in ((qp, bufs.q), (kp, bufs.k), (vp, bufs.v)):
                dst.copy_(src, non_blocking=True)
        else:
            o_h.copy_(bufs.o, non_blocking=True)
            l_h.copy_(bufs.lse, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    copies("h2d")
    copies("d2h")
    ms_h2d = min(copies("h2d") for _ in range(3))
    ms_d2h = min(copies("d2h") for _ in range(3))
    return {"value": w.flops * steps * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "h2d_gbs": h2d / (ms_h2d * 1e-3) / 1e9, "d2h_gbs": d2h / (ms_d2h * 1e-3) / 1e9,
            "copy_floor_ms": max(ms_h2d, ms_d2h),
            "copy_floor_note": "each direction's bytes copied alone (page-locked, one stream); "
                               "the two directions can overlap, so the step cannot be shorter "
                               "than the slower of them",
            "api": "attn_ring_fwd_host (C ABI; page-locked host buffers; per-chunk copies "
                   "pipelined with the per-query-chunk launches)"}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ring_32k")
    ap.add_argument("--streams", type=int, default=2,
                    help="CUDA streams the ring schedule spreads its query chunks over "
                         "(per-pair launches only)")
    ap.add_argument("--batched", type=int, default=1,
                    help="1: the ring's partials go through attn_fwd_partial_batch "
                         "(one launch for all pairs); 0: one attn_fwd_partial per pair")
    ap.add_argument("--cpu-seconds", type=float, default=None,
                    help="oracle CPU seconds (baseline sample; per step for --impl reference)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-workload", type=int, default=1,
                    help="1: also time causal_4k, gqa_128k and grid2d_64k_stress at full "
                         "size (reported under per_workload)")
    ap.add_argument("--workload-steps", type=int, default=5,
                    help="timed steps per extra workload")
    ap.add_argument("--cpu-seconds-per-workload", type=float, default=2.0)
    args = ap.parse_args(argv)
    args.cpu_seconds_set = args.cpu_seconds is not None
    if args.cpu_seconds is None:
        args.cpu_seconds = 12.0
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from workloads import get

    w = get(args.workload)
    if w.schedule != "ring":
        ap.error("the benchmark step is the ring schedule workload (ring_32k)")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
