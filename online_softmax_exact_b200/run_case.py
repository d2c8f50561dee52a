"""Run one entry point on random inputs of a given shape, for timing and profiling.

    python -m online_softmax_exact_b200.run_case fwd   --B 1 --Hq 32 --N 8192 --d 128 [--causal]
    python -m online_softmax_exact_b200.run_case merge --parts 8 --rows 131072 --d 128
    python -m online_softmax_exact_b200.run_case workload --name grid2d_64k_stress

Does ``--warmup`` untimed calls then ``--reps`` timed calls (CUDA events on the
launching stream) and prints one JSON line with the mean time and the achieved
TFLOP/s (fwd, workload) or GB/s (merge). ``workload`` runs one step of a named
workload's schedule on its seeded inputs: the single pass, the ring's batched partials
and merges, or the 2-D grid's batched cells and merges.
"""

from __future__ import annotations

import argparse
import json

import torch

import online_softmax_exact_b200 as osx


def _workload_step(name: str, dev):
    """(step callable, nominal FLOPs) of a named workload's schedule on its inputs."""
    from workloads.configs import get
    from workloads.gen import attention_inputs, grid_merge_orders

    from . import schedules

    w = get(name)
    q, k, v = (t.to(dev) for t in attention_inputs(w))
    if w.schedule == "ring":
        ws = schedules.Workspace.for_shape(schedules.ring_slots(w.n_chunks, w.causal, True),
                                           w.B, w.Hq, w.N // w.n_chunks, w.d, dev)
        return (lambda: schedules.ring_attention(q, k, v, n_chunks=w.n_chunks, causal=w.causal,
                                                 scale=w.scale, workspace=ws, batched=True),
                w.flops)
    if w.schedule == "grid2d":
        P = w.n_chunks
        ws = schedules.Workspace.for_shape(P * P, w.B, w.Hq, w.N // P, w.d, dev)
        orders = grid_merge_orders(P, w.seed)
        return (lambda: schedules.grid2d_attention(q, k, v, n_chunks=P, merge_orders=orders,
                                                   causal=w.causal, scale=w.scale, workspace=ws,
                                                   batched=True),
                w.flops)
    return (lambda: osx.attn_fwd(q, k, v, causal=w.causal, scale=w.scale), w.flops)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["fwd", "merge", "workload"])
    ap.add_argument("--name", default="grid2d_64k_stress")
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--Hq", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=None)
    ap.add_argument("--N", type=int, default=8192)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--parts", type=int, default=8)
    ap.add_argument("--rows", type=int, default=131072)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=5)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.op == "fwd":
        Hkv = a.Hkv or a.Hq
        q = torch.randn((a.B, a.Hq, a.N, a.d), device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn((a.B, Hkv, a.N, a.d), device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn((a.B, Hkv, a.N, a.d), device=dev, generator=g).to(torch.bfloat16)
        o = torch.empty((a.B, a.Hq, a.N, a.d), device=dev)
        lse = torch.empty((a.B, a.Hq, a.N), device=dev)
        run = lambda: osx.attn_fwd(q, k, v, causal=a.causal, o=o, lse=lse)  # noqa: E731
        work = 4.0 * a.B * a.Hq * a.N * a.N * a.d / (2 if a.causal else 1)
        unit = "TFLOP/s"
    elif a.op == "workload":
        run, work = _workload_step(a.name, dev)
        unit = "TFLOP/s"
    else:
        op = [torch.randn((a.rows, a.d), device=dev, generator=g) for _ in range(a.parts)]
        lp = [torch.randn((a.rows,), device=dev, generator=g) * 10 for _ in range(a.parts)]
        o = torch.empty((a.rows, a.d), device=dev)
        lse = torch.empty((a.rows,), device=dev)
        run = lambda: osx.attn_merge(op, lp, o=o, lse=lse)  # noqa: E731
        work = (a.parts + 1) * a.rows * (a.d + 1) * 4.0
        unit = "GB/s"
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    s.record()
    for _ in range(a.reps):
        run()
    e.record()
    torch.cuda.synchronize()
    if osx.attn_device_status() != osx.ATTN_OK:
        raise RuntimeError("device-side wait ran out of time")
    ms = s.elapsed_time(e) / a.reps
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"op": a.op, "ms": ms, "rate": rate, "unit": unit, "args": vars(a)}))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
