"""Run single stages of the layer on a workload's shapes, for profiler captures.

    python -m combine_top_route_counting_b200.stage_probe --workload kimi \
        --stages route,schedule --calls 5

Allocates only what the chosen stages need (routing: the logits, ids and
gates; schedule: the schedule's outputs and scratch), so a capture of the
routing and schedule kernels at the full token count holds a few hundred MB
on the device instead of the layer's tens of GB. Each call runs the chosen
stages once, in order, on the current stream; the script prints the device
time of each stage (CUDA events, median over the calls).
"""
from __future__ import annotations

import argparse
import statistics

import torch

from combine_top_route_counting_b200 import inputs, moe


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="kimi")
    ap.add_argument("--stages", default="route,schedule")
    ap.add_argument("--calls", type=int, default=5)
    args = ap.parse_args(argv)
    stages = [s for s in args.stages.split(",") if s]
    for s in stages:
        if s not in ("route", "schedule"):
            raise SystemExit(f"unknown stage {s}")
    moe.load()
    dev = torch.device("cuda")
    w = inputs.WORKLOADS[args.workload]
    sh = moe.shape(**w.shape())
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=dev)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=dev)
    if w.logits == "ids":  # the scheduler-only workload comes with its ids
        ids.copy_(inputs.make_sched_ids(w).reshape(w.n_tokens, w.k))
        stages = [s for s in stages if s != "route"]
        lg = None
    else:
        lg = inputs.make_logits(w).to(dev)
    b = moe.alloc_schedule_outputs(sh, device=dev)
    times = {s: [] for s in stages}
    for _ in range(args.calls):
        for s in stages:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if s == "route":
                moe.moe_route_topk(lg, ids, gates, sh)
            else:
                moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                                 b["dev_status"], sh)
            e1.record()
            times[s].append((e0, e1))
    torch.cuda.synchronize()
    if int(b["dev_status"].item()) != 0:
        raise SystemExit(f"device status {int(b['dev_status'].item())}")
    for s, ev in times.items():
        us = statistics.median(a.elapsed_time(c) for a, c in ev) * 1e3
        print(f"{args.workload} {s}: {us:.1f} us (median of {len(ev)} calls)")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
