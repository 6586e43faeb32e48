"""Benchmark of the deterministic MoE layer forward on B200.

python bench.py --gpus N --steps K --warmup W [--workload kimi] [--impl ours|reference]

One step = one moe_layer_forward over one batch of the workload (routing,
schedule Phi, dispatch, grouped SwiGLU FFN, combine), inputs resident in HBM.
With N > 1 (launched by torchrun) every rank runs an independent replica on
its own GPU (the layer is not sharded here): value = tokens of all ranks /
max-over-ranks device time. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (test infrastructure) on a bounded
sample of the same workload on the host cores, as the reference arm.

The line also carries a "backward" object: the training step of the same
layer (moe_layer_forward_train, which keeps the activations, and
moe_layer_backward: reverse combine, dgrad GEMMs, reverse dispatch, router
gradient, wgrad GEMMs) timed on the same batch, with per-stage rooflines.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd tokens/s @1 B200; Φ build µs; % of tensor/HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS,
                bf16_sus=FALLBACK_BF16_TFLOPS_SUSTAINED, source="fallback")


def workload_desc(w) -> str:
    return (f"{w.name}: P={w.P} peers x {w.N} tokens, H={w.H}, I={w.I}, E={w.E}, top-{w.k}, "
            f"pad {w.pad}")


# ---------------------------------------------------------------- algorithmic work
def algorithmic_work(w, rows_used: int, rows_real: int):
    """Bytes / flops each stage must move or compute (real routes only)."""
    T, R, H, I, E, k = w.n_tokens, w.n_routes, w.H, w.I, w.E, w.k
    return {
        "route": dict(bytes=T * E * 4 + R * 8),
        "schedule": dict(bytes=2 * R * 4 + rows_used * 8 + R * 4),
        "dispatch": dict(bytes=R * H * 2 + rows_used * H * 2),
        "ffn_gemm1": dict(flops=2 * rows_real * H * 2 * I),
        "ffn_gemm2": dict(flops=2 * rows_real * I * H),
        "combine": dict(bytes=R * H * 4 + T * H * 2 + R * 8),
    }


def backward_work(w, rows_used: int):
    """Bytes / flops of each backward stage (real routes only)."""
    T, R, H, I, E = w.n_tokens, w.n_routes, w.H, w.I, w.E
    return {
        "reverse_combine": dict(bytes=R * H * 2 + rows_used * H * 2),
        "dgrad_h": dict(flops=2 * R * H * I),
        "dgrad_x": dict(flops=2 * R * 2 * I * H),
        "reverse_dispatch": dict(bytes=R * H * 4 + T * H * 2 + R * 4),
        "router_bwd": dict(bytes=R * (I // 128) * 4 + R * 12 + T * E * 4),
        "wgrad_w2": dict(flops=2 * R * I * H),
        "wgrad_w13": dict(flops=2 * R * H * 2 * I),
    }


def mx_layer_work(w, rows_used: int):
    """Bytes / flops of each stage of the MXFP8 layer (real routes only): the
    dispatch reads bf16 tokens and writes E4M3 codes + E8M0 scales; the GEMMs
    do the bf16 layer's flops on E4M3 operands."""
    work = algorithmic_work(w, rows_used, w.n_routes)
    work["dispatch"] = dict(bytes=w.n_routes * w.H * 2 + rows_used * (w.H + w.H // 32))
    for g in ("ffn_gemm1", "ffn_gemm2"):
        work[g] = dict(flops=work[g]["flops"], fp8=True)
    return work


def dispatch_fused(w) -> bool:
    """Whether the layer runs the pull dispatch inside GEMM1 (the library does
    so when expert segments are padded to multiples of 256 rows)."""
    return w.pad % 256 == 0


def stage_rooflines(stage_ms: dict, work: dict, peaks: dict, fused_dispatch: bool = False) -> dict:
    out = {}
    for name, t in stage_ms.items():
        d = {"ms": t}
        if fused_dispatch and name == "dispatch":
            # only the zeroing of the landing flags is left between the events
            d.update(bytes=work[name]["bytes"], fused_into="ffn_gemm1")
            out[name] = d
            continue
        if fused_dispatch and name == "ffn_gemm1":
            d["includes"] = "the pull dispatch (run by a spare warp inside the kernel)"
        if "bytes" in work[name]:
            gbs = work[name]["bytes"] / (t / 1e3) / 1e9
            d.update(bytes=work[name]["bytes"], gbs=gbs, frac_hbm=gbs / peaks["hbm"])
        elif work[name].get("fp8"):
            # E4M3 operands: the bf16 peak x the nominal fp8/bf16 ratio (4.5 / 2.25)
            tf = work[name]["flops"] / (t / 1e3) / 1e12
            d.update(flops=work[name]["flops"], tflops=tf, frac_fp8=tf / (2.0 * peaks["bf16_sus"]),
                     frac_fp8_burst=tf / (2.0 * peaks["bf16"]))
        else:
            tf = work[name]["flops"] / (t / 1e3) / 1e12
            d.update(flops=work[name]["flops"], tflops=tf, frac_bf16=tf / peaks["bf16_sus"],
                     frac_bf16_burst=tf / peaks["bf16"])
        out[name] = d
    return out


# ---------------------------------------------------------------- the other workloads
def _flush_l2(buf):
    """Write a buffer larger than L2 (126 MB) so the next launch starts cold."""
    buf.fill_(1)


def time_configs(moe, dev, W_kimi, x_kimi, ws_big, st, steps: int, warmup: int, peaks: dict):
    """The other workloads, timed in the same run on the same device:
    sched: Phi build (ids -> Phi) on the scheduler workload, CUDA events around
    each call, L2 flushed before each; zipf: the adversarial layer on the Kimi
    shape (the Kimi weights and activations, Zipf routing), stage rooflines;
    mid: the mid layer, stage rooflines; tiny: one layer call's latency. mid and
    tiny fit in L2, so each timed call follows an L2 flush and is timed alone."""
    import torch

    from combine_top_route_counting_b200 import inputs
    out = {}
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, n, per_call_events=None):
        """Per-call device times (ms) of n calls, each after an L2 flush."""
        ts = []
        for i in range(n):
            _flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(per_call_events[i] if per_call_events else None)
            e1.record()
            ts.append((e0, e1))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ts]

    # Phi build on the scheduler workload: P=8 x 7,168 tokens, E=384, top-8 ids
    w = inputs.WORKLOADS["sched"]
    sh = moe.shape(**w.shape())
    ids = inputs.make_sched_ids(w).to(dev)
    b = moe.alloc_schedule_outputs(sh, device=dev)
    sched = lambda _ev: moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"],
                                          b["ws"], b["dev_status"], sh)
    for _ in range(warmup):
        sched(None)
    n = max(steps, 20)
    t = timed(sched, n)
    torch.cuda.synchronize()
    if int(b["dev_status"].item()) != 0:
        raise RuntimeError("device status in the scheduler workload")
    out["sched"] = {"workload": workload_desc(w), "phi_build_us_median": 1e3 * statistics.median(t),
                    "phi_build_us_min": 1e3 * min(t), "calls": n,
                    "what": "moe_schedule: count, prefixes, offsets and placement in one "
                            "cooperative launch (after a 12 KB memset of its barrier and "
                            "totals) on uniform ids; L2 flushed before each call"}
    del b, ids

    def layer_leg(name, W, x, ws, n_calls, flush_each):
        w = inputs.WORKLOADS[name]
        sh = moe.shape(**w.shape())
        lg = inputs.make_logits(w).to(dev)
        o = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.N_STAGE_EVENTS)]
              for _ in range(n_calls)]
        for row in ev:
            for e in row:
                e.record()  # creates the event (torch creates events lazily)
        call = lambda e: moe.moe_layer_forward(lg, x, *W, o, ws, st, sh, stage_events=e)
        for _ in range(warmup):
            call(None)
        torch.cuda.synchronize()
        if flush_each:
            t = timed(call, n_calls, ev)
            ms = statistics.median(t)
        else:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(n_calls):
                call(ev[i])
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / n_calls
        if int(st.item()) != 0:
            raise RuntimeError(f"device status in the {name} layer")
        stage_ms = {nm: statistics.median(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n_calls))
                    for j, nm in enumerate(moe.STAGES)}
        rows = schedule_rows(moe, w, sh, lg)
        d = {"workload": workload_desc(w), "value": w.n_tokens / (ms / 1e3), "unit": "tokens/s",
             "ms_per_step": ms, "phi_build_us": 1e3 * stage_ms["schedule"], "rows_padded": rows,
             "stages": stage_rooflines(stage_ms, algorithmic_work(w, rows, w.n_routes), peaks,
                                       dispatch_fused(w))}
        return d

    # the adversarial layer: Kimi shapes with Zipf routing (hot and empty experts)
    z = layer_leg("zipf", W_kimi, x_kimi, ws_big, steps, False)
    z["note"] = ("the Kimi workload's weights and activations with Zipf(1.2) routing and 8 "
                 "experts never chosen; inputs larger than L2")
    out["zipf"] = z
    for name in ("mid", "tiny"):
        w = inputs.WORKLOADS[name]
        sh = moe.shape(**w.shape())
        W = inputs.make_weights(w, device=dev)
        x = inputs.make_x(w, device=dev)
        ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        d = layer_leg(name, W, x, ws, max(steps, 20), True)
        d["note"] = "median of single calls, each after an L2 flush (the workload fits in L2)"
        if name == "tiny":
            d["latency_us"] = d["ms_per_step"] * 1e3
        out[name] = d
        del W, x, ws
    del flush
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid not in f[1].lower().replace("gpu-", ""):
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            for name, col in (("hw_slowdown", 6), ("hw_thermal_slowdown", 7),
                              ("sw_thermal_slowdown", 8), ("sw_power_cap", 9)):
                if f[col].lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def gpu_uuid(dev) -> str | None:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid).lower()
        return u.replace("gpu-", "") or None
    except Exception:
        return None


# ---------------------------------------------------------------- ranks
def reduce_max(values, group_ready: bool, device=None):
    """Element-wise max over ranks (device time is reported as the slowest rank)."""
    if not group_ready:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def init_dist(world: int, local_rank: int, backend: str = "nccl"):
    if world <= 1:
        return False
    import torch
    import torch.distributed as dist
    kw = dict(backend=backend, timeout=datetime.timedelta(seconds=300))
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local_rank)
    dist.init_process_group(**kw)
    return True


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(w, lg, x_cpu, W_dev, n_experts: int, n_comb: int = 256,
                  threads: int | None = None):
    """Time the CPU oracle on a bounded sample of the workload and scale it to
    tokens/s: route + schedule over the whole batch; dispatch + FFN of every
    row of n_experts experts, taken at evenly spaced ranks of the expert
    sizes; combine of n_comb tokens. tokens/s = 1 / (t_route_schedule / tokens
    + k * t_row + t_combine_per_token), each term measured.
    threads: run the oracle on that many host threads (default: all cores)."""
    import oracle

    all_cores = oracle.num_threads()
    if threads is None:
        return _oracle_sample(oracle, w, lg, x_cpu, W_dev, n_experts, n_comb, all_cores)
    oracle.set_num_threads(threads)
    try:
        return _oracle_sample(oracle, w, lg, x_cpu, W_dev, n_experts, n_comb, threads)
    finally:
        oracle.set_num_threads(all_cores)


def _oracle_sample(oracle, w, lg, x_cpu, W_dev, n_experts, n_comb, cores):
    import numpy as np
    import torch

    t0 = time.perf_counter()
    ids, g32, g64 = oracle.route_topk(lg, w.k)
    s = oracle.schedule(ids.reshape(w.P, w.N, w.k), w.P, w.N, w.k, w.E, w.pad)
    t_rs = time.perf_counter() - t0
    counts = s["counts"].sum(1)
    order = np.argsort(-counts, kind="stable")
    used = order[counts[order] > 0]
    n_experts = min(n_experts, len(used))
    pick = used[np.linspace(0, len(used) - 1, n_experts).round().astype(int)]
    rows = np.concatenate([np.arange(s["offsets"][e], s["offsets"][e] + counts[e]) for e in pick])
    ex = oracle.expert_of_rows(s["offsets"], rows)
    to_bits = lambda t: t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    Wh = tuple({int(e): to_bits(W[int(e)]) for e in pick} for W in W_dev)
    xb = to_bits(x_cpu)
    t1 = time.perf_counter()
    xg = oracle.dispatch_rows(xb, w.N, s["phi"], rows)
    _, y = oracle.ffn_rows(xg, ex, *Wh, H=w.H, I=w.I)
    t_ffn = time.perf_counter() - t1
    t_row = t_ffn / len(rows)
    n_comb = min(n_comb, w.n_tokens)
    sel = np.random.default_rng(0).integers(0, len(rows), size=(n_comb, w.k))
    t2 = time.perf_counter()
    oracle.combine_f64(y, sel, g64[:n_comb], w.k)
    t_comb = (time.perf_counter() - t2) / n_comb
    per_token = t_rs / w.n_tokens + w.k * t_row + t_comb
    sample = (f"route+schedule over all {w.n_tokens} tokens ({t_rs:.2f} s); dispatch+FFN of all "
              f"{len(rows)} rows of {n_experts} experts at evenly spaced size ranks ({t_ffn:.2f} s); "
              f"combine of {n_comb} tokens; tokens/s = 1/(t_route_sched/{w.n_tokens} + "
              f"{w.k}*t_row + t_combine), extrapolated from the sample")
    return dict(value=1.0 / per_token, cores=cores, sample=sample,
                seconds=t_rs + t_ffn + t_comb * n_comb)


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    import torch

    from combine_top_route_counting_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    lg, x = inputs.make_logits(w), inputs.make_x(w)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    W = inputs.make_weights(w, device=dev)
    vals, secs = [], []
    last = None
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w, lg, x, W, n_experts=1, n_comb=64)
        if i >= args.warmup:
            vals.append(r["value"])
            secs.append(r["seconds"])
        last = r
    value = statistics.median(vals)
    step_s = statistics.median(secs)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * step_s, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w),
                   "note": "CPU oracle (plain C++/OpenMP, fp64). Each step is a bounded sample "
                           "of the workload (route + schedule of every token, dispatch + FFN of "
                           "one expert's rows, combine of 64 tokens); ms_per_step is the "
                           "sample's measured time and value the throughput it extrapolates to",
                   "tokens_per_step_equivalent": value * step_s},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def assemble_line(args, w, world, ms, stage_ms, launches, e2e, e2e_mb, mb, mb_row, mx, bwd,
                  rows_used, peaks, mxl=None):
    """The bench's JSON line (without clocks and cpu_baseline) from the measured
    times: ms for args.steps layer steps, stage_ms {stage: ms}, and the
    optional e2e / minibatch / MXFP8 / backward legs (None when not run)."""
    tokens = w.n_tokens * world * args.steps
    value = tokens / (ms / 1e3)
    work = algorithmic_work(w, rows_used, w.n_routes)
    stages = stage_rooflines(stage_ms, work, peaks, dispatch_fused(w))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_desc(w), "tokens_per_step_per_gpu": w.n_tokens,
                   "minibatch_tokens": mb or w.N, "parallelism": f"replicas x{world}",
                   "rows_padded": rows_used,
                   "l2": "inputs larger than L2: 33.8 GB of expert weights and 14 GB of "
                         "fp32 expert outputs stream through HBM every step",
                   "weights": "random-init bf16 N(0,0.02)"},
    }
    if stage_ms:
        line["phi_build_us"] = stage_ms["schedule"] * 1e3
        g1 = stages["ffn_gemm1"]
        line["roofline"] = {
            "kernel": "ffn_gemm_kernel<0> (GEMM1 + SwiGLU)", "bound": "tensor",
            "achieved": g1["tflops"], "peak": peaks["bf16"], "unit": "TFLOP/s",
            "frac": g1["tflops"] / peaks["bf16"],
            "peak_note": f"dense bf16, burst, of {peaks['source']} (the conservative figure; "
                         "the kernel runs inside a ~1 s loop under the power cap, where the "
                         "sustained figure also applies)",
            "peak_sustained": peaks["bf16_sus"], "frac_sustained": g1["tflops"] / peaks["bf16_sus"],
            "traffic": gemm1_traffic(w.n_routes),
        }
        line["stages"] = stages
    line["gpu_launches"] = launches
    if e2e:
        line["e2e"] = {"value": w.n_tokens * world * args.e2e_steps / (e2e["ms"] / 1e3),
                       "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d"],
                       "d2h_bytes_per_step": e2e["d2h"],
                       "api": "moe_layer_forward_host_async (pinned host logits/x/out; "
                              "the output copy completes on an event, off the compute "
                              "stream)",
                       "transfer_minibatch_tokens": e2e_mb or w.N, "steps": args.e2e_steps,
                       "ms_per_step": e2e["ms"] / args.e2e_steps}
    if mb_row is not None:
        line["minibatch_row"] = {"minibatch_tokens": w.minibatch,
                                 "ms_per_step": mb_row / args.steps,
                                 "value": w.n_tokens * world * args.steps / (mb_row / 1e3),
                                 "unit": "tokens/s"}
    if mx:
        mbytes = w.n_routes * w.H * 2 + mx["rows"] * (w.H + w.H // 32)
        gbs = mbytes / (mx["ms"] / 1e3) / 1e9
        line["mxfp8"] = {"dispatch_mxfp8": {"ms": mx["ms"], "bytes": mbytes, "gbs": gbs,
                                            "frac_hbm": gbs / peaks["hbm"]},
                         "note": "pull dispatch with the MX (E4M3, E8M0 per 32) "
                                 "quantisation fused"}
    if mxl:
        mst = stage_rooflines(mxl["stage_ms"], mx_layer_work(w, rows_used), peaks,
                              fused_dispatch=True)
        line["mxfp8_layer"] = {
            "value": w.n_tokens * world * args.steps / (mxl["ms"] / 1e3), "unit": "tokens/s",
            "ms_per_step": mxl["ms"] / args.steps, "steps": args.steps,
            "api": "moe_layer_forward_mxfp8 (weights quantised once, outside the timed region)",
            "stages": mst,
            "peak_note": f"fp8 peak = 2 x dense bf16 sustained of {peaks['source']} "
                         "(the nominal fp8/bf16 ratio)",
        }
    if bwd:
        bst = stage_rooflines(bwd["stages"], backward_work(w, rows_used), peaks)
        top = max(bst, key=lambda n: bst[n]["ms"])
        tokens_b = w.n_tokens * world * args.bwd_steps
        line["backward"] = {
            "value": w.n_tokens * world / (bwd["bwd_ms"] / 1e3), "unit": "tokens/s",
            "ms_per_step": bwd["bwd_ms"],
            "train_step": {"value": tokens_b / (bwd["train_ms"] / 1e3), "unit": "tokens/s",
                           "ms_per_step": bwd["train_ms"] / args.bwd_steps,
                           "what": "moe_layer_forward_train + moe_layer_backward",
                           "gpu_launches": bwd["launches"] // args.bwd_steps},
            "steps": args.bwd_steps, "warmup": args.warmup,
            "stages": bst,
            "roofline": {"kernel": top, "bound": "tensor" if "tflops" in bst[top] else "hbm",
                         "achieved": bst[top].get("tflops", bst[top].get("gbs")),
                         "peak": peaks["bf16_sus"] if "tflops" in bst[top] else peaks["hbm"],
                         "unit": "TFLOP/s" if "tflops" in bst[top] else "GB/s",
                         "frac": bst[top].get("frac_bf16", bst[top].get("frac_hbm")),
                         "traffic": wgrad13_traffic(w.n_routes) if top == "wgrad_w13" else None},
            "dout": "bf16 N(0,1), seeded",
        }
    return line


def run_ours(args):
    import torch

    from combine_top_route_counting_b200 import inputs, moe

    rank, world, local_rank = env_rank()
    if world != args.gpus:
        print(f"bench: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ready = init_dist(world, local_rank)
    moe.load()

    w = inputs.WORKLOADS[args.workload]
    sh = moe.shape(**w.shape())
    lg_cpu, x_cpu = inputs.make_logits(w), inputs.make_x(w)
    W = inputs.make_weights(w, device=dev)
    lg, x = lg_cpu.to(dev), x_cpu.to(dev)
    ws = torch.empty(moe.layer_workspace_bytes(sh), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=dev)
    mb = args.minibatch

    def step(events=None):
        moe.moe_layer_forward(lg, x, *W, out, ws, st, sh, minibatch_tokens=mb, stage_events=events)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.N_STAGE_EVENTS)]
          for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record()  # creates the event
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} during warm-up")
    if ready:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    n0 = moe.launch_count()
    t_start.record()
    for i in range(args.steps):
        step(ev[i] if mb == 0 else None)
    t_end.record()
    torch.cuda.synchronize()
    launches = moe.launch_count() - n0
    if ready:
        torch.distributed.barrier()
    ms = t_start.elapsed_time(t_end)

    stage_ms = {}
    if mb == 0:
        for s_i, name in enumerate(moe.STAGES):
            stage_ms[name] = statistics.mean(ev[i][s_i].elapsed_time(ev[i][s_i + 1])
                                             for i in range(args.steps))

    # the same layer sliced at the workload's transfer minibatch (device-resident)
    mb_row = None
    if w.minibatch and not args.no_minibatch_row and mb == 0:
        t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            moe.moe_layer_forward(lg, x, *W, out, ws, st, sh, minibatch_tokens=w.minibatch)
        t0e.record()
        for _ in range(args.steps):
            moe.moe_layer_forward(lg, x, *W, out, ws, st, sh, minibatch_tokens=w.minibatch)
        t1e.record()
        torch.cuda.synchronize()
        mb_row = t0e.elapsed_time(t1e)

    # the MXFP8 building block: the pull dispatch with the MX quantisation fused
    mx = None
    if not args.no_mxfp8 and mb == 0:
        ids_mx = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=dev)
        gates_mx = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=dev)
        moe.moe_route_topk(lg, ids_mx, gates_mx, sh)
        bmx = moe.alloc_schedule_outputs(sh, device=dev)
        moe.moe_schedule(ids_mx, bmx["phi"], bmx["offsets"], bmx["counts"], bmx["route_row"],
                         bmx["ws"], bmx["dev_status"], sh)
        rm = moe.rows_max(sh)
        xq = torch.empty((rm, w.H), dtype=torch.uint8, device=dev)
        xs = torch.empty((rm, w.H // 32), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            moe.moe_dispatch_mxfp8(x, bmx["phi"], bmx["offsets"], xq, xs, bmx["dev_status"], sh)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record()
        for _ in range(args.steps):
            moe.moe_dispatch_mxfp8(x, bmx["phi"], bmx["offsets"], xq, xs, bmx["dev_status"], sh)
        m1.record()
        torch.cuda.synchronize()
        if int(bmx["dev_status"].item()) != 0:
            raise RuntimeError(f"device status {int(bmx['dev_status'].item())} in the MX dispatch")
        mx = dict(ms=m0.elapsed_time(m1) / args.steps, rows=int(bmx["offsets"][-1].item()))
        del xq, xs, bmx

    # the MXFP8 layer: block-scaled expert GEMMs on weights quantised once
    mxl = None
    if not args.no_mxfp8_layer and mb == 0:
        Wq = []
        for Wt in W:
            E_, K_, N_ = Wt.shape
            q = torch.empty((E_, N_, K_), dtype=torch.uint8, device=dev)
            sc = torch.empty((E_ * N_ * K_ // 32,), dtype=torch.uint8, device=dev)
            moe.moe_mx_quantize_weights(Wt, q, sc)
            Wq += [q, sc]
        evm = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.N_STAGE_EVENTS)]
               for _ in range(args.steps)]
        for row in evm:
            for e in row:
                e.record()  # creates the event
        for _ in range(args.warmup):
            moe.moe_layer_forward_mxfp8(lg, x, *Wq, out, ws, st, sh)
        torch.cuda.synchronize()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record()
        for i in range(args.steps):
            moe.moe_layer_forward_mxfp8(lg, x, *Wq, out, ws, st, sh, stage_events=evm[i])
        m1.record()
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} in the MXFP8 layer")
        mxl = dict(ms=m0.elapsed_time(m1),
                   stage_ms={name: statistics.mean(evm[i][s_i].elapsed_time(evm[i][s_i + 1])
                                                   for i in range(args.steps))
                             for s_i, name in enumerate(moe.STAGES)})
        del Wq

    # the other workloads (Phi on the scheduler workload, the Zipf, mid and
    # tiny layers), same device, same run
    cfgs = None
    if not args.no_configs and mb == 0 and w.name == "kimi":
        cfgs = time_configs(moe, dev, W, x, ws, st, args.steps, args.warmup, load_peaks())

    # end to end through the host-buffer entry: H2D of logits and x, the layer,
    # D2H of out; each call's input copy overlaps the previous call's compute
    # and its output copy the next call's compute (the async-output entry)
    e2e = None
    e2e_mb = args.e2e_minibatch if args.e2e_minibatch >= 0 else w.minibatch
    if not args.no_e2e:
        del ws
        torch.cuda.empty_cache()
        wsh = torch.empty(moe.layer_host_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        lg_h, x_h = lg_cpu.pin_memory(), x_cpu.pin_memory()
        out_h = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16).pin_memory()
        out_ready = [torch.cuda.Event() for _ in range(2)]
        for r in out_ready:
            r.record()  # creates the event

        def host_step(i):
            moe.moe_layer_forward_host_async(lg_h, x_h, *W, out_h, wsh, st, sh, out_ready[i % 2],
                                             minibatch_tokens=e2e_mb)

        for i in range(2):
            host_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        chk = 0.0
        e0.record()
        for i in range(args.e2e_steps):
            host_step(i)
        # the timed region ends when the last step's output is in host memory
        torch.cuda.current_stream().wait_event(out_ready[(args.e2e_steps - 1) % 2])
        e1.record()
        torch.cuda.synchronize()
        chk += float(out_h[0, :8].float().sum())  # the host reads the result
        e2e_ms = e0.elapsed_time(e1)
        e2e = dict(ms=e2e_ms, h2d=lg_cpu.numel() * 4 + x_cpu.numel() * 2,
                   d2h=out_h.numel() * 2, chk=chk)
        del wsh
    else:
        del ws
    torch.cuda.empty_cache()

    # the training step: forward keeping the activations, then the backward
    bwd = None
    if not args.no_backward and moe.train_workspace_bytes(sh) > 0:
        wst = torch.empty(moe.train_workspace_bytes(sh), dtype=torch.uint8, device=dev)
        dout = inputs.make_dout(w, device=dev)
        dx = torch.empty((w.n_tokens, w.H), dtype=torch.bfloat16, device=dev)
        dlg = torch.empty((w.n_tokens, w.E), dtype=torch.float32, device=dev)
        dW1 = torch.empty((w.E, w.H, w.I), dtype=torch.float32, device=dev)
        dW3 = torch.empty_like(dW1)
        dW2 = torch.empty((w.E, w.I, w.H), dtype=torch.float32, device=dev)
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(moe.N_BWD_EVENTS)]
               for _ in range(args.bwd_steps)]
        for row in bev:
            for e in row:
                e.record()

        def train_step(events=None):
            moe.moe_layer_forward_train(lg, x, *W, out, wst, st, sh)
            moe.moe_layer_backward(dout, *W, dx, dlg, dW1, dW3, dW2, wst, st, sh,
                                   stage_events=events)

        for _ in range(args.warmup):
            train_step()
        torch.cuda.synchronize()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nb0 = moe.launch_count()
        b0.record()
        for i in range(args.bwd_steps):
            train_step(bev[i])
        b1.record()
        torch.cuda.synchronize()
        bwd = dict(train_ms=b0.elapsed_time(b1), launches=moe.launch_count() - nb0,
                   bwd_ms=statistics.mean(bev[i][0].elapsed_time(bev[i][-1])
                                          for i in range(args.bwd_steps)),
                   stages={name: statistics.mean(bev[i][j].elapsed_time(bev[i][j + 1])
                                                 for i in range(args.bwd_steps))
                           for j, name in enumerate(moe.BWD_STAGES)})
        del wst, dW1, dW3, dW2
        torch.cuda.empty_cache()
    clk = clocks.stop()

    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())}")

    names = list(stage_ms)
    bnames = list(bwd["stages"]) if bwd else []
    vec = ([ms] + [stage_ms[n] for n in names] + ([e2e["ms"]] if e2e else []) +
           ([mb_row] if mb_row is not None else []) +
           ([bwd["train_ms"], bwd["bwd_ms"]] + [bwd["stages"][n] for n in bnames] if bwd else []) +
           ([mx["ms"]] if mx else []) +
           ([mxl["ms"]] + [mxl["stage_ms"][n] for n in moe.STAGES] if mxl else []))
    vec = reduce_max(vec, ready, device=dev)
    if mxl:
        mvals = vec[-(1 + len(moe.STAGES)):]
        vec = vec[:-(1 + len(moe.STAGES))]
        mxl["ms"] = mvals[0]
        mxl["stage_ms"] = dict(zip(moe.STAGES, mvals[1:]))
    if mx:
        mx["ms"] = vec.pop()
    if bwd:
        nb = 2 + len(bnames)
        bvec, vec = vec[-nb:], vec[:-nb]
        bwd["train_ms"], bwd["bwd_ms"] = bvec[0], bvec[1]
        bwd["stages"] = dict(zip(bnames, bvec[2:]))
    ms = vec[0]
    stage_ms = dict(zip(names, vec[1:1 + len(names)]))
    if mb_row is not None:
        mb_row = vec.pop()
    if e2e:
        e2e["ms"] = vec[-1]

    if rank == 0:
        peaks = load_peaks()
        rows_used = schedule_rows(moe, w, sh, lg)
        line = assemble_line(args, w, world, ms, stage_ms, launches, e2e, e2e_mb, mb, mb_row, mx,
                             bwd, rows_used, peaks, mxl=mxl)
        line["clocks"] = clk
        if cfgs:
            line["configs"] = cfgs
        if world == 1 and not args.no_cpu_baseline:
            r = oracle_sample(w, lg_cpu, x_cpu, W, n_experts=args.cpu_experts)
            line["cpu_baseline"] = {"value": r["value"], "unit": "tokens/s", "cores": r["cores"],
                                    "kind": "oracle", "sample": r["sample"],
                                    "seconds": r["seconds"]}
            if w.name in ("tiny", "mid"):  # the small configs also on one host core
                r1 = oracle_sample(w, lg_cpu, x_cpu, W, n_experts=args.cpu_experts, threads=1)
                line["cpu_baseline"]["one_core"] = {"value": r1["value"], "unit": "tokens/s",
                                                    "cores": 1, "sample": r1["sample"]}
        print(json.dumps(line), flush=True)
    if ready:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def schedule_rows(moe, w, sh, lg) -> int:
    """Padded rows the schedule uses for this batch (offsets[E]), via the library."""
    import torch
    ids = torch.empty((w.n_tokens, w.k), dtype=torch.int32, device=lg.device)
    gates = torch.empty((w.n_tokens, w.k), dtype=torch.float32, device=lg.device)
    moe.moe_route_topk(lg, ids, gates, sh)
    b = moe.alloc_schedule_outputs(sh, device=lg.device)
    moe.moe_schedule(ids, b["phi"], b["offsets"], b["counts"], b["route_row"], b["ws"],
                     b["dev_status"], sh)
    return int(b["offsets"][-1].item())


def kernel_source_hash(files=("expert_ffn.cu", "persistent_gemm.cuh", "sm100.cuh")) -> str:
    """sha256 of kernel sources (by default the forward FFN's) with comments,
    trailing blanks and empty lines removed: edits to comments keep a recorded
    measurement valid, any change to the code invalidates it."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        src = open(os.path.join(ROOT, "combine_top_route_counting_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in src.splitlines()]
        h.update("\n".join(ln for ln in lines if ln.strip()).encode())
    return h.hexdigest()


def _recorded_traffic(name: str, files, n_routes: int):
    """DRAM bytes per launch from a committed ncu summary (profiles/<name>),
    scaled to this launch by routes; None when the summary is missing or the
    kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    kv = {}
    for ln in open(path):
        if ":" in ln and not ln.startswith("#"):
            a, b = ln.split(":", 1)
            kv[a.strip()] = b.strip()
    if kv.get("kernel_source_sha256") != kernel_source_hash(files):
        return None
    try:
        return float(kv["dram_bytes_per_route"]) * n_routes
    except (KeyError, ValueError):
        return None


def gemm1_traffic(n_routes: int):
    """DRAM bytes of one GEMM1 launch (profiles/ffn_gemm1_traffic.txt)."""
    return _recorded_traffic("ffn_gemm1_traffic.txt",
                             ("expert_ffn.cu", "persistent_gemm.cuh", "sm100.cuh"), n_routes)


def wgrad13_traffic(n_routes: int):
    """DRAM bytes of one dW1|dW3 launch (profiles/ffn_wgrad13_traffic.txt)."""
    return _recorded_traffic("ffn_wgrad13_traffic.txt",
                             ("expert_ffn_bwd.cu", "persistent_gemm.cuh", "sm100.cuh"), n_routes)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="kimi")
    ap.add_argument("--minibatch", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the host-buffer leg (0: the same as --steps)")
    ap.add_argument("--e2e-minibatch", type=int, default=0,
                    help="transfer slice of the host-buffer leg (0: whole batch; "
                         "-1: the workload's transfer minibatch)")
    ap.add_argument("--no-minibatch-row", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-mxfp8", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (scheduler, zipf, mid, tiny)")
    ap.add_argument("--no-mxfp8-layer", action="store_true",
                    help="skip the moe_layer_forward_mxfp8 leg (block-scaled expert GEMMs)")
    ap.add_argument("--bwd-steps", type=int, default=10)
    ap.add_argument("--cpu-experts", type=int, default=8,
                    help="experts whose rows the CPU baseline runs through the oracle's FFN")
    args = ap.parse_args(argv)
    if args.e2e_steps <= 0:
        args.e2e_steps = args.steps
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
