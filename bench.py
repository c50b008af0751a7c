#!/usr/bin/env python
"""Benchmark of the MoE token shuffle (route -> dispatch -> grouped SwiGLU FFN -> combine) on B200.

One step = one pass of the whole path over one batch of synthetic tokens (all four C-ABI calls on
one stream), inputs and weights already resident in HBM.  Prints one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload skewed] [--also train,finegrained]
                    [--impl ours|reference]

The headline workload (default ``skewed``: T=16384, H=7168, E=128, top-2, capacity 320, the largest
configuration that fits one GPU) gives ``value``; the ``--also`` workloads are timed the same way
in the same run and reported under ``workloads``.

Multi-GPU (torchrun): every rank runs an independent replica of the workload (its own batch of T
tokens, emulated expert-parallel ranks inside each GPU), no data-path collective; the step time is
the max over ranks and ``value`` counts the tokens of all ranks ("weak" scaling).

The line's ``expert_parallel`` object times the expert-parallel step (``MoeEP``, peer-memory mode)
on the train shapes over the run's ranks: every rank owns E/N experts and its own T tokens, rows
cross the ranks through the fused exchange kernel (at N = 1, a one-rank NCCL group: the exchange
is a local move and the number shows the cost of the expert-parallel machinery).  With N > 1 it
runs only with ``--ep``.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "dispatch+FFN+combine tokens/s and shuffle HBM GB/s (% of roofline) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Nominal B200 figures, for the secondary fractions: HBM3e about 8 TB/s, dense bf16 2.25 PFLOP/s.
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
L2_FLUSH_BYTES = mi.l2_flush_bytes()
# DRAM read + write bytes per call of the FFN stage (fused_ffn_kernel, plus dequant_fp8_kernel for
# the FP8 payload): ncu dram__bytes_read.sum + dram__bytes_write.sum of the kernels as built from
# this tree.  An entry is None (or absent) once either kernel has changed since its counters were
# taken.  New counters come from small captures (one kernel, a few launches, a few GB on the
# device), scaled to a full call by the units processed, never from a capture of a full-size run.
FFN_TRAFFIC: dict = {}


# ---------------------------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while the benchmark runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9:
                    continue
                try:
                    sm.append(float(c[1]))
                    mx = float(c[2])
                    power.append(float(c[3]))
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------------------------
def max_over_ranks(local_ms: float, device) -> float:
    """The slowest rank's time (all ranks call this together; a single process returns its own)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(local_ms)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(local_ms: float, tokens_per_rank: int, steps: int, device) -> dict:
    """Whole-job throughput of independent replicas: every rank's tokens over the slowest rank's
    time (weak scaling)."""
    import torch.distributed as dist
    world = dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1
    ms = max_over_ranks(local_ms, device)
    return {"value": world * tokens_per_rank * steps / (ms * 1e-3), "ms_per_step": ms / steps,
            "total_ms": ms, "n_ranks": world}


def algorithmic(w, S: int, active_experts: int):
    """Algorithmic bytes / flops per step of each stage: what the method must move or compute.

    The FFN's algorithmic bytes are the active experts' weights, its input rows read once (bf16, or
    for the FP8 payload the e4m3 codes and fp32 scales as dispatched) and its output rows written
    once.  Traffic that this implementation adds on top (the bf16 intermediate h written and read
    back between the two GEMMs; for FP8, the dequantisation pass's bf16 rows, written once and read
    by the GEMM instead of the codes) is ``ffn_impl_overhead`` and is not counted as achieved work.
    """
    fp8 = w.payload == "fp8"
    b = 1 if fp8 else 2
    scales = S * (w.H // 128) * 4 if fp8 else 0
    route = w.T * w.E * 4 + w.T * w.k * 8 + w.E * 4
    dispatch = (w.T * w.H * 2 + S * w.H * b + scales
                + w.T * w.k * 4 * 3 + S * 4 + (w.E * 2 + 1 + w.R + 1) * 4)
    weights = active_experts * 3 * w.H * w.F * 2
    ffn_bytes = weights + S * w.H * b + scales + S * w.H * 2
    overhead = 2 * S * w.F * 2 + (4 * S * w.H if fp8 else 0)
    ffn_flops = 6 * S * w.H * w.F
    combine = S * w.H * 2 + w.T * w.k * 8 + w.T * w.H * 2
    return dict(route=route, dispatch=dispatch, ffn_bytes=ffn_bytes, ffn_weight_bytes=weights,
                ffn_impl_overhead=overhead, ffn_flops=ffn_flops, combine=combine)


def ffn_mma_rows(n: int) -> int:
    """Rows the FFN's MMAs compute for an expert of n rows: a 128-row tile up to 64 rows (one
    CTA), pairs of 128-row blocks (256 rows per 2-CTA tile) beyond."""
    if n <= 0:
        return 0
    if n <= 64:
        return 128
    return -(-n // 256) * 256


def cpu_baseline_run(w, d_cpu, budget_s: float = 12.0, n_tokens: int | None = None):
    """Oracle pipeline on a bounded token sample (the first n tokens).  Returns (tokens/s, info)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import moe

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    wg, wu, wd = bits(d_cpu["w_gate"]), bits(d_cpu["w_up"]), bits(d_cpu["w_down"])
    logits, x = d_cpu["logits"].numpy(), bits(d_cpu["x"])
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)

    def run(n):
        idx, wt, _ = moe.route(logits[:n], w.k)
        plan = moe.dispatch_plan(idx, w.E, w.R, cap)
        send, sc = moe.dispatch_payload(x[:n], plan, w.payload == "fp8")
        xin = moe.ffn_inputs(send, sc, w.payload == "fp8")
        _, y_e = moe.expert_ffn(xin, plan["expert_offsets"], wg, wu, wd)
        moe.combine(y_e, plan["slot_row"], wt, n, w.H)

    if n_tokens is None:
        n, spent, t = 1, 0.0, 0.0
        while True:
            t0 = time.perf_counter()
            run(n)
            t = time.perf_counter() - t0
            spent += t
            if t > budget_s / 4 or n >= w.T or spent > budget_s:
                break
            n = min(w.T, n * 2)
    else:
        n = min(n_tokens, w.T)
        t0 = time.perf_counter()
        run(n)
        t = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return n / t, {"cores": threads, "tokens": n, "seconds": t}


# ---------------------------------------------------------------------------------------------
def run_reference(args, w, rank: int):
    """The oracle, as it stands, timed on the host cores on bounded token samples of the workload."""
    if rank != 0:
        return
    # the same inputs as the GPU arm's rank 0 (drawn by the same generator on the GPU when there is
    # one), copied to host memory; the oracle then runs on the host cores only
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = {k: v.cpu() for k, v in mi.make_inputs(w, seed=0, device=gen_dev).items()}
    if gen_dev == "cuda":
        torch.cuda.empty_cache()
    budget = 150.0
    # size each step so that warm-up + timed steps stay within a few minutes
    _, info = cpu_baseline_run(w, d, n_tokens=1)
    per_token = max(info["seconds"], 1e-3)
    n = max(1, min(w.T, int(budget / max(args.steps + args.warmup, 1) / per_token)))
    for _ in range(args.warmup):
        cpu_baseline_run(w, d, n_tokens=n)
    total, toks = 0.0, 0
    for _ in range(args.steps):
        _, inf = cpu_baseline_run(w, d, n_tokens=n)
        total += inf["seconds"]
        toks += inf["tokens"]
    value = toks / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle",
                         "sample": f"first {n} tokens of the workload per step (route, dispatch, "
                                   f"SwiGLU FFN on their rows, combine)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, args):
    import math
    cap = math.ceil(w.capacity_factor * w.T * w.k / w.E) if w.capacity_factor else 0
    return {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "k": w.k, "R": w.R, "F": w.F,
            "payload": w.payload, "capacity": cap, "bias": w.bias,
            "parallelism": f"replicas x{args.gpus} (ranks emulated inside each GPU)",
            "l2": ("flushed before every timed step: 256 MB written" +
                   (", then another 256 MB buffer read (its clean lines evict the written ones, so "
                    "no flush data is written back inside the timed region)"
                    if args.flush == "write-read" else ""))}


# ---------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="skewed", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--also", default="train,finegrained",
                    help="comma-separated workloads timed after the headline one, reported under "
                         "'workloads' in the same line ('' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush", default="write-read", choices=["write", "write-read"])
    ap.add_argument("--no-w8", action="store_true",
                    help="skip the extra timing of the step with FP8 gate / up weights")
    ap.add_argument("--e2e-eager", action="store_true",
                    help="end-to-end loop calls forward eagerly instead of replaying CUDA graphs")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel step across the ranks when N > 1 (always at N = 1)")
    ap.add_argument("--no-ep", action="store_true", help="skip the expert-parallel timing")
    ap.add_argument("--ep-workload", default="train", choices=sorted(mi.WORKLOADS))
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = mi.get(args.workload)

    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    import datetime
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    also = [n for n in args.also.split(",") if n and n != w.name]
    for n in also:
        if n not in mi.WORKLOADS:
            raise SystemExit(f"unknown workload {n}")

    sampler = ClockSampler(local)
    sampler.start()
    head = measure(w, args, dev, world, rank, e2e=True)
    extra = {n: measure(mi.get(n), args, dev, world, rank, e2e=False) for n in also}
    ep = None
    if not args.no_ep and (world == 1 or args.ep):
        ep = measure_ep(mi.get(args.ep_workload), args, dev, world, rank)
    clocks = sampler.stop()

    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8+bf16" if w.payload == "fp8" else "bf16",
        "data": "synthetic (seeded; random-init expert weights N(0,0.02))",
        "config": config_of(w, args),
        "roofline": head["roofline"],
        "stages": head["stages"],
        "stages_note": "per-stage CUDA events on breakdown steps interleaved with the metric steps "
                       "(each event ends the programmatic launch overlap around it); value and "
                       "ms_per_step come from the metric steps' boundary events only; frac = of "
                       "the measured HBM copy rate, frac_nominal = of 8 TB/s",
        "kept_rows": head["kept_rows"], "active_experts": head["active_experts"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": clocks,
        "fp8_weights": head.get("fp8_weights"),
        "backward": head.get("backward"),
        "workloads": {n: {k: v for k, v in r.items() if k != "e2e"} for n, r in extra.items()},
        "workloads_note": "the other large workloads, each timed the same way in the same run "
                          "(own warm-up, L2 flush, metric and breakdown steps); gpu_launches counts "
                          "the headline workload's timed region only",
        "expert_parallel": ep,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        d_cpu = {k: v.cpu() for k, v in mi.make_inputs(w, seed=rank, device=str(dev)).items()}
        v, info = cpu_baseline_run(w, d_cpu)
        line["cpu_baseline"] = {
            "value": v, "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
            "sample": f"first {info['tokens']} tokens of the workload (route, dispatch, SwiGLU FFN "
                      f"on their rows, combine), {info['seconds']:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure(w, args, dev, world: int, rank: int, e2e: bool) -> dict:
    """Time K steps of workload ``w`` on this GPU (plus, with ``e2e``, the end-to-end loop through
    the public API) and return its throughput, stage breakdown and FFN roofline."""
    import math
    import torch.distributed as dist
    from combine_moe_route_10_b200 import MoeShuffle

    d = mi.make_inputs(w, seed=rank, device=str(dev))
    cap_rows = math.ceil(w.capacity_factor * w.T * w.k / w.E) if w.capacity_factor else 0
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap_rows, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_rd = (torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
                if args.flush == "write-read" else None)
    stream = torch.cuda.current_stream(dev)

    def flush_l2():
        flush.fill_(1)
        if flush_rd is not None:
            flush_rd.sum()  # evicts the dirty lines of the write, leaving clean ones

    def step():
        m.route(d["logits"])
        m.dispatch(d["x"])
        m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"])
        m.combine()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    st = m.status()
    if st != 0:
        raise SystemExit(f"{w.name}: device status {st} after warm-up")
    S = int(m.expert_offsets[w.E].item())
    active = int((m.expert_counts > 0).sum().item())
    # rows the FFN's MMAs compute: a 2-CTA tile covers 256 of an expert's rows (experts of more
    # than 64 rows), a 1-CTA tile 128 (the others); the padding is work the tensor cores do
    counts = m.expert_counts.cpu().tolist()
    padded_rows = sum(ffn_mma_rows(int(c)) for c in counts)

    # Timed region: K metric steps interleaved with K breakdown steps, so both see the same clocks.
    # Metric steps (value, ms_per_step) have events only at step boundaries, so consecutive kernels
    # keep their programmatic-launch overlap as in production use.  Breakdown steps (stage times,
    # FFN roofline) have an event between every two stages; each event ends the overlap of the two
    # launches around it, so their stage times are slightly pessimistic.
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    n_ev = 5
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        step_ev[i][0].record(stream)
        step()
        step_ev[i][1].record(stream)
        flush_l2()
        e = evs[i]
        e[0].record(stream)
        m.route(d["logits"])
        e[1].record(stream)
        m.dispatch(d["x"])
        e[2].record(stream)
        m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"])
        e[3].record(stream)
        m.combine()
        e[4].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    agg = aggregate(sum(a.elapsed_time(b) for a, b in step_ev), w.T, args.steps, dev)
    stage_ms = [[e[j].elapsed_time(e[j + 1]) for j in range(n_ev - 1)] for e in evs]
    mean_stage = [sum(s[j] for s in stage_ms) / args.steps for j in range(n_ev - 1)]

    e2e_out = None
    if e2e:
        e2e_out = e2e_run(w, m, d, args, dev, world, stream)
    st = m.status()
    if st != 0:
        raise SystemExit(f"{w.name}: device status {st} after timing")

    pk, pk_src = peaks()
    alg = algorithmic(w, S, active)
    t_route, t_disp, t_ffn, t_comb = mean_stage
    hbm = pk["hbm_gbs"]
    ffn_t_hbm = alg["ffn_bytes"] / (hbm * 1e9)
    ffn_t_tc = alg["ffn_flops"] / (pk["bf16_tflops_sustained"] * 1e12)
    if ffn_t_hbm >= ffn_t_tc:
        ach = alg["ffn_bytes"] / (t_ffn * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "frac_nominal": ach / NOMINAL["hbm_gbs"]}
    else:
        ach = alg["ffn_flops"] / (t_ffn * 1e-3) / 1e12
        p = pk["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": ach, "peak": p, "unit": "TFLOP/s", "frac": ach / p,
                "frac_burst": ach / pk["bf16_tflops"], "frac_nominal": ach / NOMINAL["bf16_tflops"]}
    roof.update({
        "kernel": ("ffn_pair_kernel (2-CTA tiles, experts of > 64 rows) + ffn_single_kernel "
                   "(experts of <= 64 rows): GEMM-1 gate|up + SwiGLU and GEMM-2 down in each"
                   + (" + dequant_fp8_kernel" if w.payload == "fp8" else "") + " = moe_expert_ffn"),
        "traffic": FFN_TRAFFIC.get(w.name), "peak_source": pk_src,
        "algorithmic_bytes": alg["ffn_bytes"], "algorithmic_flops": alg["ffn_flops"],
        "impl_overhead_bytes": alg["ffn_impl_overhead"],
        "frac_of_max_time_bound": max(ffn_t_hbm, ffn_t_tc) / (t_ffn * 1e-3),
        # the bound with the MMAs' padded rows: what the tile shapes leave the kernel to reach
        "padded_rows": padded_rows,
        "frac_of_padded_bound": max(ffn_t_hbm, alg["ffn_flops"] * padded_rows / max(S, 1)
                                    / (pk["bf16_tflops_sustained"] * 1e12)) / (t_ffn * 1e-3)})

    def gbs(b, t):
        return b / (t * 1e-3) / 1e9

    def shuffle_stage(b, t):
        return {"ms": t, "GB/s": gbs(b, t), "frac": gbs(b, t) / hbm,
                "frac_nominal": gbs(b, t) / NOMINAL["hbm_gbs"]}

    stages = {
        "route": {"ms": t_route, "GB/s": gbs(alg["route"], t_route)},
        "dispatch": shuffle_stage(alg["dispatch"], t_disp),
        "ffn": {"ms": t_ffn, "TFLOP/s": alg["ffn_flops"] / (t_ffn * 1e-3) / 1e12,
                "GB/s": gbs(alg["ffn_bytes"], t_ffn)},
        "combine": shuffle_stage(alg["combine"], t_comb),
    }
    # route, count + rank_permute (dispatch), the two FFN kernels (+ the FP8 dequantisation), combine
    launches_per_step = 6 + (1 if w.payload == "fp8" else 0)
    out = {"value": agg["value"], "ms_per_step": agg["ms_per_step"], "config": config_of(w, args),
           "roofline": roof, "stages": stages, "kept_rows": S, "active_experts": active,
           "gpu_launches": 2 * launches_per_step * args.steps,  # metric + breakdown steps
           "e2e": e2e_out}
    if not args.no_w8:
        out["fp8_weights"] = measure_w8(w, m, d, args, stream, flush_l2, world, dev, S, active, pk)
    if not args.no_backward:
        out["backward"] = measure_backward(w, m, d, args, stream, flush_l2, world, dev, S, pk)
    del m, d, flush, flush_rd
    torch.cuda.empty_cache()
    return out


def measure_backward(w, m, d, args, stream, flush_l2, world, dev, S, pk) -> dict:
    """The backward of the step (``moe_backward`` after the forward just timed, reusing its routing,
    plan and expert outputs): K steps behind an L2 flush, CUDA events around each call, max over
    ranks.  Tensor work 16 S H F flops (the recompute of g and u, dh, dx_rows and the three weight
    gradients); bytes: the weights read once, the fp32 weight gradients of all E experts written
    once, dy and the expert outputs read and dx written once (the gradient rows the kernels hand
    to each other are this implementation's own traffic)."""
    import torch.distributed as dist
    g = torch.Generator(device=dev).manual_seed(7)
    dy = torch.randn((w.T, w.H), generator=g, device=dev).to(torch.bfloat16)

    def step():
        m.backward(dy, d["logits"], d["w_gate"], d["w_up"], d["w_down"])

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if m.status() != 0:
        raise SystemExit(f"{w.name}: device status after the backward warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for a, b in ev:
        flush_l2()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev) / args.steps
    if m.status() != 0:
        raise SystemExit(f"{w.name}: device status after the backward timing")
    flops = 16.0 * S * w.H * w.F
    bytes_ = (3.0 * w.E * w.H * w.F * (2 + 4)            # weights read, fp32 gradients written
              + w.T * w.H * 2 * 2 + S * w.H * 2 * 2)     # dy, dx; expert outputs, FFN input rows
    t_tc = flops / (pk["bf16_tflops_sustained"] * 1e12)
    t_hbm = bytes_ / (pk["hbm_gbs"] * 1e9)
    tf = flops / (ms * 1e-3) / 1e12
    return {"ms": ms, "tokens_per_s": w.T / (ms * 1e-3), "TFLOP/s": tf,
            "frac_tensor": tf / pk["bf16_tflops_sustained"],
            "GB/s_algorithmic": bytes_ / (ms * 1e-3) / 1e9,
            "bound": "tensor" if t_tc >= t_hbm else "hbm",
            "frac_of_max_time_bound": max(t_tc, t_hbm) / (ms * 1e-3),
            "algorithmic_flops": flops, "algorithmic_bytes": bytes_,
            "kernels": "combine_bwd_kernel, bwd_gemm_kernel<recompute g|u + dh + SwiGLU backward>, "
                       "bwd_gemm_kernel<dx_rows>, bwd_gemm_kernel<dW, TMA-store epilogue>, "
                       "combine_kernel (unit weights) = moe_backward",
            "gpu_launches_per_step": 5}


def measure_ep(w, args, dev, world: int, rank: int) -> dict:
    """The expert-parallel step (peer-memory mode) on workload ``w``'s shapes over this run's ranks:
    rank r owns experts [r*E/N, (r+1)*E/N) and its own T tokens.  K metric steps (events at step
    boundaries, max over ranks) interleaved with K steps that time the pull and push exchange
    kernels; L2 flushed before every step."""
    import datetime
    import socket

    import torch.distributed as dist
    from combine_moe_route_10_b200 import _lib
    from combine_moe_route_10_b200.ep import MoeEP, TorchComm

    own_group = not dist.is_initialized()
    if own_group:
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    try:
        R = dist.get_world_size()
        E_loc = w.E // R
        d = mi.make_ep_inputs(w, R, seed=0, device=str(dev))
        sl = slice(rank * E_loc, (rank + 1) * E_loc)
        logits, x = d["logits"][rank], d["x"][rank]
        wg, wu, wd = (d[k][sl].contiguous() for k in ("w_gate", "w_up", "w_down"))
        del d
        ep = MoeEP(w.T, w.H, w.E, w.k, w.F, comm=TorchComm(symmetric=R > 1), payload=w.payload,
                   mode="p2p", device=dev)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        stream = torch.cuda.current_stream(dev)
        for _ in range(args.warmup):
            flush.fill_(1)
            ep.forward(logits, x, wg, wu, wd)
        torch.cuda.synchronize()
        if ep.status() != 0:
            raise SystemExit(f"expert-parallel {w.name}: device status after warm-up")
        n_recv = int(ep.local_offsets[E_loc].item())
        S = ep.send.shape[0]
        row_b = w.H * ep.send.element_size() + ep.nb * 4
        st = ep.ws_regroup
        step_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                   for _ in range(args.steps)]
        x_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
                for _ in range(args.steps)]
        dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.fill_(1)
            step_ev[i][0].record(stream)
            ep.forward(logits, x, wg, wu, wd)
            step_ev[i][1].record(stream)
            # the two exchange kernels of the step just taken, timed on their own
            flush.fill_(1)
            e = x_ev[i]
            e[0].record(stream)
            _lib.moe_ep_exchange(ep.all_counts, R, w.E, rank, _lib.MOE_EP_PULL, ep.peer_send,
                                 ep.peer_send_scales, S, ep.grouped, ep.grouped_scales, ep.cap,
                                 w.H * ep.send.element_size(), ep.nb * 4, ep.local_offsets, st)
            e[1].record(stream)
            flush.fill_(1)
            e[2].record(stream)
            _lib.moe_ep_exchange(ep.all_counts, R, w.E, rank, _lib.MOE_EP_PUSH, ep.peer_ret, None,
                                 S, ep.expert_out, None, ep.cap, w.H * 2, 0, None, st)
            e[3].record(stream)
            ep.comm.barrier(dev)  # the pushes into the other ranks end before their next step
        torch.cuda.synchronize()
        dist.barrier()
        if ep.status() != 0:
            raise SystemExit(f"expert-parallel {w.name}: device status after timing")
        agg = aggregate(sum(a.elapsed_time(b) for a, b in step_ev), w.T, args.steps, dev)
        # the backward of the last forward: d_eo to the experts' owners, the experts' backward,
        # dx_rows back (the same exchange as the forward's), K calls behind an L2 flush
        g = torch.Generator(device=dev).manual_seed(9)
        dy = torch.randn((w.T, w.H), generator=g, device=dev).to(torch.bfloat16)
        for _ in range(args.warmup):
            flush.fill_(1)
            ep.backward(dy, logits, wg, wu, wd)
        bwd_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                  for _ in range(args.steps)]
        dist.barrier()
        torch.cuda.synchronize()
        for a, b in bwd_ev:
            flush.fill_(1)
            a.record(stream)
            ep.backward(dy, logits, wg, wu, wd)
            b.record(stream)
        torch.cuda.synchronize()
        if ep.status() != 0:
            raise SystemExit(f"expert-parallel {w.name}: device status after the backward")
        bwd_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in bwd_ev), dev) / args.steps
        t_pull = sum(e[0].elapsed_time(e[1]) for e in x_ev) / args.steps
        t_push = sum(e[2].elapsed_time(e[3]) for e in x_ev) / args.steps
        pk, _ = peaks()
        hbm = pk["hbm_gbs"]

        def kern(b, t):
            g = b / (t * 1e-3) / 1e9
            return {"ms": t, "GB/s": g, "frac": g / hbm, "bytes": b}

        out = {"mode": "p2p", "workload": w.name, "ranks": R, "experts_per_rank": E_loc,
               "value": agg["value"], "unit": "tokens/s", "ms_per_step": agg["ms_per_step"],
               "backward_ms": bwd_ms,
               "train_step_tokens_per_s": R * w.T / ((agg["ms_per_step"] + bwd_ms) * 1e-3),
               "received_rows": n_recv,
               "exchange": {
                   # each received row is read once and written once; at one rank both are HBM
                   "pull": kern(2 * n_recv * row_b, t_pull),
                   "push": kern(2 * n_recv * w.H * 2, t_push)},
               "note": ("tokens/s counts every rank's T tokens over the slowest rank's step; "
                        "exchange frac is of the measured HBM copy rate (at one rank every peer "
                        "buffer is local; across GPUs the remote share is NVLink-bound)")}
        del ep, flush, wg, wu, wd
        torch.cuda.empty_cache()
        return out
    finally:
        if own_group:
            torch.cuda.synchronize()
            dist.destroy_process_group()


def measure_w8(w, m, d, args, stream, flush_l2, world, dev, S, active, pk) -> dict:
    """The same step with FP8 gate / up weights (W8A8 first projection, bf16 down projection): the
    weights are quantised once beforehand, outside the timed region; each step quantises its FFN
    input rows inside the FFN call.  K metric steps interleaved with K steps that time the FFN."""
    import torch.distributed as dist
    gq, gs, uq, us = m.quantize_expert_weights_fp8(d["w_gate"], d["w_up"])

    def step():
        m.route(d["logits"])
        m.dispatch(d["x"])
        m.expert_ffn_w8(gq, gs, uq, us, d["w_down"])
        m.combine()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if m.status() != 0:
        raise SystemExit(f"{w.name}: device status after the FP8-weight warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        e = ev[i]
        flush_l2()
        e[0].record(stream)
        step()
        e[1].record(stream)
        flush_l2()
        m.route(d["logits"])
        m.dispatch(d["x"])
        e[2].record(stream)
        m.expert_ffn_w8(gq, gs, uq, us, d["w_down"])
        e[3].record(stream)
        m.combine()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if m.status() != 0:
        raise SystemExit(f"{w.name}: device status after the FP8-weight steps")
    agg = aggregate(sum(e[0].elapsed_time(e[1]) for e in ev), w.T, args.steps, dev)
    t_ffn = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    fp8 = w.payload == "fp8"
    wbytes = active * (2 * w.H * w.F + w.H * w.F * 2 + 2 * w.F * 4)   # e4m3 gate/up + scales, bf16 down
    rows = S * w.H * (1 if fp8 else 2) + (S * (w.H // 128) * 4 if fp8 else 0) + S * w.H * 2
    ffn_bytes = wbytes + rows
    flops8, flops16 = 4 * S * w.H * w.F, 2 * S * w.H * w.F
    hbm = pk["hbm_gbs"]
    p16 = pk["bf16_tflops_sustained"]
    p8 = 2.0 * p16          # dense e4m3 = 2 x dense bf16 (nominal ratio 4.5 / 2.25 PFLOP/s)
    t_bytes = ffn_bytes / (hbm * 1e9)
    t_flops = flops8 / (p8 * 1e12) + flops16 / (p16 * 1e12)
    bound = max(t_bytes, t_flops)
    return {"value": agg["value"], "ms_per_step": agg["ms_per_step"], "ffn_ms": t_ffn,
            "ffn_GB/s": ffn_bytes / (t_ffn * 1e-3) / 1e9,
            "ffn_TFLOP/s": (flops8 + flops16) / (t_ffn * 1e-3) / 1e12,
            "roofline": {"bound": "hbm" if t_bytes >= t_flops else "tensor",
                         "frac_of_max_time_bound": bound / (t_ffn * 1e-3),
                         "algorithmic_bytes": ffn_bytes, "flops_e4m3": flops8,
                         "flops_bf16": flops16, "peak_hbm_gbs": hbm,
                         "peak_e4m3_tflops": p8, "peak_bf16_tflops": p16,
                         "peak_note": "e4m3 peak = 2 x the measured sustained bf16 figure"},
            "gpu_launches": 2 * (7 + (1 if fp8 else 0)) * args.steps,
            "note": "gate / up weights e4m3 with one fp32 scale per row (quantised before timing), "
                    "FFN input rows quantised per row inside the step, down projection bf16"}


def e2e_run(w, m, d, args, dev, world: int, stream) -> dict:
    """End to end through the public API, as a serving loop runs it: every step uploads its logits
    and tokens from pinned host memory and downloads its result to pinned host memory; uploads and
    downloads run on their own streams, double-buffered, so they overlap the neighbouring steps'
    compute (timed from the first upload to the last download)."""
    logits_h = d["logits"].cpu().pin_memory()
    x_h = d["x"].cpu().pin_memory()
    y_h = [torch.empty(m.y.shape, dtype=m.y.dtype).pin_memory() for _ in range(2)]
    logits_d = [d["logits"].clone() for _ in range(2)]
    x_d = [d["x"].clone() for _ in range(2)]
    y_stage = [torch.empty_like(m.y) for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_steps = max(3, min(args.steps, 50))
    # each buffer slot's step (forward + copy of y) is one captured CUDA graph (--e2e-eager: not;
    # with several ranks the loop stays eager, as no graph is recorded next to a communicator)
    use_graphs = not args.e2e_eager and world == 1
    graphs = (None if not use_graphs else
              [m.capture(logits_d[b], x_d[b], d["w_gate"], d["w_up"], d["w_down"], out=y_stage[b])
               for b in range(2)])

    def e2e_loop(n):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        h2d = [ev(), ev()]
        fwd = [ev(), ev()]
        d2h = [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(fwd[b])          # step i-2 finished reading buffer b
                logits_d[b].copy_(logits_h, non_blocking=True)
                x_d[b].copy_(x_h, non_blocking=True)
                h2d[b].record(up)
            stream.wait_event(h2d[b])
            if graphs is not None:
                if i >= 2:
                    stream.wait_event(d2h[b])      # step i-2's download finished reading y_stage[b]
                graphs[b].replay()
            else:
                m.forward(logits_d[b], x_d[b], d["w_gate"], d["w_up"], d["w_down"])
                if i >= 2:
                    stream.wait_event(d2h[b])      # step i-2's download finished reading y_stage[b]
                y_stage[b].copy_(m.y)
            fwd[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(fwd[b])
                y_h[b].copy_(y_stage[b], non_blocking=True)
                d2h[b].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_loop(3)  # warm-up
    agg = aggregate(e2e_loop(e2e_steps), w.T, e2e_steps, dev)
    weights_gb = 3 * w.E * w.H * w.F * 2 / 1e9
    del graphs
    return {"value": agg["value"], "unit": "tokens/s",
            "method": ("each step one replay of a captured CUDA graph (forward + copy of y); "
                       if use_graphs else "eager forward per step; ") +
                      "uploads/downloads on two copy streams, double-buffered, overlapping "
                      "the neighbouring steps' compute; L2 not flushed inside this loop (each "
                      f"step streams up to {weights_gb:.2f} GB of weights)",
            "h2d_bytes_per_step": d["logits"].numel() * 4 + d["x"].numel() * 2,
            "d2h_bytes_per_step": m.y.numel() * 2}


if __name__ == "__main__":
    main()
