"""Benchmark of the dropless MoE expert-MLP forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole forward (zero out, route, sparse map, GEMM1, GEMM2) through the C ABI over one
batch of seeded synthetic inputs. Default workload: the Mixtral-8x7B-shaped prefill layer
(S=4096, D=4096, F=14336, E=8, top-2, bf16). With N > 1 (launched by torch.distributed.run) every
rank runs its own replica on its own batch (weak scaling, no data-path collective); the timed
region is bracketed by a barrier and device synchronisation, and the max over ranks is reported.
`--impl reference` times the CPU oracle instead (rank 0 only), on a bounded token sample.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_workloads as W  # noqa: E402

METRIC = "MoE-layer fwd tokens/s and TFLOP/s (bf16) as % of B200 peak; sparse-map GB/s"
NOMINAL_TFLOPS = {"bf16": 2250.0, "f32": 1125.0}   # dense bf16; tf32 for fp32 inputs
NOMINAL_HBM_GBS = 8000.0


def flops_of(w: W.Workload) -> dict:
    R = w.R
    return {
        "router": 2.0 * w.S * w.D * w.E,
        "gemm1": 4.0 * R * w.D * w.F,
        "gemm2": 2.0 * R * w.F * w.D,
    }


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


def gemm_source_hash() -> str:
    """Hash of the sources that define the grouped GEMM kernels (a recorded DRAM traffic figure is
    only reported while they are unchanged)."""
    h = hashlib.sha256()
    for name in ("grouped_gemm.cu", "grouped_gemm_2sm.cu", "gemm_common.cuh", "moe_internal.cuh"):
        with open(os.path.join(ROOT, "sparse_mixture_experts_02_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str):
    """DRAM bytes per launch of `kernel_key` from the committed ncu summary, if the kernel source
    is unchanged since it was captured (the summary records the source hash)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        text = open(path).read()
        sha = gemm_source_hash()
    except OSError:
        return None
    m = re.search(r"^\|\s*" + re.escape(kernel_key) + r"\s*\|\s*([0-9]+)\s*\|\s*([0-9a-f]+)\s*\|",
                  text, re.M)
    if not m or m.group(2) != sha:
        return None
    return int(m.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return None
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.file.name)
        if not rows:
            return None
        mx = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * mx] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows)}


def run_oracle_sample(w, inp_cpu, n_tokens, seed=0):
    """Times the CPU oracle on n_tokens tokens of the workload; returns (seconds, tokens, cores)."""
    import numpy as np

    import oracle
    toks = np.random.default_rng(seed).choice(w.S, size=min(n_tokens, w.S),
                                              replace=False).astype(np.int32)
    t0 = time.perf_counter()
    oracle.mlp_forward(inp_cpu["x"], inp_cpu["w_gate"], inp_cpu["w_gate_e"], inp_cpu["w_up"],
                       inp_cpu["w_down"], w.k, bias=inp_cpu["logit_bias"], tokens=toks)
    return time.perf_counter() - t0, len(toks), oracle.num_threads()


def host_inputs(inp):
    return {k: (v.float().cpu().numpy() if v is not None else None) for k, v in inp.items()}


def calibrate_oracle(w, inp_cpu, budget_s):
    """Number of tokens the oracle covers in about budget_s seconds, from a probe that keeps
    every host thread busy (one token per thread; its time is the per-wave cost)."""
    import oracle
    n_probe = max(1, min(w.S, oracle.num_threads()))
    t, n, _ = run_oracle_sample(w, inp_cpu, n_probe, seed=123)
    per_token = max(t, 1e-6) / n
    return max(1, min(w.S, int(budget_s / per_token)))


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def bench_reference(args, w, ws, rank):
    """The oracle on the host cores: each step a bounded token sample of the workload."""
    if rank != 0:
        return None
    inp = W.make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    inp_cpu = host_inputs(inp)
    del inp
    # each step a bounded sample: the whole warm-up + timed run stays near 150 s of oracle work
    step_s = args.ref_step_s or min(4.0, max(0.2, 150.0 / (args.steps + args.warmup)))
    per_step = calibrate_oracle(w, inp_cpu, step_s)
    for i in range(args.warmup):
        run_oracle_sample(w, inp_cpu, per_step, seed=1000 + i)
    t_total, n_total, cores = 0.0, 0, 1
    for i in range(args.steps):
        t, n, cores = run_oracle_sample(w, inp_cpu, per_step, seed=i)
        t_total += t
        n_total += n
    value = n_total / t_total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * t_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, **{k: getattr(w, k) for k in "SDFEk"},
                   "input_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} seeded tokens of {w.S} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    return line


def bench_ours(args, w, ws, rank, local):
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", local)
    seed = rank  # every rank its own batch; rank 0 is the N=1 workload
    inp = W.make_inputs(w, device=dev, seed=seed)
    wsp = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
    out = torch.empty((w.S, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        if events is not None:
            moe.profile_events(events)
        moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"],
                        w.k, logit_bias=inp["logit_bias"], out=out, ws=wsp)

    for _ in range(args.warmup):
        step()
    moe.check_device_status(wsp)
    launches_per_step = moe.last_launch_count()

    # events for the per-stage breakdown, 5 per step, created and recorded once up front
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if ws > 1:
            torch.distributed.barrier()
    ms_total = t0.elapsed_time(t1)
    moe.check_device_status(wsp)
    if ws > 1:
        t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(t.item())
    stage = {"route": [], "sparse_map": [], "gemm1": [], "gemm2": []}
    for row in evs:
        stage["route"].append(row[0].elapsed_time(row[1]))
        stage["sparse_map"].append(row[1].elapsed_time(row[2]))
        stage["gemm1"].append(row[2].elapsed_time(row[3]))
        stage["gemm2"].append(row[3].elapsed_time(row[4]))
    stage_ms = {k: sum(v) / len(v) for k, v in stage.items()}

    # End to end: every step copies its x in from pinned host memory and its fp32 out back to
    # pinned host memory, inside the timed region. The copies run on two side streams with two
    # device buffers each, so step i's forward overlaps step i+1's input copy and step i-1's
    # output copy (a pipelined caller); the timed region ends when the last output has landed.
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty((w.S, w.D), dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    out_dev = [out, torch.empty_like(out)]
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    fwd_done = [None, None]
    out_read = [None, None]

    def e2e_step(i):
        b = i & 1
        with torch.cuda.stream(h2d):
            if fwd_done[b] is not None:
                h2d.wait_event(fwd_done[b])  # the forward two steps back has read x_dev[b]
            x_dev[b].copy_(x_host, non_blocking=True)
            x_ready = torch.cuda.Event()
            x_ready.record(h2d)
        stream.wait_event(x_ready)
        if out_read[b] is not None:
            stream.wait_event(out_read[b])  # out_dev[b] of two steps back has been copied out
        moe.mlp_forward(x_dev[b], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"],
                        w.k, logit_bias=inp["logit_bias"], out=out_dev[b], ws=wsp)
        fwd_done[b] = torch.cuda.Event()
        fwd_done[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(fwd_done[b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            out_read[b] = torch.cuda.Event()
            out_read[b].record(d2h)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(out_read[(args.steps - 1) & 1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if ws > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    # the pipelined copies must reproduce the device result of the same input
    b_last = (args.steps - 1) & 1
    torch.testing.assert_close(out_host[b_last], out_dev[b_last].cpu(), rtol=0, atol=0)

    counts = wsp.view("expert_counts").cpu()
    hist = {"max": int(counts.max()), "min": int(counts.min()),
            "empty": int((counts == 0).sum()), "mean": float(counts.float().mean())}

    if rank != 0:
        return None

    fl = flops_of(w)
    flop_step = sum(fl.values())
    s_per_step = ms_total / 1000.0 / args.steps
    tokens_per_s = w.S * ws / s_per_step
    tflops = flop_step / s_per_step / 1e12
    pk, pk_kind = peaks()
    dt = w.dtype
    ratio = 1.0 if dt == "bf16" else NOMINAL_TFLOPS["f32"] / NOMINAL_TFLOPS["bf16"]
    peak_burst = pk["bf16_tflops"] * ratio
    peak_sust = pk["bf16_tflops_sustained"] * ratio
    map_bytes = w.R * 4 + 2 * w.R * 4 + (2 * w.E + 1) * 4
    g1_tflops = fl["gemm1"] / (stage_ms["gemm1"] / 1000.0) / 1e12
    key = f"gemm1_gateup_swiglu@{w.name}"
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dt, "data": "synthetic",
        "config": {"workload": w.name, **{k: getattr(w, k) for k in "SDFEk"},
                   "router": w.router_std, "zipf_s": w.zipf_s, "seed": "rank",
                   "parallelism": f"replicas{ws}",
                   "l2": "inputs larger than L2 (all expert weights streamed every step)"},
        "tflops": tflops,
        "tflops_frac": {"of_measured_sustained": tflops / peak_sust,
                        "of_measured_burst": tflops / peak_burst,
                        "of_nominal": tflops / NOMINAL_TFLOPS[dt], "peaks": pk_kind},
        "stage_ms": stage_ms,
        "sparse_map_gbs": map_bytes / (stage_ms["sparse_map"] / 1000.0) / 1e9,
        "expert_hist": hist,
        "roofline": {"kernel": "gemm1_gateup_swiglu", "bound": "tensor", "achieved": g1_tflops,
                     "peak": peak_sust, "unit": "TFLOP/s", "frac": g1_tflops / peak_sust,
                     "peak_kind": f"{pk_kind} sustained bf16"
                                  + ("" if dt == "bf16" else " x tf32/bf16 nominal ratio"),
                     "traffic": recorded_traffic(key)},
        "e2e": {"value": w.S * ws / (e2e_ms / 1000.0 / args.steps), "unit": "tokens/s",
                "copies": "pinned host, two side streams, double-buffered, overlapping the forwards",
                "h2d_bytes_per_step": w.S * w.D * inp["x"].element_size(),
                "d2h_bytes_per_step": w.S * w.D * 4},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if ws == 1 and not args.no_cpu_baseline:
        inp_cpu = host_inputs(inp)
        n = calibrate_oracle(w, inp_cpu, args.cpu_budget_s)
        t, ntok, cores = run_oracle_sample(w, inp_cpu, n)
        line["cpu_baseline"] = {"value": ntok / t, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{ntok} seeded tokens of {w.S} ({t:.1f} s)"}
    return line


def map_sweep(args):
    """Sparse-map bandwidth over route counts 2^20..2^26 and E in {8, 64, 128, 256} (k = 8,
    distinct experts per token, uniform marginals). Each point is the median of CUDA-event-timed
    moe_sparse_map calls on the launch stream, L2 flushed (a 256 MiB write) before every call.
    Algorithmic bytes: top_experts read (4R), sparse_rows and sorted_rows written (8R), counts and
    offsets ((2E+1)*4)."""
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    pk, pk_kind = peaks()
    points = []
    grid = [(log_r, E) for log_r in range(20, 27) for E in (8, 64, 128, 256)]
    if args.map_points:
        grid = [tuple(int(v) for v in pt.split(":")) for pt in args.map_points.split(",")]
    for log_r, E in grid:
        R = 1 << log_r
        k = 8
        te = W.make_top_experts(R // k, k, E, seed=log_r * 1000 + E, mode="stride", device=dev)
        need = moe.workspace_size("sparse_map", R // k, 0, 0, E, k, moe.MOE_BF16)
        wsp = moe.alloc_workspace(need, dev)
        reps = args.steps if args.map_points else max(5, min(args.steps, (1 << 27) // R))
        times = []
        for i in range(args.warmup + reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            moe.sparse_map(te, E, ws=wsp)
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                times.append(e0.elapsed_time(e1))
        moe.check_device_status(wsp)
        t_ms = sorted(times)[len(times) // 2]
        nbytes = 4 * R + 8 * R + (2 * E + 1) * 4
        gbs = nbytes / (t_ms * 1e-3) / 1e9
        points.append({"R": R, "E": E, "us": round(t_ms * 1e3, 2), "GB/s": round(gbs, 1),
                       "frac_of_hbm_peak": round(gbs / pk["hbm_gbs"], 3)})
        del te, wsp
    return {"metric": "sparse-map GB/s sweep", "unit": "GB/s", "n_gpus": 1,
            "data": "synthetic (seeded stride routing: k = 8 distinct experts per token)",
            "l2": "flushed before every call", "launches_per_call": 3,
            "peak_hbm_gbs": pk["hbm_gbs"], "peak_kind": pk_kind, "points": points}


def backward_bench(args, w):
    """Time moe_mlp_backward on workload w (bf16): one forward fills the workspace with routing,
    map and h, then W warm-up and K timed backward steps (CUDA events on the launch stream). A
    step's algorithmic work: 12*R*D*F expert FLOPs (dh, dW_down, dx, dW_gate_e, dW_up) plus the
    router's 2*S*D*E (dW_gate) and 2*S*k*D (dx); the kernels also recompute a and b (4*R*D*F)."""
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_inputs(w, device=dev, seed=0)
    fws = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
    out = torch.empty((w.S, w.D), dtype=torch.float32, device=dev)
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k,
                    logit_bias=inp["logit_bias"], out=out, ws=fws)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1)
    dout = torch.randn((w.S, w.D), generator=gen, device=dev)
    bws = moe.alloc_workspace(moe.workspace_size("mlp_backward", w.S, w.D, w.F, w.E, w.k,
                                                 inp["x"].dtype), dev)

    def step(evs=None):
        if evs is not None:
            moe.profile_events(evs)
        return moe.mlp_backward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                inp["w_down"], w.k, dout, fws, ws=bws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    moe.check_device_status(bws)
    launches = moe.last_launch_count()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record()
        for i in range(args.steps):
            step(evs[i])
        t1.record()
        torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    names = ["dh", "gemm1_recompute_with_swiglu_bwd", "dW_down", "dx", "dW_gate_e_and_dW_up",
             "router"]
    stage = {n: sum(r[q].elapsed_time(r[q + 1]) for r in evs) / args.steps
             for q, n in enumerate(names)}
    R = w.S * w.k
    flop = 12.0 * R * w.D * w.F + 2.0 * w.S * w.D * w.E + 2.0 * w.S * w.k * w.D
    pk, pk_kind = peaks()
    tflops = flop / (ms * 1e-3) / 1e12
    return {"metric": "MoE-layer backward tokens/s and TFLOP/s (bf16)", "value": w.S / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "S": w.S, "D": w.D, "F": w.F, "E": w.E, "k": w.k,
                       "l2": "inputs larger than L2 (all expert weights streamed every step)"},
            "tflops": tflops, "flop_per_step": flop,
            "tflops_frac": {"of_measured_sustained": tflops / pk["bf16_tflops_sustained"],
                            "of_nominal": tflops / 2250.0, "peaks": pk_kind},
            "extra_flop_recompute": 4.0 * R * w.D * w.F, "stage_ms": stage,
            # dominant stage: the weight gradients of the gate and up projections (two grouped
            # weight-gradient GEMMs, 2 R D F FLOPs each)
            "roofline": {"kernel": "dW_gate_e_and_dW_up (grouped_wgrad_kernel x2)",
                         "bound": "tensor",
                         "achieved": 4.0 * R * w.D * w.F / (stage["dW_gate_e_and_dW_up"] * 1e-3) / 1e12,
                         "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": 4.0 * R * w.D * w.F / (stage["dW_gate_e_and_dW_up"] * 1e-3) / 1e12
                         / pk["bf16_tflops_sustained"],
                         "peak_kind": "measured sustained bf16" if pk_kind == "measured" else pk_kind,
                         "traffic": None},
            "gpu_launches": launches * args.steps, "clocks": clk.summary()}


def ep_bench(args, w):
    """Expert-parallel forward (expert_parallel.ep_mlp_forward) on N ranks, one GPU each: the E
    experts split into N contiguous ranges, every rank routing its own S tokens (weak scaling).
    The timed region includes the count exchange's host synchronisation and the three
    all-to-alls (NCCL); time is the max over ranks of CUDA-event time."""
    import datetime
    import socket

    import sparse_mixture_experts_02_b200 as moe  # noqa: F401 (loads the library)
    from sparse_mixture_experts_02_b200.expert_parallel import STAGES, ep_mlp_forward

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if "MASTER_ADDR" not in os.environ:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
        os.environ["MASTER_ADDR"] = "127.0.0.1"
    torch.distributed.init_process_group("nccl", rank=rank, world_size=ws,
                                         timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        if w.E % ws != 0:
            raise SystemExit(f"E={w.E} does not split over {ws} ranks")
        el = w.E // ws
        inp = W.make_inputs(w, device=dev, seed=0)  # the same weights on every rank
        sl = slice(rank * el, (rank + 1) * el)
        wge, wup, wd = (inp[n][sl].contiguous() for n in ("w_gate_e", "w_up", "w_down"))
        del inp["w_gate_e"], inp["w_up"], inp["w_down"]
        g = torch.Generator(device=dev)
        g.manual_seed(1000 + rank)  # every rank its own tokens
        x = torch.randn((w.S, w.D), generator=g, device=dev).to(inp["x"].dtype)

        def step(evs=None):
            return ep_mlp_forward(x, inp["w_gate"], wge, wup, wd, w.E, w.k,
                                  logit_bias=inp["logit_bias"], events=evs)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)]
               for _ in range(args.steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(torch.cuda.current_device()) as clk:
            t0.record()
            for i in range(args.steps):
                step(evs[i])
            t1.record()
            torch.cuda.synchronize(dev)
        torch.distributed.barrier()
        ms = t0.elapsed_time(t1) / args.steps
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_max = float(t.item())
        stage = {n: sum(r[q].elapsed_time(r[q + 1]) for r in evs) / args.steps
                 for q, n in enumerate(STAGES)}
        if rank != 0:
            return None
        fl = flops_of(w)
        flop = ws * (fl["router"] + fl["gemm1"] + fl["gemm2"])
        return {"metric": "expert-parallel MoE-layer fwd tokens/s (bf16)",
                "value": ws * w.S / (ms_max * 1e-3), "unit": "tokens/s", "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "dtype": w.dtype,
                "data": "synthetic",
                "config": {"workload": w.name, "S_per_rank": w.S, "D": w.D, "F": w.F, "E": w.E,
                           "k": w.k, "experts_per_rank": el, "parallelism": f"ep{ws}",
                           "l2": "inputs larger than L2 (expert weights streamed)"},
                "tflops": flop / (ms_max * 1e-3) / 1e12, "stage_ms_rank0": stage,
                # dominant stage: the local experts on the received rows (GEMM1 + GEMM2)
                "roofline": {"kernel": "experts (grouped GEMMs on received rows, rank 0)",
                             "bound": "tensor",
                             "achieved": (fl["gemm1"] + fl["gemm2"]) / (stage["experts"] * 1e-3) / 1e12,
                             "peak": peaks()[0]["bf16_tflops_sustained"], "unit": "TFLOP/s",
                             "frac": (fl["gemm1"] + fl["gemm2"]) / (stage["experts"] * 1e-3) / 1e12
                             / peaks()[0]["bf16_tflops_sustained"],
                             "traffic": None},
                "clocks": clk.summary()}
    finally:
        torch.distributed.destroy_process_group()


def moa_flops(w: W.MoaWorkload) -> dict:
    """Algorithmic FLOPs of one Mixture-of-Attention forward: router, shared key/value projection,
    routed query projection, causal attention (route at token s: 4*dh*(s+1) per head, summed over
    the k routes of every token) and routed output projection."""
    return {
        "router": 2.0 * w.S * w.D * w.E,
        "kv_projection": 2.0 * w.S * w.D * 2 * w.HD,
        "q_projection": 2.0 * w.R * w.D * w.HD,
        "attention": 2.0 * w.HD * w.k * w.S * (w.S + 1),
        "o_projection": 2.0 * w.R * w.HD * w.D,
    }


def moa_bench(args, w):
    """Time moe_moa_forward on workload w (bf16): W warm-up and K timed steps, CUDA events on the
    launch stream, per-stage events from the library."""
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_moa_inputs(w, device=dev, seed=0)
    ws = moe.MoaWorkspace(w.S, w.D, w.HD, w.E, w.k, dev)
    out = torch.empty((w.S, w.D), dtype=torch.float32, device=dev)

    def step(evs=None):
        if evs is not None:
            moe.profile_events(evs)
        return moe.moa_forward(inp["x"], inp["w_gate"], inp["w_q"], inp["w_kv"], inp["w_o"], w.k,
                               w.H, logit_bias=inp["logit_bias"], out=out, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    moe.check_device_status(ws)
    launches = moe.last_launch_count()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record()
        for i in range(args.steps):
            step(evs[i])
        t1.record()
        torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    names = ["route", "sparse_map", "kv_projection", "q_projection", "attention", "o_projection"]
    stage = {n: sum(r[q].elapsed_time(r[q + 1]) for r in evs) / args.steps
             for q, n in enumerate(names)}
    fl = moa_flops(w)
    flop = sum(fl.values())
    pk, pk_kind = peaks()
    tflops = flop / (ms * 1e-3) / 1e12
    att = fl["attention"] / (stage["attention"] * 1e-3) / 1e12
    return {"metric": "MoA-layer fwd tokens/s and TFLOP/s (bf16)", "value": w.S / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "S": w.S, "D": w.D, "H": w.H, "dh": w.dh, "E": w.E,
                       "k": w.k, "l2": "inputs larger than L2 (expert weights streamed)"},
            "tflops": tflops, "flop_per_step": flop, "flop_by_stage": fl,
            "tflops_frac": {"of_measured_sustained": tflops / pk["bf16_tflops_sustained"],
                            "of_nominal": tflops / 2250.0, "peaks": pk_kind},
            "roofline": {"kernel": "attention core", "bound": "tensor", "achieved": att,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": att / pk["bf16_tflops"], "traffic": None},
            "stage_ms": stage, "gpu_launches": launches * args.steps, "clocks": clk.summary(),
            "cpu_baseline": None if args.no_cpu_baseline else moa_oracle_baseline(w, inp,
                                                                                  args.cpu_budget_s)}


def moa_oracle_baseline(w, inp, budget_s):
    """The oracle's MoA forward on a causal prefix of the sequence (tokens 0..n-1 depend on
    nothing later), n sized from a 16-token probe to take about budget_s seconds."""
    import oracle
    cpu = host_inputs(inp)
    HD = w.HD

    def run(n):
        t0 = time.perf_counter()
        oracle.moa_forward(cpu["x"][:n], cpu["w_gate"], cpu["w_q"], cpu["w_kv"][:, :HD],
                           cpu["w_kv"][:, HD:], cpu["w_o"], w.k, w.H, bias=cpu["logit_bias"])
        return time.perf_counter() - t0

    n0 = min(w.S, 16)
    t = run(n0)
    n = max(n0, min(w.S, int(n0 * budget_s / max(t, 1e-6))))
    t = run(n)
    return {"value": n / t, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": ("the whole sequence" if n >= w.S else
                       f"the first {n} tokens of the sequence (a causal prefix: shorter attention "
                       f"spans than the full sequence's average)")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral_prefill",
                    choices=list(W.WORKLOADS) + list(W.PROFILE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=None)
    ap.add_argument("--map-sweep", action="store_true",
                    help="instead of the forward: sparse-map GB/s over R = 2^20..2^26 routes")
    ap.add_argument("--backward", action="store_true",
                    help="instead of the forward: time moe_mlp_backward on --workload")
    ap.add_argument("--moa", action="store_true",
                    help="instead of the MLP forward: time moe_moa_forward (Mixture of Attention)")
    ap.add_argument("--ep", action="store_true",
                    help="instead of the replicated forward: the expert-parallel forward, experts "
                         "split over the ranks (all-to-all dispatch and combine over NCCL)")
    ap.add_argument("--map-points", default="",
                    help="with --map-sweep: only these points, 'log2R:E,...' (e.g. 26:256)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.map_sweep:
        print(json.dumps(map_sweep(args)), flush=True)
        return
    if args.ep:
        wl = {**W.WORKLOADS, **W.PROFILE_WORKLOADS}[args.workload]
        line = ep_bench(args, wl)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.moa:
        print(json.dumps(moa_bench(args, W.MOA_WORKLOADS["moa_prefill"])), flush=True)
        return
    if args.backward:
        wl = {**W.WORKLOADS, **W.PROFILE_WORKLOADS}[args.workload]
        print(json.dumps(backward_bench(args, wl)), flush=True)
        return
    w = {**W.WORKLOADS, **W.PROFILE_WORKLOADS}[args.workload]
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks have nothing to do
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            line = bench_reference(args, w, ws, rank)
            print(json.dumps(line), flush=True)
        return
    ws, rank, local = dist_setup()
    try:
        line = bench_ours(args, w, ws, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
