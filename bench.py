"""Benchmark of the dropless MoE expert-MLP forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole forward (zero out, route, sparse map, GEMM1, GEMM2) through the C ABI over one
batch of seeded synthetic inputs. Default workload: the Mixtral-8x7B-shaped prefill layer
(S=4096, D=4096, F=14336, E=8, top-2, bf16). With N > 1 (launched by torch.distributed.run) every
rank runs its own replica on its own batch (weak scaling, no data-path collective); the timed
region is bracketed by a barrier and device synchronisation, and the max over ranks is reported.
At N = 1 the line also carries a `workloads` object: every other configuration (the fp32 tiny
layer, Mixtral decode, the 128-expert layer and the Zipf-skewed layer), each timed the same way
with its own clocks and its own roofline. `--impl reference` times the CPU oracle instead (rank 0
only), on a bounded token sample.

`python bench.py --record-traffic LAUNCHES.csv --workload NAME` reads an ncu CSV of
`dram__bytes_read.sum`, `dram__bytes_write.sum` and `gpu__time_duration.sum` per launch and
records the DRAM bytes per launch of each kernel class in profiles/dram_traffic.json, with a hash
of the sources that define that kernel; the bench reports a recorded figure only while those
sources are unchanged.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
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
L2_BYTES = 126 * 1000 * 1000
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "dram_traffic.json")
CSRC = os.path.join(ROOT, "sparse_mixture_experts_02_b200", "csrc")
# sources that define each kernel class (a recorded DRAM figure is void once any of them changes)
KERNEL_SOURCES = {
    "x_copy": ("backward.cu", "moe_internal.cuh"),
    "gemm1": ("grouped_gemm.cu", "grouped_gemm_2sm.cu", "gemm_common.cuh", "moe_internal.cuh"),
    "gemm2": ("grouped_gemm.cu", "grouped_gemm_2sm.cu", "gemm_common.cuh", "moe_internal.cuh"),
    "router": ("route.cu", "grouped_gemm.cu", "gemm_common.cuh", "moe_internal.cuh"),
    "sparse_map": ("sparse_map.cu", "moe_internal.cuh"),
}
# forward stages in the order the library records its events; x_copy (the x rows copied to slot
# order before GEMM1, for large experts and F >= 2048) takes no time when the forward makes none
STAGES = ("route", "sparse_map", "x_copy", "gemm1", "gemm2")


def elt_bytes(w: W.Workload) -> int:
    return 2 if w.dtype == "bf16" else 4


def flops_of(w: W.Workload) -> dict:
    R = w.R
    return {
        "router": 2.0 * w.S * w.D * w.E,
        "gemm1": 4.0 * R * w.D * w.F,
        "gemm2": 2.0 * R * w.F * w.D,
    }


def bytes_of(w: W.Workload, e_act: int) -> dict:
    """Algorithmic DRAM bytes of each stage: what the method must move, once. e_act = experts with
    at least one route (only their weights stream)."""
    b = elt_bytes(w)
    R = w.R
    return {
        # x read, W_gate read, top experts and weights written
        "route": w.S * w.D * b + w.D * w.E * b + 8 * R,
        # routes read, slots and inverse permutation written, counts and offsets written
        "sparse_map": 12 * R + (2 * w.E + 1) * 4,
        # an implementation step, not the method's: its 4 R D bytes are not algorithmic
        "x_copy": 0,
        # x read, gate and up weights of active experts read, h written, out zeroed
        "gemm1": w.S * w.D * b + 2 * e_act * w.D * w.F * b + R * w.F * b + w.S * w.D * 4,
        # h read, down weights of active experts read, out read and written by the reductions
        "gemm2": R * w.F * b + e_act * w.F * w.D * b + 2 * w.S * w.D * 4,
    }


def input_bytes(w: W.Workload) -> int:
    b = elt_bytes(w)
    return w.S * w.D * b + w.D * w.E * b + 3 * w.E * w.D * w.F * b


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


def tensor_peak(dtype: str, clocks, timed_s):
    """The dense tensor peak that matches the timed region: the burst figure when the SM clock
    stayed within 5% of its maximum (or, without clock samples, when the region lasted under a
    second), else the sustained figure (measured over seconds under the power cap). fp32 inputs
    run as tf32: the bf16 figure times the nominal tf32 / bf16 ratio (1/2)."""
    pk, pk_kind = peaks()
    ratio = 1.0 if dtype == "bf16" else NOMINAL_TFLOPS["f32"] / NOMINAL_TFLOPS["bf16"]
    if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        burst = clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"]
        why = f"median SM clock {clocks['sm_mhz']:.0f} of max {clocks['sm_max_mhz']:.0f} MHz"
    else:
        burst = timed_s < 1.0
        why = f"no clock samples; timed region {timed_s:.2f} s"
    kind = "burst" if burst else "sustained"
    value = (pk["bf16_tflops"] if burst else pk["bf16_tflops_sustained"]) * ratio
    label = f"{pk_kind} {kind} bf16" + ("" if ratio == 1.0 else " x tf32/bf16 nominal ratio")
    return value, f"{label} ({why})"


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, path: str = TRAFFIC_JSON):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/dram_traffic.json, if the
    sources that define the kernel are unchanged since the capture; else None."""
    try:
        with open(path) as f:
            rec = json.load(f)["entries"][f"{kernel}@{workload}"]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("sources_sha16") != source_hash(kernel):
        return None
    return int(rec["dram_bytes_per_launch"])


def kernel_class(name: str):
    """Kernel class of an ncu kernel name (template arguments print as 0/1)."""
    m = re.search(r"(grouped_gemm_2sm_kernel|grouped_gemm_kernel)<([^>]*)>", name)
    if m:
        a = [int(v) for v in re.findall(r"-?\d+", m.group(2))]
        gather, glu, scatter = a[1], a[2], a[3]
        router = m.group(1) == "grouped_gemm_kernel" and len(a) > 4 and a[4] == 1
        if router:
            return "router"
        if glu and not scatter:  # x rows gathered on load or copied to slot order first
            return "gemm1"
        if scatter and not gather and not glu:
            return "gemm2"
        return None
    if re.search(r"\broute\w*_kernel", name):
        return "router"
    if re.search(r"\bmap_\w+_kernel", name):
        return "sparse_map"
    if re.search(r"\bgather_rows_kernel", name):
        return "x_copy"
    return None


def record_traffic(csv_path: str, workload: str, command: str, path: str = TRAFFIC_JSON):
    """Writes the mean DRAM bytes (read + write) per launch of each kernel class found in an ncu
    CSV into profiles/dram_traffic.json (entries keyed "<class>@<workload>")."""
    text = open(csv_path).read()
    start = text.find('"ID"')
    rows = csv.DictReader(io.StringIO(text[start:]))
    launches = {}
    for r in rows:
        d = launches.setdefault(r["ID"], {"name": r["Kernel Name"]})
        v = r["Metric Value"].replace(",", "")
        d[r["Metric Name"]] = float(v)
    per = {}
    for d in launches.values():
        c = kernel_class(d["name"])
        if c is None or "dram__bytes_read.sum" not in d:
            continue
        per.setdefault(c, []).append(d)
    try:
        with open(path) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        doc = {"about": "DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum), "
                        "mean over the captured launches of each kernel class; written by "
                        "`bench.py --record-traffic`", "entries": {}}
    out = {}
    for c, ds in per.items():
        rd = statistics.mean(d["dram__bytes_read.sum"] for d in ds)
        wr = statistics.mean(d["dram__bytes_write.sum"] for d in ds)
        ent = {"dram_bytes_per_launch": int(round(rd + wr)), "dram_bytes_read": int(round(rd)),
               "dram_bytes_write": int(round(wr)), "launches": len(ds),
               "kernel_names": sorted({d["name"].split("(")[0] for d in ds}),
               "sources_sha16": source_hash(c), "command": command,
               "recorded": datetime.date.today().isoformat()}
        if all("gpu__time_duration.sum" in d for d in ds):
            ent["ncu_duration_us_mean"] = statistics.mean(
                d["gpu__time_duration.sum"] for d in ds) / 1e3
        doc["entries"][f"{c}@{workload}"] = ent
        out[c] = ent
    with open(path, "w") as f:
        json.dump(doc, f, indent=1, sort_keys=True)
        f.write("\n")
    return out


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
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def n_x_buffers(w: W.Workload) -> int:
    """Copies of x the timed loop rotates through so that the router reads x from DRAM: enough
    that the copies together exceed the L2 (the weights, streamed every step, evict them too)."""
    xb = w.S * w.D * elt_bytes(w)
    return int(min(1024, max(2, math.ceil(1.25 * L2_BYTES / max(xb, 1)))))


def flush_l2_each_step(w: W.Workload) -> bool:
    """Workloads whose inputs fit in the L2 are timed step by step with an L2 flush in between."""
    return input_bytes(w) < 2 * L2_BYTES


def workload_config(w: W.Workload, ws: int) -> dict:
    """The `config` object of a bench line (the same for the GPU arm and the oracle arm)."""
    if flush_l2_each_step(w):
        l2 = ("inputs smaller than L2: a 256 MiB write flushes L2 before every step; steps timed "
              "one by one with CUDA events, flushes excluded")
    else:
        l2 = (f"inputs larger than L2 (all expert weights streamed every step); x rotated over "
              f"{n_x_buffers(w)} device copies")
    return {"workload": w.name, **{k: getattr(w, k) for k in "SDFEk"},
            "router": w.router_std, "zipf_s": w.zipf_s, "seed": "rank",
            "parallelism": f"replicas{ws}", "l2": l2}


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
        "config": workload_config(w, ws),
        "input_dtype": w.dtype,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} seeded tokens of {w.S} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    return line


def roofline(w: W.Workload, stage_ms: dict, e_act: int, clocks, timed_s: float):
    """Roofline of the dominant kernel, GEMM1 (gathered x, fused gate+up, SwiGLU: two thirds of
    the FLOPs and of the weight bytes). Both ceilings are computed; `bound` is the one whose
    minimum time is longer at the measured peaks (the other is reported under `other`)."""
    pk, pk_kind = peaks()
    t = stage_ms["gemm1"] / 1000.0
    flop = flops_of(w)["gemm1"]
    nbytes = bytes_of(w, e_act)["gemm1"]
    tf_peak, tf_kind = tensor_peak(w.dtype, clocks, timed_s)
    tensor = {"bound": "tensor", "achieved": flop / t / 1e12, "peak": tf_peak,
              "unit": "TFLOP/s", "frac": flop / t / 1e12 / tf_peak, "peak_kind": tf_kind}
    hbm = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
           "frac": nbytes / t / 1e9 / pk["hbm_gbs"], "peak_kind": f"{pk_kind} copy bandwidth"}
    t_tensor = flop / (tf_peak * 1e12)
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    main, other = (hbm, tensor) if t_hbm > t_tensor else (tensor, hbm)
    return {"kernel": "gemm1_gateup_swiglu", **main,
            "traffic": recorded_traffic("gemm1", w.name),
            "algorithmic_bytes": nbytes, "flop": flop, "launch_ms": stage_ms["gemm1"],
            "other": other}


def time_forward(moe, w, steps, warmup, dev, ws=1, seed=0):
    """Times `steps` forwards of workload w after `warmup` untimed ones. Returns the inputs, the
    workspace, the output buffer and the measurements. Inputs larger than the L2 are timed as one
    bracket of K steps (barrier + device sync on both sides, x rotated over several copies);
    smaller ones step by step with an L2 flush before each step."""
    inp = W.make_inputs(w, device=dev, seed=seed)
    wsp = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
    out = torch.empty((w.S, w.D), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = flush_l2_each_step(w)
    nx = 1 if flush else n_x_buffers(w)
    xs = [inp["x"]] + [inp["x"].clone() for _ in range(nx - 1)]
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None

    def step(i, events=None):
        if events is not None:
            moe.profile_events(events)
        moe.mlp_forward(xs[i % nx], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"],
                        w.k, logit_bias=inp["logit_bias"], out=out, ws=wsp)

    for i in range(warmup):
        step(i)
    moe.check_device_status(wsp)
    launches_per_step = moe.last_launch_count()

    # events for the per-stage breakdown, one more than the stages per step, created and
    # recorded once up front
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)]
           for _ in range(steps)]
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
        if flush:
            ms_total = 0.0
            for i in range(steps):
                flush_buf.zero_()
                step(i, evs[i])
            torch.cuda.synchronize(dev)
            ms_total = sum(r[0].elapsed_time(r[len(STAGES)]) for r in evs)
        else:
            t0.record(stream)
            for i in range(steps):
                step(i, evs[i])
            t1.record(stream)
            torch.cuda.synchronize(dev)
            ms_total = t0.elapsed_time(t1)
        if ws > 1:
            torch.distributed.barrier()
    moe.check_device_status(wsp)
    if ws > 1:
        t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(t.item())
    stage_ms = {n: sum(r[q].elapsed_time(r[q + 1]) for r in evs) / steps
                for q, n in enumerate(STAGES)}
    counts = wsp.view("expert_counts").cpu()
    e_act = int((counts > 0).sum())
    hist = {"max": int(counts.max()) if w.E else 0, "min": int(counts.min()) if w.E else 0,
            "empty": int((counts == 0).sum()), "mean": float(counts.float().mean())}
    clocks = clk.summary()
    s_per_step = ms_total / 1000.0 / steps
    fl = flops_of(w)
    by = bytes_of(w, e_act)
    meas = {
        "ms_per_step": ms_total / steps,
        "tokens_per_s": w.S * ws / s_per_step,
        "tflops": sum(fl.values()) / s_per_step / 1e12,
        "gbs": sum(by.values()) / s_per_step / 1e9,
        "stage_ms": stage_ms,
        "stage_gbs": {n: by[n] / (stage_ms[n] / 1000.0) / 1e9 for n in STAGES
                      if stage_ms[n] > 0 and by[n] > 0},
        "expert_hist": hist,
        "roofline": roofline(w, stage_ms, e_act, clocks, ms_total / 1000.0),
        "clocks": clocks,
        "gpu_launches": launches_per_step * steps,
        "x_buffers": nx,
        "timed_s": ms_total / 1000.0,
    }
    return inp, wsp, out, meas


def e2e_measure(moe, w, inp, wsp, out, steps, warmup, dev, ws=1):
    """End to end: every step copies its x in from pinned host memory and its fp32 out back to
    pinned host memory, inside the timed region. The copies run on two side streams with two
    device buffers each, so step i's forward overlaps step i+1's input copy and step i-1's output
    copy (a pipelined caller); the timed region ends when the last output has landed."""
    stream = torch.cuda.current_stream(dev)
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

    for i in range(warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    h2d.wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    stream.wait_event(out_read[(steps - 1) & 1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if ws > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    # the pipelined copies must reproduce the device result of the same input
    b_last = (steps - 1) & 1
    torch.testing.assert_close(out_host[b_last], out_dev[b_last].cpu(), rtol=0, atol=0)
    return {"value": w.S * ws / (e2e_ms / 1000.0 / steps), "unit": "tokens/s",
            "copies": "pinned host, two side streams, double-buffered, overlapping the forwards",
            "h2d_bytes_per_step": w.S * w.D * inp["x"].element_size(),
            "d2h_bytes_per_step": w.S * w.D * 4}


def workload_entry(w, meas):
    """One entry of the `workloads` object: the measurements plus the fractions of peak."""
    pk, pk_kind = peaks()
    tf_peak, tf_kind = tensor_peak(w.dtype, meas["clocks"], meas["timed_s"])
    return {"config": {k: getattr(w, k) for k in ("S", "D", "F", "E", "k", "dtype",
                                                   "router_std", "zipf_s")},
            "ms_per_step": meas["ms_per_step"], "tokens_per_s": meas["tokens_per_s"],
            "tflops": meas["tflops"], "gbs": meas["gbs"],
            "tflops_frac": {"of_measured_peak": meas["tflops"] / tf_peak, "peak_kind": tf_kind,
                            "of_nominal": meas["tflops"] / NOMINAL_TFLOPS[w.dtype]},
            "gbs_frac": {"of_measured": meas["gbs"] / pk["hbm_gbs"],
                         "of_nominal": meas["gbs"] / NOMINAL_HBM_GBS},
            "stage_ms": meas["stage_ms"], "stage_gbs": meas["stage_gbs"],
            "expert_hist": meas["expert_hist"], "roofline": meas["roofline"],
            "clocks": meas["clocks"], "gpu_launches": meas["gpu_launches"],
            "l2": workload_config(w, 1)["l2"]}


def bench_ours(args, w, ws, rank, local):
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", local)
    seed = rank  # every rank its own batch; rank 0 is the N=1 workload
    inp, wsp, out, meas = time_forward(moe, w, args.steps, args.warmup, dev, ws=ws, seed=seed)
    e2e = e2e_measure(moe, w, inp, wsp, out, args.steps, args.warmup, dev, ws=ws)
    if rank != 0:
        return None
    pk, pk_kind = peaks()
    tf_peak, tf_kind = tensor_peak(w.dtype, meas["clocks"], meas["timed_s"])
    line = {
        "metric": METRIC, "value": meas["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": meas["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, ws),
        "tflops": meas["tflops"],
        "tflops_frac": {"of_measured_peak": meas["tflops"] / tf_peak, "peak_kind": tf_kind,
                        "of_nominal": meas["tflops"] / NOMINAL_TFLOPS[w.dtype]},
        "gbs": meas["gbs"],
        "stage_ms": meas["stage_ms"], "stage_gbs": meas["stage_gbs"],
        "sparse_map_gbs": meas["stage_gbs"].get("sparse_map"),
        "expert_hist": meas["expert_hist"],
        "roofline": meas["roofline"],
        "e2e": e2e,
        "gpu_launches": meas["gpu_launches"],
        "clocks": meas["clocks"],
    }
    del inp, wsp, out
    if ws == 1 and not args.no_workloads:
        # every other configuration, timed the same way (one GPU; parity cases, not bench lines)
        others = {}
        for name in W.WORKLOADS:
            if name == w.name:
                continue
            wl = W.WORKLOADS[name]
            i2, ws2, o2, m2 = time_forward(moe, wl, args.steps, args.warmup, dev)
            others[name] = workload_entry(wl, m2)
            del i2, ws2, o2
            torch.cuda.empty_cache()
        line["workloads"] = others
    if ws == 1 and not args.no_cpu_baseline:
        inp_cpu = host_inputs(W.make_inputs(w, device=dev, seed=0))
        n = calibrate_oracle(w, inp_cpu, args.cpu_budget_s)
        t, ntok, cores = run_oracle_sample(w, inp_cpu, n)
        line["cpu_baseline"] = {"value": ntok / t, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle",
                                "sample": f"{ntok} seeded tokens of {w.S} ({t:.1f} s)"}
    return line


def torch_map_reference_ms(te, E, flush, warmup, reps):
    """The same map from library calls, as a reference timing for the sweep: a stable radix sort
    of the expert ids (sorted_rows), their histogram and its exclusive prefix (counts, offsets) and
    the inverse permutation (sparse_rows). Median CUDA-event time, L2 flushed before every call."""
    flat = te.reshape(-1)
    R = flat.numel()
    ar = torch.arange(R, dtype=torch.int64, device=flat.device)
    times = []
    for i in range(warmup + reps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        _, sorted_rows = torch.sort(flat, stable=True)
        counts = torch.bincount(flat, minlength=E)
        offsets = torch.cumsum(counts, 0) - counts
        sparse_rows = torch.empty_like(sorted_rows)
        sparse_rows.scatter_(0, sorted_rows, ar)
        e1.record()
        torch.cuda.synchronize(flat.device)
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    del offsets
    return sorted(times)[len(times) // 2]


def forward_torch_reference(args):
    """The expert-MLP forward built from torch calls (a cuBLAS GEMM per expert: gather, x W_gate_e,
    x W_up, SwiGLU, h W_down, router weight, index_add into the output), timed beside
    moe_mlp_forward on the same inputs and the library's routing, for every workload; also the
    reference's GEMMs alone on pre-gathered rows. Median of CUDA-event-timed calls, L2 flushed
    (a 256 MiB write) before each. A context measurement: the product path is the library."""
    import sparse_mixture_experts_02_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= args.warmup:
                ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2]

    results = {}
    for name in ("mixtral_prefill", "mixtral_decode", "e128", "zipf64"):
        w = W.WORKLOADS[name]
        inp = W.make_inputs(w, device=dev, seed=0)
        ws = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
        out = torch.empty((w.S, w.D), dtype=torch.float32, device=dev)
        t_lib = timed(lambda: moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                              inp["w_down"], w.k, logit_bias=inp["logit_bias"],
                                              out=out, ws=ws))
        # the reference is handed the library's routing (its top-k is not timed)
        flat = ws.view("top_experts").reshape(-1).long()
        order = torch.sort(flat, stable=True).indices
        counts = ws.view("expert_counts").cpu().tolist()
        offs = [0]
        for c in counts:
            offs.append(offs[-1] + c)
        tok = order // w.k
        gates = ws.view("top_weights").reshape(-1)[order]
        x, wg, wu, wd = inp["x"], inp["w_gate_e"], inp["w_up"], inp["w_down"]

        def ref():
            y = torch.zeros((w.S, w.D), dtype=torch.float32, device=dev)
            for e in range(w.E):
                a, b = offs[e], offs[e + 1]
                if a == b:
                    continue
                t = tok[a:b]
                xe = x.index_select(0, t)
                h = torch.nn.functional.silu(xe @ wg[e]) * (xe @ wu[e])
                y.index_add_(0, t, (h @ wd[e]).float() * gates[a:b, None])
            return y

        t_ref = timed(ref)
        xs = [x.index_select(0, tok[offs[e]:offs[e + 1]]) for e in range(w.E)]
        hs = [torch.empty((counts[e], w.F), dtype=x.dtype, device=dev) for e in range(w.E)]

        def gemms():
            for e in range(w.E):
                if counts[e]:
                    xs[e] @ wg[e]
                    xs[e] @ wu[e]
                    hs[e] @ wd[e]

        t_gemm = timed(gemms)
        fl = 6.0 * w.S * w.k * w.D * w.F
        results[name] = {"library_ms": round(t_lib, 4), "torch_forward_ms": round(t_ref, 4),
                         "torch_gemms_only_ms": round(t_gemm, 4),
                         "library_tflops": round(fl / t_lib / 1e9, 1),
                         "torch_gemms_only_tflops": round(fl / t_gemm / 1e9, 1)}
        del inp, ws, out, xs, hs
        torch.cuda.empty_cache()
    return {"metric": "expert-MLP forward: library against a torch per-expert (cuBLAS) forward",
            "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "data": "synthetic", "l2": "flushed before every call", "workloads": results}


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
        pt = {"R": R, "E": E, "us": round(t_ms * 1e3, 2), "GB/s": round(gbs, 1),
              "frac_of_hbm_peak": round(gbs / pk["hbm_gbs"], 3)}
        if args.map_torch_ref:
            pt["torch_ref_us"] = round(torch_map_reference_ms(te, E, flush, args.warmup, reps) * 1e3, 2)
        points.append(pt)
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
    clocks = clk.summary()
    tf_peak, tf_kind = tensor_peak(w.dtype, clocks, ms * args.steps / 1e3)
    tflops = flop / (ms * 1e-3) / 1e12
    return {"metric": "MoE-layer backward tokens/s and TFLOP/s (bf16)", "value": w.S / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "S": w.S, "D": w.D, "F": w.F, "E": w.E, "k": w.k,
                       "l2": "inputs larger than L2 (all expert weights streamed every step)"},
            "tflops": tflops, "flop_per_step": flop,
            "tflops_frac": {"of_measured_peak": tflops / tf_peak, "peak_kind": tf_kind,
                            "of_nominal": tflops / 2250.0},
            "extra_flop_recompute": 4.0 * R * w.D * w.F, "stage_ms": stage,
            # dominant stage: the weight gradients of the gate and up projections (two grouped
            # weight-gradient GEMMs, 2 R D F FLOPs each)
            "roofline": {"kernel": "dW_gate_e_and_dW_up (grouped_wgrad_kernel x2)",
                         "bound": "tensor",
                         "achieved": 4.0 * R * w.D * w.F / (stage["dW_gate_e_and_dW_up"] * 1e-3) / 1e12,
                         "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": 4.0 * R * w.D * w.F / (stage["dW_gate_e_and_dW_up"] * 1e-3) / 1e12
                         / tf_peak,
                         "peak_kind": tf_kind, "traffic": None},
            "gpu_launches": launches * args.steps, "clocks": clocks}


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
        clocks = clk.summary()
        tf_peak, tf_kind = tensor_peak(w.dtype, clocks, ms_max * args.steps / 1e3)
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
                             "peak": tf_peak, "unit": "TFLOP/s",
                             "frac": (fl["gemm1"] + fl["gemm2"]) / (stage["experts"] * 1e-3) / 1e12
                             / tf_peak, "peak_kind": tf_kind, "traffic": None},
                "clocks": clocks}
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
    clocks = clk.summary()
    tf_peak, tf_kind = tensor_peak("bf16", clocks, ms * args.steps / 1e3)
    tflops = flop / (ms * 1e-3) / 1e12
    att = fl["attention"] / (stage["attention"] * 1e-3) / 1e12
    return {"metric": "MoA-layer fwd tokens/s and TFLOP/s (bf16)", "value": w.S / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "S": w.S, "D": w.D, "H": w.H, "dh": w.dh, "E": w.E,
                       "k": w.k, "l2": "inputs larger than L2 (expert weights streamed)"},
            "tflops": tflops, "flop_per_step": flop, "flop_by_stage": fl,
            "tflops_frac": {"of_measured_peak": tflops / tf_peak, "peak_kind": tf_kind,
                            "of_nominal": tflops / 2250.0},
            "roofline": {"kernel": "attention core", "bound": "tensor", "achieved": att,
                         "peak": tf_peak, "unit": "TFLOP/s", "frac": att / tf_peak,
                         "peak_kind": tf_kind, "traffic": None},
            "stage_ms": stage, "gpu_launches": launches * args.steps, "clocks": clocks,
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
    ap.add_argument("--forward-torch-ref", action="store_true",
                    help="instead of the forward: time moe_mlp_forward beside a torch per-expert "
                         "(cuBLAS) forward on every workload")
    ap.add_argument("--map-torch-ref", action="store_true",
                    help="with --map-sweep: also time the same map built from torch calls "
                         "(stable sort, bincount, cumsum, scatter) at every point")
    ap.add_argument("--backward", action="store_true",
                    help="instead of the forward: time moe_mlp_backward on --workload")
    ap.add_argument("--moa", action="store_true",
                    help="instead of the MLP forward: time moe_moa_forward (Mixture of Attention)")
    ap.add_argument("--ep", action="store_true",
                    help="instead of the replicated forward: the expert-parallel forward, experts "
                         "split over the ranks (all-to-all dispatch and combine over NCCL)")
    ap.add_argument("--map-points", default="",
                    help="with --map-sweep: only these points, 'log2R:E,...' (e.g. 26:256)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="headline workload only (no `workloads` object with the other configs)")
    ap.add_argument("--record-traffic", default="", metavar="CSV",
                    help="instead of timing: record the DRAM bytes per launch of each kernel "
                         "class in an ncu CSV into profiles/dram_traffic.json for --workload")
    ap.add_argument("--traffic-command", default="",
                    help="with --record-traffic: the ncu command line that wrote the CSV")
    args = ap.parse_args()
    if args.record_traffic:
        out = record_traffic(args.record_traffic, args.workload, args.traffic_command)
        print(json.dumps(out, indent=1))
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.map_sweep:
        print(json.dumps(map_sweep(args)), flush=True)
        return
    if args.forward_torch_ref:
        print(json.dumps(forward_torch_reference(args)), flush=True)
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
