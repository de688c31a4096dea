"""The bench's Python paths on the CPU: bench_ours runs against a stand-in for the CUDA library and
for torch.cuda's events and streams (no GPU, no kernel), and its JSON line carries every key the
bench contract asks for, for the headline workload and for each entry of `workloads`. Timings here
are the stand-in's, so only the structure and the bookkeeping are checked."""
import contextlib
import os
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import moe_workloads as W  # noqa: E402


class _Event:
    def __init__(self, *a, **k):
        pass

    def record(self, *a):
        pass

    def elapsed_time(self, other):
        return 0.25


class _Stream:
    cuda_stream = 0

    def wait_event(self, e):
        pass


def _fake_library(launches_per_step=4):
    lib = types.ModuleType("sparse_mixture_experts_02_b200")

    class ForwardWorkspace:
        def __init__(self, S, D, F, E, k, dtype, dev):
            self.shape = (S, D, F, E, k)

        def view(self, name):
            S, D, F, E, k = self.shape
            assert name == "expert_counts"
            c = torch.full((E,), S * k // E, dtype=torch.int32)
            c[0] += S * k - int(c.sum())
            return c

    calls = {"forward": 0}

    def mlp_forward(x, w_gate, w_gate_e, w_up, w_down, k, logit_bias=None, out=None, ws=None):
        calls["forward"] += 1
        assert out is not None and out.shape == (x.shape[0], w_gate_e.shape[1])
        out.copy_(x.float())  # deterministic, so the bench's host-vs-device check compares values
        return out

    lib.ForwardWorkspace = ForwardWorkspace
    lib.mlp_forward = mlp_forward
    lib.profile_events = lambda ev: None
    lib.check_device_status = lambda ws: None
    lib.last_launch_count = lambda: launches_per_step
    lib.calls = calls
    return lib


@pytest.fixture
def cpu_bench(monkeypatch):
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "Stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    real_device = torch.device
    monkeypatch.setattr(bench.torch, "device", lambda *a, **k: real_device("cpu"))
    lib = _fake_library()
    monkeypatch.setitem(sys.modules, "sparse_mixture_experts_02_b200", lib)
    # small stand-ins with every workload's E, k, dtype and router, so the run stays quick
    small = {n: W.Workload(w.name, S=min(w.S, 64), D=64, F=32, E=w.E, k=w.k, dtype=w.dtype,
                           router_std=w.router_std, zipf_s=w.zipf_s)
             for n, w in W.WORKLOADS.items()}
    monkeypatch.setattr(W, "WORKLOADS", small)
    return lib, small


def _args(**kw):
    a = types.SimpleNamespace(steps=2, warmup=3, no_workloads=False, no_cpu_baseline=True,
                              cpu_budget_s=1.0)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_bench_line_has_every_contract_key(cpu_bench):
    lib, small = cpu_bench
    w = small["mixtral_prefill"]
    line = bench.bench_ours(_args(), w, 1, 0, 0)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "workloads"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["config"] == bench.workload_config(w, 1)
    assert line["gpu_launches"] == 4 * 2
    r = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic", "other"):
        assert key in r, key
    assert r["bound"] in ("hbm", "tensor") and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    e2e = line["e2e"]
    assert e2e["h2d_bytes_per_step"] == w.S * w.D * 2 and e2e["d2h_bytes_per_step"] == w.S * w.D * 4
    assert set(line["stage_ms"]) == set(bench.STAGES)
    # every other workload is measured, each with its own roofline and clocks
    assert set(line["workloads"]) == set(small) - {w.name}
    for name, ent in line["workloads"].items():
        for key in ("ms_per_step", "tokens_per_s", "tflops", "gbs", "roofline", "clocks",
                    "stage_ms", "expert_hist", "l2"):
            assert key in ent, (name, key)
    # the warm-up and timed forwards of every workload, and the e2e leg of the headline
    per = 2 + 3
    assert lib.calls["forward"] == per * 2 + per * (len(small) - 1)


def test_bench_line_without_other_workloads(cpu_bench):
    lib, small = cpu_bench
    line = bench.bench_ours(_args(no_workloads=True), small["e128"], 1, 0, 0)
    assert "workloads" not in line
    assert line["config"]["workload"] == "e128"
