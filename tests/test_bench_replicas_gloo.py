"""The bench's multi-rank path on the CPU: two ranks over gloo run bench_ours against the same
stand-ins for the CUDA library and torch.cuda as the single-rank dry run. Every rank must take the
same collective steps (barriers around the timed regions, max-reductions of the times), rank 0's
line must count the tokens of both ranks over the slowest rank's time, and only a one-rank run
carries the `workloads` object. Timings are the stand-in's, so only the bookkeeping is checked."""
import contextlib
import os
import socket
import sys
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, TESTS)
    import bench
    import moe_workloads as W
    import test_bench_dryrun as dry

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # the dry run's stand-ins, set by hand (no pytest fixture in a spawned process)
        torch.cuda.Event = dry._Event
        torch.cuda.synchronize = lambda *a, **k: None
        torch.cuda.current_stream = lambda *a, **k: dry._Stream()
        torch.cuda.Stream = lambda *a, **k: dry._Stream()
        torch.cuda.stream = lambda s: contextlib.nullcontext()
        torch.cuda.current_device = lambda: 0
        torch.cuda.empty_cache = lambda: None
        torch.Tensor.pin_memory = lambda self: self
        real_device = torch.device
        bench.torch.device = lambda *a, **k: real_device("cpu")
        sys.modules["sparse_mixture_experts_02_b200"] = dry._fake_library()
        base = W.WORKLOADS["mixtral_prefill"]
        w = W.Workload(base.name, S=64, D=64, F=32, E=base.E, k=base.k, dtype=base.dtype,
                       router_std=base.router_std, zipf_s=base.zipf_s)
        args = types.SimpleNamespace(steps=2, warmup=3, no_workloads=False, no_cpu_baseline=True,
                                     cpu_budget_s=1.0)
        line = bench.bench_ours(args, w, ws, rank, 0)
        out[rank] = line
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(300)
def test_bench_two_ranks_over_gloo():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True,
                           start_method="spawn")
        lines = dict(out)
    assert lines[1] is None  # only rank 0 reports
    line = lines[0]
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["parallelism"] == "replicas2"
    # the stand-in's events report 0.25 ms per interval; the loop spans the 2 timed steps
    assert line["value"] > 0 and abs(line["value"] - 64 * 2 / (line["ms_per_step"] / 1000.0)) \
        < 1e-6 * line["value"]
    assert "workloads" not in line  # the other workloads are measured in one-rank runs only
    assert line["e2e"]["value"] > 0
