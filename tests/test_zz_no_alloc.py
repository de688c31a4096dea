"""moe_sparse_map_noalloc: the sparse map for callers that cannot obtain device scratch memory
(plugin-style interfaces with fixed input/output bindings, or runtimes whose device memory is all
held in their own pool). Its scratch is a fixed array inside the library, so the call allocates
nothing. This file is collected last on purpose: it must pass both on its own in a fresh process
and after every other test.

Checked through the C ABI: two calls in a row (different routings, so a stale result from the
first call would show) give outputs bit-identical to moe_sparse_map with a workspace, and sizes
beyond the fixed scratch are rejected before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_workloads as W

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(S, k, E):
    dev = torch.device("cuda")
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((S * k,), -7, dtype=torch.int32, device=dev),
            torch.full((S * k,), -7, dtype=torch.int32, device=dev))


def _run_noalloc(moe, te, E):
    S, k = te.shape
    outs = _outputs(S, k, E)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib.moe_sparse_map_noalloc(_p(te), S, k, E, *[_p(o) for o in outs], stream)
    assert rc == 0, moe.lib.moe_last_error()
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


def _run_with_workspace(moe, te, E):
    S, k = te.shape
    outs = _outputs(S, k, E)
    ws = moe.alloc_workspace(moe.workspace_size("sparse_map", S, 0, 0, E, k, 1), te.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib.moe_sparse_map(_p(te), S, k, E, *[_p(o) for o in outs], _p(ws), ws.numel(),
                                stream)
    assert rc == 0, moe.lib.moe_last_error()
    moe.check_device_status(ws)
    return [o.cpu().numpy() for o in outs]


def test_noalloc_matches_workspace_map_twice(moe):
    cases = [(W.make_top_experts(20000, 6, 64, seed=11, mode="zipf"), 64),
             (W.make_top_experts(4096, 2, 8, seed=12, mode="uniform"), 8)]
    for te_cpu, E in cases:          # two calls in a row
        te = te_cpu.cuda()
        got = _run_noalloc(moe, te, E)
        ref = _run_with_workspace(moe, te, E)
        for name, a, b in zip(("counts", "offsets", "sparse_rows", "sorted_rows"), got, ref):
            assert np.array_equal(a, b), name
        assert got[1][E] == te.numel()


def test_noalloc_rejects_sizes_beyond_its_scratch(moe):
    # (ceil(S*k/4096) + 1) * E * 4 bytes must fit in 1 MiB: 2^23 routes at E = 256 need 2 MiB
    te = torch.zeros((1 << 20, 8), dtype=torch.int32, device="cuda")
    outs = _outputs(1 << 20, 8, 256)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib.moe_sparse_map_noalloc(_p(te), 1 << 20, 8, 256, *[_p(o) for o in outs], stream)
    assert rc == -1
    assert b"scratch" in moe.lib.moe_last_error()
    # nothing was launched: the outputs keep their fill value
    assert int(outs[0][0].item()) == -7
