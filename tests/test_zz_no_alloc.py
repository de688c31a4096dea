"""moe_sparse_map_noalloc: the sparse map for callers that cannot obtain device scratch memory
(plugin-style interfaces with fixed input/output bindings, or runtimes whose device memory is all
held in their own pool). Its scratch is a fixed array inside the library, so the call allocates
nothing. This file is collected last on purpose: it must pass both on its own in a fresh process
and after every other test.

Checked through the C ABI against moe_sparse_map with a workspace, bit-exactly:
- two calls in a row that both run the multi-block count / scan / assign kernels (the path that
  keeps per-block counters in the fixed array): first a 256-expert routing whose counters fill the
  array to exactly its limit, then a 64-expert routing of a different size, so that a counter left
  over from the first call and read by the second would show;
- the size limit itself: the largest accepted size uses exactly the 1 MiB of counters, and one
  more map block above it is rejected before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_workloads as W

pytestmark = pytest.mark.gpu

LIMIT = 1 << 20          # bytes of per-(block, expert) counters in the fixed array
BLOCK_ROUTES = 4096      # routes per map block at these sizes
SMALL_PATH_ROUTES = 16384  # up to here the map runs as one block without the counters


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(S, k, E):
    dev = torch.device("cuda")
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((S * k,), -7, dtype=torch.int32, device=dev),
            torch.full((S * k,), -7, dtype=torch.int32, device=dev))


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _run_noalloc(moe, te, E):
    S, k = te.shape
    outs = _outputs(S, k, E)
    rc = moe.lib.moe_sparse_map_noalloc(_p(te), S, k, E, *[_p(o) for o in outs], _stream())
    assert rc == 0, moe.lib.moe_last_error()
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


def _run_with_workspace(moe, te, E):
    S, k = te.shape
    outs = _outputs(S, k, E)
    ws = moe.alloc_workspace(moe.workspace_size("sparse_map", S, 0, 0, E, k, 1), te.device)
    rc = moe.lib.moe_sparse_map(_p(te), S, k, E, *[_p(o) for o in outs], _p(ws), ws.numel(),
                                _stream())
    assert rc == 0, moe.lib.moe_last_error()
    moe.check_device_status(ws)
    return [o.cpu().numpy() for o in outs]


def _counter_bytes(R, E):
    return (-(-R // BLOCK_ROUTES) + 1) * E * 4


# S*k = 4,190,208 routes at E = 256: 1023 map blocks, (1023 + 1) * 256 * 4 bytes = 1 MiB exactly
S_EDGE, K_EDGE, E_EDGE = 523776, 8, 256


def test_noalloc_matches_workspace_map_twice(moe):
    assert _counter_bytes(S_EDGE * K_EDGE, E_EDGE) == LIMIT
    cases = [
        (W.make_top_experts(S_EDGE, K_EDGE, E_EDGE, seed=11, mode="stride", device="cuda"),
         E_EDGE),
        (W.make_top_experts(20001, 6, 64, seed=12, mode="zipf").cuda(), 64),
    ]
    for te, E in cases:          # two calls in a row, both on the multi-block path
        assert te.numel() > SMALL_PATH_ROUTES
        got = _run_noalloc(moe, te, E)
        ref = _run_with_workspace(moe, te, E)
        for name, a, b in zip(("counts", "offsets", "sparse_rows", "sorted_rows"), got, ref):
            assert np.array_equal(a, b), name
        assert got[1][E] == te.numel()
        assert np.array_equal(got[0], np.bincount(te.cpu().numpy().reshape(-1), minlength=E))


def test_noalloc_rejects_one_block_beyond_its_scratch(moe):
    # one more map block than the exact-limit case above: (1024 + 1) * 256 * 4 bytes > 1 MiB
    S = S_EDGE + 1
    assert _counter_bytes(S * K_EDGE, E_EDGE) > LIMIT
    te = torch.zeros((S, K_EDGE), dtype=torch.int32, device="cuda")
    outs = _outputs(S, K_EDGE, E_EDGE)
    rc = moe.lib.moe_sparse_map_noalloc(_p(te), S, K_EDGE, E_EDGE, *[_p(o) for o in outs],
                                        _stream())
    assert rc == -1
    assert b"scratch" in moe.lib.moe_last_error()
    torch.cuda.synchronize()
    # nothing was launched: the outputs keep their fill value
    assert int(outs[0][0].item()) == -7
    assert int(outs[2][0].item()) == -7
