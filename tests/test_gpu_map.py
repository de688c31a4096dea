"""Sparse map on the GPU against the oracle's counting sort: bit-exact on every output, plus the
invariants of "4. Correctness Validation" in "Add scalable sparse map kernel for large MoE models
(128+ experts)" (unique rows, rows inside their expert's range, histogram counts, non-overlapping
ranges, deterministic across runs), over that page's expert-count grid and the route counts of
every workload."""
import numpy as np
import pytest
import torch

import moe_workloads as W
from test_oracle_pins import check_map_invariants

pytestmark = pytest.mark.gpu


def _run(moe, te_cpu, E):
    te = te_cpu.to("cuda")
    out = moe.sparse_map(te, E)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in out]


def _compare(oracle_lib, moe, te_cpu, E):
    got = _run(moe, te_cpu, E)
    ref = oracle_lib.sparse_map(te_cpu.numpy(), E)
    for name, a, b in zip(("counts", "offsets", "sparse_rows", "sorted_rows"), got, ref):
        assert np.array_equal(a, b), f"{name} differs at {np.nonzero(a != b)[0][:10]}"
    check_map_invariants(te_cpu.numpy(), E, *got)
    return got


@pytest.mark.parametrize("E", [4, 8, 16, 32, 64, 96, 128, 256])
@pytest.mark.parametrize("mode", ["uniform", "zipf"])
def test_map_expert_grid(oracle_lib, moe, E, mode):
    k = min(4, E)
    te = W.make_top_experts(3001, k, E, seed=E + 7, mode=mode)
    _compare(oracle_lib, moe, te, E)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_map_workload_sizes(oracle_lib, moe, name):
    w = W.WORKLOADS[name]
    mode = "zipf" if w.zipf_s > 0 else "uniform"
    te = W.make_top_experts(w.S, w.k, w.E, seed=1, mode=mode)
    _compare(oracle_lib, moe, te, w.E)


def test_map_deterministic(oracle_lib, moe):
    te = W.make_top_experts(40000, 6, 64, seed=3, mode="zipf")
    first = _compare(oracle_lib, moe, te, 64)
    for _ in range(3):
        again = _run(moe, te, 64)
        for a, b in zip(first, again):
            assert np.array_equal(a, b)


@pytest.mark.parametrize("S,k,E", [(1, 1, 1), (1, 3, 7), (511, 1, 5), (512, 1, 5), (513, 1, 5),
                                   (70000, 2, 3)])
def test_map_edges(oracle_lib, moe, S, k, E):
    te = W.make_top_experts(S, k, E, seed=S, mode="any")
    _compare(oracle_lib, moe, te, E)


# One-block path: the block runs ceil(R / (32 IT)) warps of IT steps, IT the smallest power of two
# that keeps the warps at or below 32. Each pair straddles a switch of IT (1, 2, 4, 8, 16).
@pytest.mark.parametrize("R", [1, 31, 33, 1024, 1025, 2048, 2049, 4096, 4097, 8192, 8193, 16384])
@pytest.mark.parametrize("E", [8, 256])
def test_map_one_block_step_switches(oracle_lib, moe, R, E):
    te = W.make_top_experts(R, 1, E, seed=R * 3 + E, mode="any")
    _compare(oracle_lib, moe, te, E)


def test_map_all_one_expert_and_empty(oracle_lib, moe):
    te = W.make_top_experts(5000, 4, 32, mode="one")
    counts, offsets, _, _ = _compare(oracle_lib, moe, te, 32)
    assert counts[0] == 20000 and counts[1:].sum() == 0
    # S = 0: counts and offsets all zero
    got = _run(moe, torch.zeros((0, 2), dtype=torch.int32), 6)
    assert got[0].tolist() == [0] * 6 and got[1].tolist() == [0] * 7


def test_map_large_route_count(oracle_lib, moe):
    te = W.make_top_experts(1 << 18, 8, 256, seed=9, mode="zipf")  # 2^21 routes
    _compare(oracle_lib, moe, te, 256)


# Grid-parallel path: routes per count/assign block = 8 warps x 512; sizes one past and one short
# of block multiples, and the first size past the one-block path.
@pytest.mark.parametrize("R", [16385, 4096 * 5 - 1, 4096 * 5 + 1, 4096 * 64, 4096 * 1024 + 7])
def test_map_block_edges(oracle_lib, moe, R):
    te = W.make_top_experts(R, 1, 64, seed=R, mode="any")
    _compare(oracle_lib, moe, te, 64)


# Below 148 blocks of 8 x 512 routes the grid path shrinks its warp units to 256, 128, 64 or 32
# routes (148 blocks = one per SM). Each pair straddles one switch of the unit size: the last
# route count that keeps the smaller unit and the first that takes the larger one.
@pytest.mark.parametrize("R", [75264, 75265, 150528, 150529, 301056, 301057, 602112, 602113])
@pytest.mark.parametrize("E", [8, 256])
def test_map_unit_size_switches(oracle_lib, moe, R, E):
    te = W.make_top_experts(R, 1, E, seed=R + E, mode="any")
    _compare(oracle_lib, moe, te, E)


def test_map_bad_expert_id_grid_path(moe):
    """An out-of-range id on the grid path with 64-route units (R = 98304): reported by the
    device status, its route gets slot -1, every other route is still mapped."""
    S, k, E = 16384, 6, 64
    te = W.make_top_experts(S, k, E, seed=4, mode="zipf").clone()
    te[9000, 3] = E
    tg = te.to("cuda")
    ws = moe.alloc_workspace(moe.workspace_size("sparse_map", S, 0, 0, E, k, 1), tg.device)
    _, _, sparse_rows, _ = moe.sparse_map(tg, E, ws=ws)
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_status(ws)
    assert ei.value.code == -5
    sp = sparse_rows.cpu().numpy()
    assert sp[9000 * k + 3] == -1
    valid = np.delete(np.arange(S * k), 9000 * k + 3)
    assert np.array_equal(np.sort(sp[valid]), np.arange(S * k - 1))


@pytest.mark.parametrize("E,mode", [(8, "stride"), (64, "zipf"), (128, "stride"), (256, "zipf")])
def test_map_2pow20_routes(oracle_lib, moe, E, mode):
    te = W.make_top_experts(1 << 17, 8, E, seed=E, mode=mode)
    _compare(oracle_lib, moe, te, E)


def test_map_2pow23_routes_256_experts(oracle_lib, moe):
    te = W.make_top_experts(1 << 20, 8, 256, seed=23, mode="stride")
    _compare(oracle_lib, moe, te, 256)


def test_map_bad_expert_id_is_reported(moe):
    te = W.make_top_experts(100, 2, 8, seed=2).clone()
    te[17, 1] = 8
    te[50, 0] = -3
    tg = te.to("cuda")
    need = moe.workspace_size("sparse_map", 100, 0, 0, 8, 2, 1)
    ws = moe.alloc_workspace(need, tg.device)
    counts = torch.empty(8, dtype=torch.int32, device="cuda")
    offsets = torch.empty(9, dtype=torch.int32, device="cuda")
    sp = torch.empty(200, dtype=torch.int32, device="cuda")
    so = torch.empty(200, dtype=torch.int32, device="cuda")
    import ctypes
    rc = moe.lib.moe_sparse_map(ctypes.c_void_p(tg.data_ptr()), 100, 2, 8,
                                ctypes.c_void_p(counts.data_ptr()),
                                ctypes.c_void_p(offsets.data_ptr()), ctypes.c_void_p(sp.data_ptr()),
                                ctypes.c_void_p(so.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_status(ws)
    assert ei.value.code == -5
    # the valid routes are still mapped, the bad ones get -1
    spn = sp.cpu().numpy()
    assert spn[17 * 2 + 1] == -1 and spn[50 * 2] == -1
    assert counts.sum().item() == 198
    # the status clears on the next call
    moe.sparse_map(W.make_top_experts(100, 2, 8, seed=2).to("cuda"), 8, ws=ws)
    moe.check_device_status(ws)


@pytest.mark.parametrize("E", [8, 256])
def test_map_unaligned_buffers(oracle_lib, moe, E):
    """top_experts and the two row arrays starting 4 bytes past a 16-byte boundary (the grid path's
    vector loads and stores then take their one-route-at-a-time form): same map as the oracle."""
    S, k = 40001, 4
    te_cpu = W.make_top_experts(S, k, E, seed=E + 1, mode="stride")
    R = S * k
    te_buf = torch.empty(R + 1, dtype=torch.int32, device="cuda")
    te_buf[1:] = te_cpu.reshape(-1).to("cuda")
    te = te_buf[1:]
    assert te.data_ptr() % 16 == 4
    rows = torch.empty(2 * (R + 1), dtype=torch.int32, device="cuda")
    sparse_rows, sorted_rows = rows[1:R + 1], rows[R + 2:]
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    need = moe.workspace_size("sparse_map", S, 0, 0, E, k, 1)
    ws = moe.alloc_workspace(need, te.device)
    lib = moe.lib
    rc = lib.moe_sparse_map(te.data_ptr(), S, k, E, counts.data_ptr(), offsets.data_ptr(),
                            sparse_rows.data_ptr(), sorted_rows.data_ptr(), ws.data_ptr(),
                            ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    moe.check_device_status(ws)
    got = [t.cpu().numpy() for t in (counts, offsets, sparse_rows, sorted_rows)]
    ref = oracle_lib.sparse_map(te_cpu.numpy(), E)
    for name, a, b in zip(("counts", "offsets", "sparse_rows", "sorted_rows"), got, ref):
        assert np.array_equal(a, b), name


@pytest.mark.parametrize("E", [8, 200])
def test_map_past_2pow23_routes(oracle_lib, moe, E):
    """2050 map blocks of 4096 routes: the scan of the block counts takes its row form (more than
    2048 blocks); eight experts assign with a lane per run of routes, 200 with a lane per route."""
    S = (2050 * 4096 - 3000) // 8
    te = W.make_top_experts(S, 8, E, seed=E + 5, mode="stride")
    _compare(oracle_lib, moe, te, E)
