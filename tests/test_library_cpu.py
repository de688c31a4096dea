"""The C-ABI library loads, exports every symbol include/moe.h declares, and its host-side logic
(workspace sizing, argument checks) behaves, all without a GPU. No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def moe():
    from sparse_mixture_experts_02_b200 import build
    build.build()
    import sparse_mixture_experts_02_b200 as m
    return m


def test_header_symbols_exported(moe):
    names = _header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(moe.lib, n), n
    assert sorted(moe.EXPORTS) == names


def test_debug_library_exports_the_same_symbols(moe):
    """The MOE_DEBUG build (device bounds checks) has every entry point of the release build and
    says which build it is."""
    names = _header_functions()
    dbg = moe.debug_lib()
    for n in names:
        assert hasattr(dbg, n), n
    assert dbg.moe_debug_build() == 1
    assert moe.lib.moe_debug_build() == 0


def test_library_targets_sm100a_only():
    from sparse_mixture_experts_02_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)


def test_workspace_sizes(moe):
    lib = moe.lib
    # map scratch grows with S*k*E; forward holds h [S*k, F]
    small = moe.workspace_size("mlp_forward", 512, 256, 512, 8, 2, moe.MOE_F32)
    assert small >= 512 * 2 * 512 * 4
    big = moe.workspace_size("mlp_forward", 4096, 4096, 14336, 8, 2, moe.MOE_BF16)
    assert big >= 8192 * 14336 * 2
    assert moe.workspace_size("sparse_map", 0, 0, 0, 8, 2, 1) >= 256
    assert moe.workspace_size("scatter_linear", 10, 8, 8, 4, 2, 1) == 256
    assert moe.workspace_size("nope", 10, 8, 8, 4, 2, 1) == 0
    assert moe.workspace_size("mlp_forward", 10, 8, 8, 300, 2, 1) == 0   # E > 256
    assert moe.workspace_size("mlp_forward", 10, 8, 8, 4, 9, 1) == 0     # k > 8
    assert moe.workspace_size("mlp_forward", 2**30, 8, 8, 4, 2, 1) == 0  # S*k >= 2^31
    # views are 256-byte aligned, disjoint and inside the workspace
    S, D, F, E, k = 100, 64, 96, 5, 2
    total = moe.workspace_size("mlp_forward", S, D, F, E, k, moe.MOE_BF16)
    names = ["top_experts", "top_weights", "expert_counts", "expert_offsets", "sparse_rows",
             "sorted_rows", "h"]
    sizes = [S * k * 4, S * k * 4, E * 4, (E + 1) * 4, S * k * 4, S * k * 4, S * k * F * 2]
    spans = []
    for n, sz in zip(names, sizes):
        off = moe.workspace_view(n, S, D, F, E, k, moe.MOE_BF16)
        assert off >= 256 and off % 256 == 0
        assert off + sz <= total
        spans.append((off, off + sz))
    spans.sort()
    for a, b in zip(spans, spans[1:]):
        assert a[1] <= b[0]
    assert moe.workspace_view("bogus", S, D, F, E, k, 1) == -1


def test_forward_workspace_slot_ordered_x(moe):
    # bf16 forwards with experts of >= 384 rows on average and F >= 2048 copy x to slot order
    # before GEMM1: their workspace carries an "x_sorted" region [S*k, D] after h
    def size_view(S, D, F, E, k, dt):
        return (moe.workspace_size("mlp_forward", S, D, F, E, k, dt),
                moe.workspace_view("x_sorted", S, D, F, E, k, dt),
                moe.workspace_view("h", S, D, F, E, k, dt))
    S, D, F, E, k = 4096, 4096, 14336, 8, 2          # the Mixtral-shaped prefill layer
    total, xs, h = size_view(S, D, F, E, k, moe.MOE_BF16)
    R = S * k
    assert xs >= h + R * F * 2 and xs % 256 == 0 and xs + R * D * 2 <= total
    # the same layer without the copy is that region smaller, everything before it unchanged
    for S2, F2, E2, dt in [(192 * 8 - 1, F, E, moe.MOE_BF16),   # R / E = 383
                           (S, 2040, E, moe.MOE_BF16),          # F < 2048
                           (S, F, E, moe.MOE_F32)]:             # fp32
        t2, x2, h2 = size_view(S2, D, F2, E2, k, dt)
        assert x2 == -1
    t_edge, x_edge, _ = size_view(192 * 8, D, 2048, E, k, moe.MOE_BF16)  # R / E = 384, F = 2048
    assert x_edge > 0 and x_edge + 192 * 8 * k * D * 2 <= t_edge
    # the expert-parallel forward gathers its rows on load and has no such region
    t_ep = moe.workspace_size("expert_mlp_forward", R, D, F, E, 1, moe.MOE_BF16)
    assert t_ep < total


@pytest.mark.parametrize("R", [16385, 32768, 75264, 75265, 98304, 300000, 602112, 602113,
                               1 << 22, (1 << 22) + 1])
@pytest.mark.parametrize("E", [8, 256])
def test_sparse_map_workspace_bound(moe, R, E):
    """The grid map keeps (blocks + 1) x E int32 counters. Blocks: ceil(R / 4096) from 148 such
    blocks up (602,113 routes); below that the warp units shrink, with at most 294 blocks."""
    got = moe.workspace_size("sparse_map", R, 0, 0, E, 1, 1)
    bound = 256 + (max(-(-R // 4096), 294) + 1) * E * 4
    assert 256 < got <= bound + 255
    if R > 602112:
        assert got >= 256 + (-(-R // 4096) + 1) * E * 4


def test_host_argument_errors_before_any_launch(moe):
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: validation fails first
    # k > E
    rc = lib.moe_route_topk(fake, fake, None, 8, 64, 4, 5, moe.MOE_BF16, fake, fake, None)
    assert rc == -1 and b"k must be" in lib.moe_last_error()
    # D not a multiple of 8
    rc = lib.moe_route_topk(fake, fake, None, 8, 60, 4, 2, moe.MOE_BF16, fake, fake, None)
    assert rc == -1 and b"D must be" in lib.moe_last_error()
    # misaligned pointer
    rc = lib.moe_route_topk(P(4097), fake, None, 8, 64, 4, 2, moe.MOE_BF16, fake, fake, None)
    assert rc == -1 and b"aligned" in lib.moe_last_error()
    # bad dtype
    rc = lib.moe_route_topk(fake, fake, None, 8, 64, 4, 2, 7, fake, fake, None)
    assert rc == -2
    # workspace too small / null / misaligned
    rc = lib.moe_sparse_map(fake, 8, 2, 4, fake, fake, fake, fake, fake, 16, None)
    assert rc == -3 and b"too small" in lib.moe_last_error()
    rc = lib.moe_sparse_map(fake, 8, 2, 4, fake, fake, fake, fake, None, 1 << 20, None)
    assert rc == -3
    rc = lib.moe_sparse_map(fake, 8, 2, 4, fake, fake, fake, fake, P(4096 + 64), 1 << 20, None)
    assert rc == -3 and b"aligned" in lib.moe_last_error()
    # E out of range, S negative, S*k too large
    rc = lib.moe_sparse_map(fake, 8, 2, 300, fake, fake, fake, fake, fake, 1 << 20, None)
    assert rc == -1
    rc = lib.moe_sparse_map(fake, -1, 2, 4, fake, fake, fake, fake, fake, 1 << 20, None)
    assert rc == -1
    rc = lib.moe_sparse_map(fake, 2**30, 4, 4, fake, fake, fake, fake, fake, 1 << 20, None)
    assert rc == -1
    # null required pointer
    rc = lib.moe_mlp_forward(fake, None, None, fake, fake, fake, 8, 64, 64, 4, 2, 1, fake, fake,
                             1 << 30, None)
    assert rc == -1 and b"w_gate is null" in lib.moe_last_error()
    # profile events arguments
    assert lib.moe_profile_events(None, 3) == -1
    assert lib.moe_profile_events(None, 0) == 0
    # debug wait limit range
    assert lib.moe_debug_wait_timeout(0, fake, 256, None) == -1


def test_python_binding_rejects_cpu_tensors(moe):
    import torch
    x = torch.zeros(4, 8)
    with pytest.raises(ValueError):
        moe.route_topk(x, torch.zeros(8, 4), 2)
