"""ParallelLinear(X, W, I, G) on the tcgen05 grouped GEMM against the oracle, for every input /
output mode, both dtypes, with and without router weights, at sizes that span several M, N and K
tiles with ragged tails, plus empty experts.

Source: "ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs", "1. The Anatomy of
ParallelLinear" and "The ParallelLinear Core Abstraction" figure (Steps 1-3).

Tolerances: bf16 inputs are exact in fp32 and the tensor cores accumulate in fp32, so a float32
result differs from the fp64 oracle by accumulation rounding only (~1e-6 relative); a bf16
result adds one rounding (2^-9 relative). fp32 inputs multiply as tf32 (10-bit mantissa,
~1e-3 relative).
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import rel_frob

pytestmark = pytest.mark.gpu


def _tol(dtype, scatter_out):
    if dtype == "f32":
        return 6e-3
    return 2e-5 if scatter_out else 6e-3


SHAPES = [
    # S, k, E, Din, Dout, mode
    (700, 2, 3, 200, 328, "uniform"),    # 4 M tiles per expert, K tail, N tail
    (300, 4, 9, 64, 512, "zipf"),        # skew, empty experts likely, N exactly 2 tiles
    (129, 1, 1, 8, 8, "uniform"),        # smallest dims, one expert, 2 M tiles
    (1000, 6, 64, 136, 264, "zipf"),
]


@pytest.fixture(params=["cta1", "cta2"])
def gemm_kernel(request, monkeypatch):
    """Runs a test once on the one-CTA grouped GEMM and once on the CTA-pair (cta_group::2)
    kernel; the library reads MOE_GEMM_2SM at every launch."""
    monkeypatch.setenv("MOE_GEMM_2SM", "1" if request.param == "cta2" else "0")
    return request.param


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("gather_in,scatter_out", [(True, True), (False, True), (True, False),
                                                   (False, False)])
@pytest.mark.parametrize("gated", [True, False])
def test_scatter_linear(oracle_lib, moe, gemm_kernel, shape, dtype, gather_in, scatter_out, gated):
    S, k, E, Din, Dout, mode = shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gen = torch.Generator().manual_seed(S + E + Din)
    te = W.make_top_experts(S, k, E, seed=S, mode=mode)
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    rows = S if gather_in else S * k
    X = torch.randn(rows, Din, generator=gen).to(tdt)
    Wt = (torch.randn(E, Din, Dout, generator=gen) * 0.05).to(tdt)
    g = torch.rand(S * k, generator=gen) if gated else None
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, g, gather_in=gather_in,
                                    scatter_out=scatter_out, S=S)
    Y = moe.scatter_linear(X.cuda(), Wt.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
                           torch.from_numpy(offsets).cuda(),
                           None if g is None else g.cuda(), gather_in=gather_in,
                           scatter_out=scatter_out, S=S)
    torch.cuda.synchronize()
    got = Y.float().cpu().numpy()
    assert got.shape == ref.shape
    err = rel_frob(got, ref)
    assert err < _tol(dtype, scatter_out), err
    scale = np.abs(ref).max() + 1e-30
    assert np.abs(got - ref).max() / scale < 10 * _tol(dtype, scatter_out)


def test_scatter_linear_accumulates_into_out(oracle_lib, moe, gemm_kernel):
    S, k, E, Din, Dout = 200, 2, 4, 64, 64
    te = W.make_top_experts(S, k, E, seed=4)
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    X = torch.randn(S, Din).to(torch.bfloat16)
    Wt = (torch.randn(E, Din, Dout) * 0.05).to(torch.bfloat16)
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, None, S=S)
    base = torch.full((S, Dout), 3.0, device="cuda")
    Y = moe.scatter_linear(X.cuda(), Wt.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
                           torch.from_numpy(offsets).cuda(), out=base)
    torch.cuda.synchronize()
    assert rel_frob(Y.cpu().numpy() - 3.0, ref) < 2e-5


def test_scatter_linear_all_routes_one_expert(oracle_lib, moe, gemm_kernel):
    # every route on expert 2 of 4: three empty experts and one long run of M tiles
    S, k, E, Din, Dout = 1100, 1, 4, 128, 256
    te = torch.full((S, k), 2, dtype=torch.int32)
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    X = torch.randn(S, Din).to(torch.bfloat16)
    Wt = (torch.randn(E, Din, Dout) * 0.05).to(torch.bfloat16)
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, None, S=S)
    Y = moe.scatter_linear(X.cuda(), Wt.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
                           torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    assert rel_frob(Y.cpu().numpy(), ref) < 2e-5


EDGE_COUNTS = [1, 64, 65, 128, 129, 256, 257, 384, 385]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("gather_in,scatter_out", [(True, True), (False, True), (True, False),
                                                   (False, False)])
def test_scatter_linear_tile_edges(oracle_lib, moe, gemm_kernel, gather_in, scatter_out, dtype):
    # experts whose row counts sit on every tile edge: 64 (an M=64 one-CTA tile), 128 (a one-CTA
    # tile, an M=128 pair tile), 256 (a pair tile), 384 (a pair tile + an M=128 pair tile) and
    # one past each
    k, Din, Dout = 1, 96, 264
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    E = len(EDGE_COUNTS)
    owners = np.repeat(np.arange(E, dtype=np.int32), EDGE_COUNTS)
    perm = np.random.default_rng(7).permutation(len(owners))
    te = torch.from_numpy(owners[perm].reshape(-1, k).copy())
    S = te.shape[0]
    counts, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    assert list(counts) == EDGE_COUNTS
    gen = torch.Generator().manual_seed(11)
    X = torch.randn(S, Din, generator=gen).to(tdt)
    Wt = (torch.randn(E, Din, Dout, generator=gen) * 0.05).to(tdt)
    g = torch.rand(S * k, generator=gen)
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, g, gather_in=gather_in,
                                    scatter_out=scatter_out, S=S)
    Y = moe.scatter_linear(X.cuda(), Wt.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
                           torch.from_numpy(offsets).cuda(), g.cuda(), gather_in=gather_in,
                           scatter_out=scatter_out, S=S)
    torch.cuda.synchronize()
    got = Y.float().cpu().numpy()
    assert rel_frob(got, ref) < _tol(dtype, scatter_out)
    scale = np.abs(ref).max()
    assert np.abs(got - ref).max() / scale < 10 * _tol(dtype, scatter_out)
