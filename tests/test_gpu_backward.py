"""ParallelLinear backward on the GPU against the oracle ("3. Fused Backward Pass Dynamics" of the
ScatterMoE guide): the input gradient (the forward's grouped GEMM with W read transposed and the
gather / scatter roles exchanged), the weight gradient (a grouped GEMM reducing over each expert's
slots) and the gate gradient, for every input / output mode, bf16.

Tolerances: dY is rounded to bf16 once (relative 2^-9 per element, ~1e-3 relative on a sum of
many terms with random signs); operands are otherwise exact in bf16 and the tensor cores
accumulate in fp32; a bf16 dX adds one more rounding. So relative Frobenius 6e-3 and a max error
of 3e-2 of the largest reference entry, inside the 1e-2 / 2e-2 bars.
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import rel_frob

pytestmark = pytest.mark.gpu

REL, MAXREL = 6e-3, 3e-2

SHAPES = [
    # S, k, E, Din, Dout, mode
    (700, 2, 3, 200, 328, "uniform"),    # M, N and K tails in every GEMM
    (300, 4, 9, 64, 512, "zipf"),        # skew, experts without slots likely
    (129, 1, 1, 8, 8, "uniform"),        # smallest feature sizes, one expert
    (1000, 6, 64, 136, 264, "zipf"),
]


@pytest.fixture(params=["cta1", "cta2"])
def gemm_kernel(request, monkeypatch):
    monkeypatch.setenv("MOE_GEMM_2SM", "1" if request.param == "cta2" else "0")
    return request.param


def _check(name, got, ref):
    got = got.float().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert got.shape == ref.shape, name
    scale = np.abs(ref).max() + 1e-30
    assert rel_frob(got, ref) < REL, (name, rel_frob(got, ref))
    assert np.abs(got - ref).max() / scale < MAXREL, (name, np.abs(got - ref).max() / scale)


def _run(oracle_lib, moe, te, E, Din, Dout, seed, gather_in, scatter_out, gated):
    S, k = te.shape
    gen = torch.Generator().manual_seed(seed)
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    R = S * k
    X = torch.randn(S if gather_in else R, Din, generator=gen).to(torch.bfloat16)
    Wt = (torch.randn(E, Din, Dout, generator=gen) * 0.05).to(torch.bfloat16)
    g = torch.rand(R, generator=gen) if gated else None
    dY = torch.randn(S if scatter_out else R, Dout, generator=gen)
    if not scatter_out:
        dY = dY.to(torch.bfloat16)
    ref = oracle_lib.scatter_linear_backward(X, Wt, dY, k, sorted_rows, offsets, g,
                                             gather_in=gather_in, scatter_out=scatter_out, S=S)
    got = moe.scatter_linear_backward(
        X.cuda(), Wt.cuda(), dY.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
        torch.from_numpy(offsets).cuda(), None if g is None else g.cuda(), gather_in=gather_in,
        scatter_out=scatter_out, S=S)
    torch.cuda.synchronize()
    for name in ref:
        _check(name, got[name], ref[name])
    return counts


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("gather_in,scatter_out", [(True, True), (False, True), (True, False),
                                                   (False, False)])
@pytest.mark.parametrize("gated", [True, False])
def test_scatter_linear_backward(oracle_lib, moe, gemm_kernel, shape, gather_in, scatter_out,
                                 gated):
    S, k, E, Din, Dout, mode = shape
    te = W.make_top_experts(S, k, E, seed=S + 1, mode=mode)
    _run(oracle_lib, moe, te, E, Din, Dout, S + Din, gather_in, scatter_out, gated)


EDGE_COUNTS = [1, 63, 64, 65, 127, 128, 129, 256, 257, 0]


@pytest.mark.parametrize("gather_in,scatter_out", [(True, True), (False, False)])
def test_backward_expert_size_edges(oracle_lib, moe, gather_in, scatter_out):
    # the weight gradient's K loop runs over an expert's slots in stages of 64; the input
    # gradient's M tiles are 128 (64-row MMAs at the tail); one expert has no slot
    E = len(EDGE_COUNTS)
    owners = np.repeat(np.arange(E, dtype=np.int32), EDGE_COUNTS)
    te = torch.from_numpy(owners[np.random.default_rng(8).permutation(len(owners))].reshape(-1, 1).copy())
    counts = _run(oracle_lib, moe, te, E, 96, 136, 21, gather_in, scatter_out, True)
    assert list(counts) == EDGE_COUNTS


def test_backward_outputs_are_optional_and_checked(oracle_lib, moe):
    S, k, E, Din, Dout = 64, 2, 4, 32, 40
    te = W.make_top_experts(S, k, E, seed=3)
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    X = torch.randn(S, Din).to(torch.bfloat16).cuda()
    Wt = (torch.randn(E, Din, Dout) * 0.05).to(torch.bfloat16).cuda()
    dY = torch.randn(S, Dout).cuda()
    sr, off = torch.from_numpy(sorted_rows).cuda(), torch.from_numpy(offsets).cuda()
    only_dw = moe.scatter_linear_backward(X, Wt, dY, k, sr, off, need=("dW",))
    assert set(only_dw) == {"dW"}
    ref = oracle_lib.scatter_linear_backward(X.cpu(), Wt.cpu(), dY.cpu(), k, sorted_rows, offsets)
    _check("dW", only_dw["dW"], ref["dW"])
    # dgates needs the forward's gates; fp32 inputs are not supported by the backward
    with pytest.raises(moe.MoeError):
        dg = torch.empty(S * k, device="cuda")
        ws = moe.alloc_workspace(moe.workspace_size("scatter_linear_backward", S, Din, Dout, E, k,
                                                    torch.bfloat16), "cuda")
        moe._check(moe.lib.moe_scatter_linear_backward(
            moe._ptr(X), moe._ptr(Wt), moe._ptr(dY), S, Din, Dout, E, k, moe._ptr(sr),
            moe._ptr(off), None, 1, 1, moe.MOE_BF16, None, None, moe._ptr(dg), moe._ptr(ws),
            ws.numel(), moe._stream(X.device)))
    with pytest.raises(moe.MoeError):
        moe.scatter_linear_backward(X.float(), Wt.float(), dY, k, sr, off)


def test_backward_without_routes(moe):
    E, Din, Dout = 3, 16, 24
    X = torch.zeros((0, Din), dtype=torch.bfloat16, device="cuda")
    Wt = torch.randn(E, Din, Dout).to(torch.bfloat16).cuda()
    dY = torch.zeros((0, Dout), device="cuda")
    sr = torch.zeros(0, dtype=torch.int32, device="cuda")
    off = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    out = moe.scatter_linear_backward(X, Wt, dY, 2, sr, off, S=0)
    torch.cuda.synchronize()
    assert out["dX"].shape == (0, Din)
    assert torch.all(out["dW"] == 0)
