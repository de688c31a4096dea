"""Expert-MLP backward on the GPU against the oracle's backward run on the GPU's routing.

Tolerances: the GPU rounds dout, the recomputed pre-activations, dh, [da | db] and the router's dl
to bf16 once each (relative 2^-9 per element); accumulation is fp32. Relative Frobenius 1e-2
(the bar) and a max error of 5e-2 of the largest reference entry.
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import rel_frob

pytestmark = pytest.mark.gpu

REL, MAXREL = 1e-2, 5e-2

CASES = [
    # S, D, F, E, k, zipf bias
    (256, 256, 512, 8, 2, False),
    (300, 136, 192, 16, 4, True),
    (130, 64, 128, 8, 1, False),
    (200, 128, 128, 64, 6, True),
]


@pytest.fixture(params=["cta1", "cta2"])
def gemm_kernel(request, monkeypatch):
    monkeypatch.setenv("MOE_GEMM_2SM", "1" if request.param == "cta2" else "0")
    return request.param


def _inputs(S, D, F, E, k, zipf, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(S, D, generator=g).to(torch.bfloat16)
    wg = (torch.randn(D, E, generator=g) / D ** 0.5).to(torch.bfloat16)
    wge = (torch.randn(E, D, F, generator=g) / D ** 0.5).to(torch.bfloat16)
    wu = (torch.randn(E, D, F, generator=g) / D ** 0.5).to(torch.bfloat16)
    wd = (torch.randn(E, F, D, generator=g) / F ** 0.5).to(torch.bfloat16)
    bias = None
    if zipf:
        rank = torch.randperm(E, generator=g)
        bias = torch.empty(E)
        bias[rank] = -1.2 * torch.log(torch.arange(E, dtype=torch.float32) + 1.0)
    dout = torch.randn(S, D, generator=g)
    return x, wg, wge, wu, wd, bias, dout


@pytest.mark.parametrize("case", CASES)
def test_mlp_backward_matches_oracle(oracle_lib, moe, gemm_kernel, case):
    S, D, F, E, k, zipf = case
    x, wg, wge, wu, wd, bias, dout = _inputs(S, D, F, E, k, zipf, seed=S + E)
    dev = torch.device("cuda")
    cu = [t.to(dev) for t in (x, wg, wge, wu, wd)]
    ws = moe.ForwardWorkspace(S, D, F, E, k, torch.bfloat16, dev)
    moe.mlp_forward(*cu, k, logit_bias=None if bias is None else bias.to(dev), ws=ws)
    grads = moe.mlp_backward(*cu, k, dout.to(dev), ws)
    torch.cuda.synchronize()
    moe.check_device_status(ws.buf)
    te = ws.view("top_experts").cpu().numpy()
    ref = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k, bias=bias, given_top_experts=te)
    for name, r in ref.items():
        got = grads[name].cpu().numpy()
        assert got.shape == r.shape, name
        assert rel_frob(got, r) < REL, (name, rel_frob(got, r))
        assert np.abs(got - r).max() / (np.abs(r).max() + 1e-30) < MAXREL, name


def test_mlp_backward_argument_errors(moe):
    dev = torch.device("cuda")
    S, D, F, E, k = 16, 64, 128, 6, 2     # E not a multiple of 8
    x, wg, wge, wu, wd, bias, dout = _inputs(S, D, F, E, k, False, seed=1)
    cu = [t.to(dev) for t in (x, wg, wge, wu, wd)]
    ws = moe.ForwardWorkspace(S, D, F, E, k, torch.bfloat16, dev)
    moe.mlp_forward(*cu, k, ws=ws)
    with pytest.raises(moe.MoeError):
        moe.mlp_backward(*cu, k, dout.to(dev), ws)


def test_mlp_backward_full_size_sampled_dx(oracle_lib, moe):
    """The Mixtral-shaped prefill layer in the configuration the bench's backward times: the input
    gradient of seeded sample tokens against the oracle's backward run on those tokens alone (a
    token's dx depends on that token only). This covers the dh GEMM, the fused SwiGLU backward,
    the dx GEMM and the router backward at full size; the weight gradients are sums over all
    tokens and are checked at the smaller sizes above."""
    w = W.WORKLOADS["mixtral_prefill"]
    dev = torch.device("cuda")
    inp = W.make_inputs(w, device=dev, seed=0)
    ws = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, torch.bfloat16, dev)
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k,
                    logit_bias=inp["logit_bias"], ws=ws)
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    dout = torch.randn((w.S, w.D), generator=g, device=dev)
    grads = moe.mlp_backward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                             inp["w_down"], w.k, dout, ws)
    torch.cuda.synchronize()
    moe.check_device_status(ws.buf)
    te = ws.view("top_experts").cpu().numpy()
    toks = np.sort(np.random.default_rng(3).choice(w.S, size=12, replace=False))
    cpu = {n: inp[n].float().cpu().numpy() for n in ("x", "w_gate", "w_gate_e", "w_up", "w_down")}
    ref = oracle_lib.mlp_backward(cpu["x"][toks], cpu["w_gate"], cpu["w_gate_e"], cpu["w_up"],
                                  cpu["w_down"], dout.cpu().numpy()[toks], w.k,
                                  given_top_experts=te[toks], want=("dx",))["dx"]
    got = grads["dx"].cpu().numpy()[toks]
    assert rel_frob(got, ref) < REL, rel_frob(got, ref)
    assert np.abs(got - ref).max() / (np.abs(ref).max() + 1e-30) < MAXREL
