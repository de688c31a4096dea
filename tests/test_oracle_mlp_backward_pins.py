"""Pins of the oracle's expert-MLP backward (the ScatterMoE guide's backward of each ParallelLinear,
"3. Fused Backward Pass Dynamics", chained through SwiGLU and the router softmax).

Independent of the oracle's loops:
  * torch float64 autograd of the dense all-experts-then-mask formulation: every expert runs on
    every token, and the top-k mask (fixed, from the oracle's routing) times the softmax of the
    selected logits weights the sum; autograd differentiates it;
  * central finite differences of L = <dout, forward> for a few entries of every input, on
    inputs whose routing has a clear margin (so the selection does not change under the step).
"""
import numpy as np
import pytest
import torch

import moe_workloads as W


def _inputs(S, D, F, E, k, seed, bias_scale=0.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(S, D, generator=g)
    wg = torch.randn(D, E, generator=g) * (1.0 / D ** 0.5)
    wge = torch.randn(E, D, F, generator=g) * 0.3
    wu = torch.randn(E, D, F, generator=g) * 0.3
    wd = torch.randn(E, F, D, generator=g) * 0.3
    dout = torch.randn(S, D, generator=g)
    bias = (torch.randn(E, generator=g) * bias_scale) if bias_scale else None
    return x, wg, wge, wu, wd, dout, bias


def _dense_autograd(x, wg, wge, wu, wd, dout, J, bias=None):
    t = {n: v.double().clone().requires_grad_(True) for n, v in
         (("x", x), ("wg", wg), ("wge", wge), ("wu", wu), ("wd", wd))}
    l = t["x"] @ t["wg"]
    if bias is not None:
        l = l + bias.double()
    Jt = torch.from_numpy(J.astype(np.int64))
    w = torch.softmax(l.gather(1, Jt), dim=1)
    y = torch.zeros(x.shape[0], wd.shape[2], dtype=torch.float64)
    for e in range(wge.shape[0]):
        a = t["x"] @ t["wge"][e]
        b = t["x"] @ t["wu"][e]
        v = (torch.nn.functional.silu(a) * b) @ t["wd"][e]
        c = (w * (Jt == e).double()).sum(dim=1, keepdim=True)
        y = y + c * v
    (dout.double() * y).sum().backward()
    return {"dx": t["x"].grad, "dw_gate": t["wg"].grad, "dw_gate_e": t["wge"].grad,
            "dw_up": t["wu"].grad, "dw_down": t["wd"].grad}


@pytest.mark.parametrize("S,D,F,E,k,bias", [(9, 6, 5, 4, 2, 0.0), (13, 8, 7, 6, 3, 1.5),
                                            (7, 5, 4, 3, 1, 0.0), (6, 4, 3, 3, 3, 0.0)])
def test_mlp_backward_matches_dense_autograd(oracle_lib, S, D, F, E, k, bias):
    x, wg, wge, wu, wd, dout, b = _inputs(S, D, F, E, k, seed=S + E, bias_scale=bias)
    _, te, _ = oracle_lib.mlp_forward(x, wg, wge, wu, wd, k, bias=b)
    got = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k, bias=b)
    ref = _dense_autograd(x, wg, wge, wu, wd, dout, te, bias=b)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name].numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)


def test_mlp_backward_given_routing_is_used(oracle_lib):
    S, D, F, E, k = 8, 6, 5, 5, 2
    x, wg, wge, wu, wd, dout, _ = _inputs(S, D, F, E, k, seed=3)
    forced = np.tile(np.array([[4, 1]], dtype=np.int32), (S, 1))
    got = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k, given_top_experts=forced)
    ref = _dense_autograd(x, wg, wge, wu, wd, dout, forced)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name].numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)
    # experts outside the forced pair get no gradient
    assert np.all(got["dw_down"][[0, 2, 3]] == 0.0)


def test_mlp_backward_finite_differences(oracle_lib):
    S, D, F, E, k = 5, 4, 3, 4, 2
    x, wg, wge, wu, wd, dout, _ = _inputs(S, D, F, E, k, seed=11)
    logits, _ = oracle_lib.router_logits(x.numpy(), wg.numpy())
    srt = np.sort(logits, axis=1)[:, ::-1]
    assert np.all(srt[:, k - 1] - srt[:, k] > 1e-3), "routing margin too small for the step"
    got = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k)
    arrays = {"dx": x, "dw_gate": wg, "dw_gate_e": wge, "dw_up": wu, "dw_down": wd}

    def loss(vals):
        y, _, _ = oracle_lib.mlp_forward(vals["dx"], vals["dw_gate"], vals["dw_gate_e"],
                                         vals["dw_up"], vals["dw_down"], k)
        return float(np.sum(dout.numpy().astype(np.float64) * y))

    rng = np.random.default_rng(0)
    for name, arr in arrays.items():
        base = {n: a.numpy().copy() for n, a in arrays.items()}
        for _ in range(3):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            up = {n: a.copy() for n, a in base.items()}
            dn = {n: a.copy() for n, a in base.items()}
            up[name][idx] = np.float32(base[name][idx] + np.float32(2.0 ** -9))
            dn[name][idx] = np.float32(base[name][idx] - np.float32(2.0 ** -9))
            step = float(up[name][idx]) - float(dn[name][idx])
            fd = (loss(up) - loss(dn)) / step
            assert fd == pytest.approx(got[name][idx], rel=2e-4, abs=2e-6), (name, idx)


def test_dx_only_and_per_token(oracle_lib):
    """Asking for dx alone (tokens in parallel) gives the same dx as the full backward, and the dx
    rows of a token subset equal those of the whole batch (a token's dx depends on it alone)."""
    g = np.random.default_rng(5)
    S, D, F, E, k = 40, 24, 32, 6, 2
    x = g.standard_normal((S, D)).astype(np.float32)
    wg = (g.standard_normal((D, E)) / D ** 0.5).astype(np.float32)
    wge = (g.standard_normal((E, D, F)) / D ** 0.5).astype(np.float32)
    wu = (g.standard_normal((E, D, F)) / D ** 0.5).astype(np.float32)
    wd = (g.standard_normal((E, F, D)) / F ** 0.5).astype(np.float32)
    dout = g.standard_normal((S, D)).astype(np.float32)
    full = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k)
    only = oracle_lib.mlp_backward(x, wg, wge, wu, wd, dout, k, want=("dx",))
    assert set(only) == {"dx"}
    np.testing.assert_allclose(only["dx"], full["dx"], rtol=1e-12, atol=1e-14)
    _, te, _ = oracle_lib.mlp_forward(x, wg, wge, wu, wd, k)
    toks = np.array([3, 17, 29, 38])
    sub = oracle_lib.mlp_backward(x[toks], wg, wge, wu, wd, dout[toks], k,
                                  given_top_experts=te[toks], want=("dx",))
    np.testing.assert_allclose(sub["dx"], full["dx"][toks], rtol=1e-12, atol=1e-14)
