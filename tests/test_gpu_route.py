"""Router on the GPU against the oracle: top-k experts equal except at justified near-ties (the
fp32 rounding bound on the oracle's fp64 logits), weights within fp32 rounding of the oracle's
softmax over the GPU's own choice.

Source: "ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs", "1. The Dynamic Routing
Imbalance Dilemma" (H(X) = Softmax(TopK(X W_gate, k))).
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import check_routing

pytestmark = pytest.mark.gpu


def _route_and_check(oracle_lib, moe, inp, k, tokens=None, max_diff_frac=0.01):
    x, wg, bias = inp["x"], inp["w_gate"], inp["logit_bias"]
    S, D = x.shape
    te, tw = moe.route_topk(x.cuda(), wg.cuda(), k, None if bias is None else bias.cuda())
    torch.cuda.synchronize()
    te, tw = te.cpu().numpy(), tw.cpu().numpy()
    if tokens is None:
        tokens = np.arange(S, dtype=np.int32)
    logits, absdot = oracle_lib.router_logits(x, wg, bias, tokens=tokens)
    ote, otw = oracle_lib.topk_softmax(logits, k)
    diff = check_routing(te[tokens], ote, logits, absdot, D)
    assert diff <= max(1, int(max_diff_frac * len(tokens)))
    # weights: the oracle's softmax over the GPU's experts, in the GPU's order
    ow = oracle_lib.weights_for(logits, te[tokens])
    assert np.max(np.abs(tw[tokens] - ow)) < 1e-5
    assert np.allclose(tw.sum(axis=1), 1.0, atol=2e-6)
    assert np.all(np.diff(tw, axis=1) <= 1e-7)
    return te, tw


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("E,k", [(1, 1), (5, 2), (8, 2), (32, 8), (33, 3), (64, 6), (96, 4),
                                 (128, 4), (200, 8), (256, 8)])
def test_route_small(oracle_lib, moe, dtype, E, k):
    w = W.custom("r", S=300, D=136, F=8, E=E, k=k, dtype=dtype, router_std="1/sqrt(D)")
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=E * 31 + k), k)


@pytest.mark.parametrize("S", [1, 7, 128, 2048, 2049, 5000])
def test_route_eight_experts_every_batch_size(oracle_lib, moe, S):
    # bf16 with eight experts: the warp-MMA router at every batch size, 16 tokens per block (one
    # partly filled block at S = 1 and 7, ragged last blocks at 2049 and 5000)
    w = W.custom("r8", S=S, D=4096, F=8, E=8, k=2, dtype="bf16")
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=S), 2)


@pytest.mark.parametrize("D", [8, 200, 2880, 6144, 9792])
def test_route_eight_experts_feature_sizes(oracle_lib, moe, D):
    # the warp-MMA router's d split: D not a multiple of 32 (zero rows past D in the last group),
    # fewer groups of 32 d than warps (D = 8, 200), one block per SM at the largest sizes
    w = W.custom("r8d", S=2100, D=D, F=8, E=8, k=3, dtype="bf16", router_std="1/sqrt(D)")
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=D), 3)


@pytest.mark.parametrize("E,k,D", [(16, 2, 200), (24, 3, 2880), (64, 6, 2048), (72, 8, 136),
                                   (120, 4, 520), (128, 4, 2880)])
def test_route_many_experts_tensor_cores(oracle_lib, moe, E, k, D):
    # bf16, 16-128 experts and S > 2048: the tensor-core router, 17 tiles of 128 tokens (a ragged
    # last one at S = 2100), D in 64-wide stages with a ragged last one, E not a power of two
    w = W.custom("rm", S=2100, D=D, F=8, E=E, k=k, dtype="bf16", router_std="1/sqrt(D)")
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=E * 7 + D), k)


@pytest.mark.parametrize("S,E,k", [(40000, 128, 4), (20000, 256, 8), (19000, 64, 6)])
def test_route_tensor_core_several_tiles_per_cta(oracle_lib, moe, S, E, k):
    # more 128-token tiles than SMs: each CTA of the tensor-core router runs two or three tiles
    # through its two TMEM accumulators
    w = W.custom("rt", S=S, D=64, F=8, E=E, k=k, dtype="bf16", router_std="1/sqrt(D)")
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=S + E), k)


def test_route_bias_zipf(oracle_lib, moe):
    w = W.custom("z", S=2000, D=256, F=8, E=64, k=6, router_std="1/sqrt(D)", zipf_s=1.2)
    te, _ = _route_and_check(oracle_lib, moe, W.make_inputs(w), 6)
    counts = np.bincount(te.reshape(-1), minlength=64)
    assert counts.max() > 4 * counts.mean()   # the bias produces the skew


def test_route_exact_ties_pick_lower_id(moe):
    # x = 0: every logit is 0 (a tie everywhere), so the experts are 0..k-1 with weight 1/k
    x = torch.zeros(70, 64, dtype=torch.bfloat16, device="cuda")
    wg = torch.randn(64, 12, device="cuda").to(torch.bfloat16)
    te, tw = moe.route_topk(x, wg, 3)
    assert torch.equal(te.cpu(), torch.tensor([[0, 1, 2]] * 70, dtype=torch.int32))
    assert torch.allclose(tw.cpu(), torch.full((70, 3), 1 / 3))


@pytest.mark.parametrize("name", ["mixtral_prefill", "e128", "zipf64"])
def test_route_full_workloads(oracle_lib, moe, name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, device="cuda")
    cpu = {k: (v.cpu() if v is not None else None) for k, v in inp.items()
           if k in ("x", "w_gate", "logit_bias")}
    toks = np.random.default_rng(0).choice(w.S, size=2048, replace=False).astype(np.int32)
    _route_and_check(oracle_lib, moe, cpu, w.k, tokens=np.sort(toks))


@pytest.mark.parametrize("k", [1, 2, 8])
def test_route_eight_experts_large_batch(oracle_lib, moe, k):
    """The eight-expert router used above 2048 tokens (W_gate staged in shared memory); D = 264
    gives 33 pieces per row, a ragged last round across the lanes; k = 2 adds a skewing bias."""
    w = W.custom("e8", S=2500, D=264, F=8, E=8, k=k, router_std="1/sqrt(D)",
                 zipf_s=1.2 if k == 2 else 0.0)
    _route_and_check(oracle_lib, moe, W.make_inputs(w, seed=k), k)


def test_route_eight_experts_exact_ties(moe):
    x = torch.zeros(3000, 64, dtype=torch.bfloat16, device="cuda")
    wg = torch.randn(64, 8, device="cuda").to(torch.bfloat16)
    te, tw = moe.route_topk(x, wg, 3)
    assert torch.equal(te.cpu(), torch.tensor([[0, 1, 2]] * 3000, dtype=torch.int32))
    assert torch.allclose(tw.cpu(), torch.full((3000, 3), 1 / 3))


def test_route_tensor_core_exact_ties(moe):
    """The tensor-core router (bf16, E > 64): all logits equal, so experts 0..k-1 in order with
    weight 1/k. x = -0.0 makes some logits -0 and others +0; they compare equal as numbers and
    must tie like the +0 logits of x = +0.0."""
    for zero in (0.0, -0.0):
        x = torch.full((300, 136), zero, dtype=torch.bfloat16, device="cuda")
        wg = torch.randn(136, 128, generator=torch.Generator().manual_seed(5)).to(
            torch.bfloat16).cuda()
        te, tw = moe.route_topk(x, wg, 4)
        assert torch.equal(te.cpu(), torch.tensor([[0, 1, 2, 3]] * 300, dtype=torch.int32))
        assert torch.allclose(tw.cpu(), torch.full((300, 4), 0.25))


def test_route_tensor_core_infinite_logits(moe):
    """x[5, 0] = +inf gives row 5 logits of +inf (W_gate[0, e] > 0), -inf (< 0) or NaN (= 0,
    counted as -inf): its experts are the k smallest ids with W_gate[0, e] > 0, tied at +inf. The
    other rows are unaffected."""
    E, k = 128, 5
    g = torch.Generator().manual_seed(11)
    x = torch.randn(300, 136, generator=g).to(torch.bfloat16)
    wg = torch.randn(136, E, generator=g).to(torch.bfloat16)
    wg[0, 3] = 0.0
    x[5, 0] = float("inf")
    te, tw = moe.route_topk(x.cuda(), wg.cuda(), k)
    te = te.cpu()
    pos = [e for e in range(E) if float(wg[0, e]) > 0][:k]
    assert te[5].tolist() == pos
    ref_te, _ = moe.route_topk(x[6:].cuda(), wg.cuda(), k)  # rows without inf, routed alone
    assert torch.equal(te[6:], ref_te.cpu())
    assert bool(torch.isfinite(tw[6:]).all())
