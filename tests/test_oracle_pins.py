"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each check reaches the oracle's result by an independent route: brute force on tiny inputs, a dense
all-experts-then-mask formulation with numpy float64 matmuls, closed forms, special cases that reduce
to a dense SwiGLU MLP, hand-worked fixtures under tests/golden/, and the sparse-map invariants listed
in "4. Correctness Validation" of "Add scalable sparse map kernel for large MoE models (128+
experts)". Every pin is chosen so that a plausible slip in the oracle (a swapped gate/up half, a
transposed weight, a dropped renormalisation, a wrong tie-break, an off-by-one slot) fails it.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import moe_workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(v) if "." in v else int(v) for v in rest]
    return vals


def _np(t):
    return t.detach().float().numpy().astype(np.float64)


def _silu_np(z):
    # numpy's logistic via tanh: sigma(z) = (1 + tanh(z/2)) / 2, an identity independent of the
    # oracle's exp form.
    return z * 0.5 * (1.0 + np.tanh(0.5 * z))


# ----------------------------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------------------------

def _bruteforce_topk(l, k):
    """The unique k-subset whose every member beats every non-member under (logit desc, id asc),
    found by enumerating all subsets; members listed in that order."""
    E = len(l)
    better = lambda a, b: (l[a] > l[b]) or (l[a] == l[b] and a < b)
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(better(a, b) for a in sub for b in rest):
            return sorted(sub, key=lambda e: (-l[e], e))
    raise AssertionError("no dominating subset")


def test_route_golden_ties(oracle_lib):
    fx = _read_fixture("route_hand_ties.txt")
    l = np.array([fx["logits"]], dtype=np.float64)
    for k in range(1, 5):
        te, tw = oracle_lib.topk_softmax(l, k)
        assert te[0].tolist() == fx[f"k{k}"]
    # weights in closed form for k = 2, 3
    _, tw = oracle_lib.topk_softmax(l, 2)
    assert np.allclose(tw[0], [0.5, 0.5], rtol=0, atol=1e-15)
    _, tw = oracle_lib.topk_softmax(l, 3)
    den = 2.0 + math.exp(-2.0)
    assert np.allclose(tw[0], [1 / den, 1 / den, math.exp(-2.0) / den], rtol=1e-14, atol=0)


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (4, 3), (5, 2), (6, 4), (8, 8)])
def test_route_bruteforce_with_ties(oracle_lib, E, k):
    gen = torch.Generator().manual_seed(E * 10 + k)
    S, D = 16, 3
    # small integers: every logit is an exact small integer, so ties are frequent and exact
    x = torch.randint(-2, 3, (S, D), generator=gen).float()
    wg = torch.randint(-2, 3, (D, E), generator=gen).float()
    logits, absdot = oracle_lib.router_logits(x, wg)
    assert np.array_equal(logits, _np(x) @ _np(wg))
    te, tw = oracle_lib.topk_softmax(logits, k)
    for s in range(S):
        assert te[s].tolist() == _bruteforce_topk(logits[s].tolist(), k)
        # weights: logistic form of the softmax over the selected logits
        sel = logits[s, te[s]]
        for j in range(k):
            ref = 1.0 / np.sum(np.exp(sel - sel[j]))
            assert abs(tw[s, j] - ref) < 1e-14
        assert abs(tw[s].sum() - 1.0) < 1e-14
        assert np.all(np.diff(tw[s]) <= 0)


def test_router_absdot_magnitude_sum(oracle_lib):
    """The magnitude sum a[s,e] = sum_d |x[s,d] W_gate[d,e]| that sets the GPU routing tie band
    equals |x| @ |W_gate| in float64 (every term is non-negative, so any summation order agrees to
    a few ulps), with and without a bias (the bias is not part of the dot product) and on a token
    subset. Dropping the absolute value, summing |x_d| alone or adding the bias fails this."""
    gen = torch.Generator().manual_seed(7)
    S, D, E = 40, 96, 12
    x = (torch.randn((S, D), generator=gen)).to(torch.bfloat16).float()
    wg = (0.05 * torch.randn((D, E), generator=gen)).to(torch.bfloat16).float()
    bias = torch.randn(E, generator=gen)
    ref = np.abs(_np(x)) @ np.abs(_np(wg))
    for b in (None, bias):
        _, a = oracle_lib.router_logits(x, wg, bias=b)
        assert np.allclose(a, ref, rtol=1e-13, atol=0)
    toks = np.array([39, 0, 17, 17, 5], dtype=np.int32)
    _, a = oracle_lib.router_logits(x, wg, bias=bias, tokens=toks)
    assert np.allclose(a, ref[toks], rtol=1e-13, atol=0)
    # integer inputs with mixed signs: exact, and different from |sum| and from sum |x_d|
    xi = torch.randint(-3, 4, (9, 5), generator=gen).float()
    wi = torch.randint(-3, 4, (5, 4), generator=gen).float()
    l, a = oracle_lib.router_logits(xi, wi)
    assert np.array_equal(a, np.abs(_np(xi)) @ np.abs(_np(wi)))
    assert np.all(a >= np.abs(l))
    assert np.any(a > np.abs(l))


def test_router_absdot_closed_form(oracle_lib):
    # x_d = (-1)^d and W[d, e] = (e + 1) (-1)^(d + e): every product is (e + 1) (-1)^e in
    # magnitude e + 1, so a[s, e] = D (e + 1) while the logit is D (e + 1) (-1)^e.
    D, E = 10, 5
    x = np.array([[(-1.0) ** d for d in range(D)]], np.float32)
    wg = np.array([[(e + 1) * (-1.0) ** (d + e) for e in range(E)] for d in range(D)], np.float32)
    l, a = oracle_lib.router_logits(x, wg)
    assert a[0].tolist() == [D * (e + 1.0) for e in range(E)]
    assert l[0].tolist() == [D * (e + 1.0) * (-1.0) ** e for e in range(E)]


def test_router_tie_band_bounds_fp32_logits(oracle_lib):
    """The tie band built from the magnitude sum (Higham's bound gamma_D * a for a float32 dot
    product of exact inputs) contains the float32 logits that torch computes on the CPU, in two
    summation orders, at the Mixtral width D = 4096 and the 128-expert width D = 2880."""
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from parity import fp32_dot_bound
    for D, E, seed in ((4096, 8, 1), (2880, 16, 2)):
        gen = torch.Generator().manual_seed(seed)
        x = (torch.randn((64, D), generator=gen)).to(torch.bfloat16).float()
        wg = (torch.randn((D, E), generator=gen) / math.sqrt(D)).to(torch.bfloat16).float()
        l, a = oracle_lib.router_logits(x, wg)
        band = fp32_dot_bound(D, a)
        l32 = (x @ wg).double().numpy()
        l32_seq = torch.zeros((64, E))
        for d0 in range(0, D, 512):  # a blocked order: partial sums of 512 added in sequence
            l32_seq += x[:, d0:d0 + 512] @ wg[d0:d0 + 512]
        for got in (l32, l32_seq.double().numpy()):
            assert np.all(np.abs(got - l) <= band)
        # the band is not vacuous: a few percent of the logits' spread (a worst-case bound, so
        # wider than the errors themselves)
        assert np.median(band) < 0.05 * np.std(l)


def test_route_bias_forces_expert(oracle_lib):
    w = W.custom("b", S=64, D=32, F=16, E=6, k=2, dtype="f32")
    inp = W.make_inputs(w)
    bias = torch.zeros(6)
    bias[4] = 1.0e3
    te, tw = oracle_lib.route(inp["x"], inp["w_gate"], 2, bias=bias)
    assert np.all(te[:, 0] == 4)
    assert np.all(tw[:, 0] > 0.999999)
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, 6)
    assert counts[4] == 64
    # expert 4 is every token's first route: its slots hold routes 0, k, 2k, ...
    assert sorted_rows[offsets[4]:offsets[5]].tolist() == list(range(0, 128, 2))


def test_route_all_tied(oracle_lib):
    # x = 0: all logits are 0, so the experts are 0..k-1 in order with weight 1/k each
    logits, _ = oracle_lib.router_logits(np.zeros((5, 8), np.float32),
                                         np.ones((8, 6), np.float32))
    te, tw = oracle_lib.topk_softmax(logits, 3)
    assert np.all(te == np.array([0, 1, 2]))
    assert np.allclose(tw, 1.0 / 3.0, rtol=0, atol=1e-16)


# ----------------------------------------------------------------------------------------------
# sparse map
# ----------------------------------------------------------------------------------------------

def _map_bruteforce(te, E):
    """O(R*E) direct scan: for each expert in order, walk the flat routes in order."""
    te = np.asarray(te).reshape(-1)
    sorted_rows = []
    counts = []
    for e in range(E):
        rows = [i for i in range(te.shape[0]) if te[i] == e]
        counts.append(len(rows))
        sorted_rows += rows
    sparse_rows = [0] * len(sorted_rows)
    for p, i in enumerate(sorted_rows):
        sparse_rows[i] = p
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    return counts, offsets, sparse_rows, sorted_rows


def check_map_invariants(te, E, counts, offsets, sparse_rows, sorted_rows):
    """The invariants of "4. Correctness Validation" plus stability and exact histogram."""
    te = np.asarray(te).reshape(-1)
    R = te.shape[0]
    counts, offsets = np.asarray(counts), np.asarray(offsets)
    sparse_rows, sorted_rows = np.asarray(sparse_rows), np.asarray(sorted_rows)
    assert counts.sum() == R
    assert np.array_equal(counts, np.bincount(te, minlength=E)[:E])
    assert offsets[0] == 0 and offsets[E] == R
    assert np.all(np.diff(offsets) == counts)              # ranges contiguous, non-overlapping
    assert np.array_equal(np.sort(sparse_rows), np.arange(R))  # unique slots
    assert np.array_equal(sorted_rows[sparse_rows], np.arange(R))  # mutual inverses
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        seg = sorted_rows[lo:hi]
        assert np.all(te[seg] == e)                       # each slot inside its expert's range
        assert np.all(np.diff(seg) > 0)                   # stable: increasing route index


def test_map_golden(oracle_lib):
    fx = _read_fixture("map_hand_s4_k2_e3.txt")
    te = np.array(fx["top_experts"], dtype=np.int32)
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, fx["E"][0])
    assert counts.tolist() == fx["counts"]
    assert offsets.tolist() == fx["offsets"]
    assert sorted_rows.tolist() == fx["sorted_rows"]
    assert sparse_rows.tolist() == fx["sparse_rows"]


@pytest.mark.parametrize("E", [4, 8, 16, 32, 64, 96, 128, 256])
@pytest.mark.parametrize("mode", ["uniform", "zipf", "any"])
def test_map_bruteforce_and_invariants(oracle_lib, E, mode):
    k = min(4, E)
    S = 97
    te = W.make_top_experts(S, k, E, seed=E, mode=mode).numpy()
    res = oracle_lib.sparse_map(te, E)
    bf = _map_bruteforce(te, E)
    for a, b in zip(res, bf):
        assert np.array_equal(np.asarray(a), np.asarray(b))
    check_map_invariants(te, E, *res)
    # deterministic across runs
    for _ in range(2):
        again = oracle_lib.sparse_map(te, E)
        for a, b in zip(res, again):
            assert np.array_equal(a, b)


def test_map_k_equals_E_closed_form(oracle_lib):
    S, E = 9, 5
    gen = torch.Generator().manual_seed(3)
    te = torch.stack([torch.randperm(E, generator=gen) for _ in range(S)]).int().numpy()
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, E)
    assert counts.tolist() == [S] * E
    assert offsets.tolist() == [e * S for e in range(E + 1)]
    for e in range(E):
        for s in range(S):
            j = int(np.where(te[s] == e)[0][0])
            assert sorted_rows[e * S + s] == s * E + j


def test_map_empty_experts_and_one_expert(oracle_lib):
    te = W.make_top_experts(50, 3, 7, mode="one").numpy()
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, 7)
    assert counts.tolist() == [150, 0, 0, 0, 0, 0, 0]
    assert offsets.tolist() == [0] + [150] * 7
    assert sorted_rows.tolist() == list(range(150))
    # empty input
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(np.zeros(0, np.int32), 4)
    assert counts.tolist() == [0] * 4 and offsets.tolist() == [0] * 5


def test_map_rejects_bad_id(oracle_lib):
    with pytest.raises(ValueError):
        oracle_lib.sparse_map(np.array([0, 4, 1], np.int32), 4)
    with pytest.raises(ValueError):
        oracle_lib.sparse_map(np.array([0, -1, 1], np.int32), 4)


# ----------------------------------------------------------------------------------------------
# expert FFN and the full forward
# ----------------------------------------------------------------------------------------------

def test_swiglu_closed_form(oracle_lib):
    # D = F = E = k = 1: y = silu(x a) * (x b) * c. With x = 1 and a = ln 3, sigma(a) = 3/4, so
    # y = 0.75 ln 3 * b * c. A swapped gate/up half or a sign slip in the logistic breaks it.
    ln3 = math.log(3.0)
    x = np.array([[1.0]], np.float32)
    wg = np.zeros((1, 1), np.float32)
    a = np.float32(ln3)
    y, te, tw = oracle_lib.mlp_forward(x, wg, np.array([[[a]]], np.float32),
                                       np.array([[[2.0]]], np.float32),
                                       np.array([[[0.5]]], np.float32), 1)
    assert te.tolist() == [[0]] and tw.tolist() == [[1.0]]
    assert abs(y[0, 0] - 0.75 * ln3) < 1e-7
    # the negative side: silu(-ln 3) = -ln 3 / 4
    y, _, _ = oracle_lib.mlp_forward(x, wg, np.array([[[-a]]], np.float32),
                                     np.array([[[2.0]]], np.float32),
                                     np.array([[[0.5]]], np.float32), 1)
    assert abs(y[0, 0] - (-0.25 * ln3)) < 1e-7


def _dense_masked_forward(inp, k):
    """All experts on all tokens, then masked by the top-k routing and weighted: numpy float64
    matmuls, a formulation independent of the oracle's per-token loops."""
    x = _np(inp["x"])
    wg = _np(inp["w_gate"])
    E = wg.shape[1]
    logits = x @ wg
    if inp.get("logit_bias") is not None:
        logits = logits + _np(inp["logit_bias"])[None, :]
    S = x.shape[0]
    order = np.lexsort((np.broadcast_to(np.arange(E), logits.shape), -logits), axis=1)
    J = order[:, :k]
    sel = np.take_along_axis(logits, J, axis=1)
    wts = np.exp(sel - sel.max(axis=1, keepdims=True))
    wts = wts / wts.sum(axis=1, keepdims=True)
    M = np.zeros((S, E))
    np.put_along_axis(M, J, wts, axis=1)
    y = np.zeros((S, x.shape[1]))
    for e in range(E):
        g = x @ _np(inp["w_gate_e"][e])
        u = x @ _np(inp["w_up"][e])
        y += M[:, e:e + 1] * ((_silu_np(g) * u) @ _np(inp["w_down"][e]))
    return y, J, wts


@pytest.mark.parametrize("wl", [W.WORKLOADS["tiny"], W.custom("z", S=96, D=48, F=40, E=6, k=3,
                                                              dtype="bf16", router_std="1/sqrt(D)",
                                                              zipf_s=1.2)])
def test_forward_matches_dense_mask(oracle_lib, wl):
    inp = W.make_inputs(wl)
    y_ref, J, wts = _dense_masked_forward(inp, wl.k)
    y, te, tw = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                       inp["w_down"], wl.k, bias=inp["logit_bias"])
    assert np.array_equal(te, J)
    assert np.allclose(tw, wts, rtol=1e-12, atol=1e-15)
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel < 1e-12, rel


def test_forward_single_expert_is_dense_swiglu(oracle_lib):
    wl = W.custom("e1", S=40, D=24, F=36, E=1, k=1, dtype="f32")
    inp = W.make_inputs(wl)
    x = _np(inp["x"])
    y_ref = (_silu_np(x @ _np(inp["w_gate_e"][0])) * (x @ _np(inp["w_up"][0]))) @ \
        _np(inp["w_down"][0])
    y, te, tw = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                       inp["w_down"], 1)
    assert np.all(te == 0) and np.all(tw == 1.0)
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-14)


def test_forward_identical_experts(oracle_lib):
    # all experts equal: the weights sum to one, so y = FFN(x) whatever the routing
    wl = W.custom("same", S=30, D=16, F=20, E=5, k=3, dtype="f32")
    inp = W.make_inputs(wl)
    for name in ("w_gate_e", "w_up", "w_down"):
        inp[name] = inp[name][0:1].expand_as(inp[name]).contiguous()
    x = _np(inp["x"])
    y_ref = (_silu_np(x @ _np(inp["w_gate_e"][0])) * (x @ _np(inp["w_up"][0]))) @ \
        _np(inp["w_down"][0])
    y, _, _ = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                     inp["w_down"], 3)
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-14)


def test_forward_zero_input(oracle_lib):
    wl = W.custom("z0", S=7, D=16, F=8, E=4, k=2, dtype="f32")
    inp = W.make_inputs(wl)
    inp["x"] = torch.zeros_like(inp["x"])
    y, te, tw = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                       inp["w_down"], 2)
    assert np.all(y == 0.0)
    assert np.all(te == np.array([0, 1])) and np.allclose(tw, 0.5)


def test_forward_k_equals_E_full_softmax(oracle_lib):
    wl = W.custom("kE", S=12, D=16, F=8, E=4, k=4, dtype="f32")
    inp = W.make_inputs(wl)
    y, te, tw = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                       inp["w_down"], 4)
    full = torch.softmax(torch.from_numpy(_np(inp["x"]) @ _np(inp["w_gate"])), dim=1).numpy()
    for s in range(12):
        assert np.allclose(tw[s], full[s, te[s]], rtol=1e-12, atol=1e-15)


def test_forward_given_routing(oracle_lib):
    wl = W.custom("g", S=20, D=16, F=8, E=5, k=2, dtype="f32")
    inp = W.make_inputs(wl)
    given = W.make_top_experts(20, 2, 5, seed=1).numpy()
    y, te, tw = oracle_lib.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                       inp["w_down"], 2, given_top_experts=given)
    assert np.array_equal(te, given)
    # forced routing = a mask in the dense formulation
    x = _np(inp["x"])
    logits = x @ _np(inp["w_gate"])
    sel = np.take_along_axis(logits, given, axis=1)
    w = np.exp(sel - sel.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    y_ref = np.zeros_like(y)
    for s in range(20):
        for j in range(2):
            e = given[s, j]
            h = _silu_np(x[s] @ _np(inp["w_gate_e"][e])) * (x[s] @ _np(inp["w_up"][e]))
            y_ref[s] += w[s, j] * (h @ _np(inp["w_down"][e]))
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-14)


def test_token_subset_matches_full(oracle_lib):
    wl = W.custom("sub", S=33, D=16, F=24, E=4, k=2, dtype="bf16")
    inp = W.make_inputs(wl)
    args = (inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], 2)
    y, te, tw = oracle_lib.mlp_forward(*args)
    sub = np.array([32, 0, 17], np.int32)
    ys, tes, tws = oracle_lib.mlp_forward(*args, tokens=sub)
    assert np.array_equal(ys, y[sub]) and np.array_equal(tes, te[sub])


def test_expert_hidden_matches_numpy(oracle_lib):
    wl = W.custom("h", S=10, D=24, F=40, E=3, k=1, dtype="bf16")
    inp = W.make_inputs(wl)
    x = _np(inp["x"])
    for s, e in [(0, 0), (9, 2), (4, 1)]:
        h = oracle_lib.expert_hidden(inp["x"], inp["w_gate_e"], inp["w_up"], s, e)
        ref = _silu_np(x[s] @ _np(inp["w_gate_e"][e])) * (x[s] @ _np(inp["w_up"][e]))
        assert np.allclose(h, ref, rtol=1e-12, atol=1e-15)
    # the batched form returns the same rows, in the order of the pairs
    toks, exps = np.array([4, 0, 9, 4], np.int32), np.array([1, 0, 2, 2], np.int32)
    hb = oracle_lib.expert_hidden_rows(inp["x"], inp["w_gate_e"], inp["w_up"], toks, exps)
    for i in range(4):
        assert np.array_equal(hb[i], oracle_lib.expert_hidden(inp["x"], inp["w_gate_e"],
                                                              inp["w_up"], toks[i], exps[i]))


# ----------------------------------------------------------------------------------------------
# ParallelLinear (scatter_linear)
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("gather_in", [True, False])
@pytest.mark.parametrize("scatter_out", [True, False])
@pytest.mark.parametrize("gated", [True, False])
def test_scatter_linear_dense_mask(oracle_lib, gather_in, scatter_out, gated):
    S, k, E, Din, Dout = 23, 2, 5, 12, 9
    gen = torch.Generator().manual_seed(11)
    te = W.make_top_experts(S, k, E, seed=5).numpy()
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, E)
    Wt = torch.randn(E, Din, Dout, generator=gen).numpy().astype(np.float64)
    g = torch.rand(S, k, generator=gen).numpy().astype(np.float64) if gated else None
    if gather_in:
        X = torch.randn(S, Din, generator=gen).numpy().astype(np.float64)
    else:
        X = torch.randn(S * k, Din, generator=gen).numpy().astype(np.float64)
    Y = oracle_lib.scatter_linear(X.astype(np.float32), Wt.astype(np.float32), k, sorted_rows,
                                  offsets, None if g is None else g.astype(np.float32),
                                  gather_in=gather_in, scatter_out=scatter_out, S=S)
    Xf, Wf = X.astype(np.float32).astype(np.float64), Wt.astype(np.float32).astype(np.float64)
    gf = None if g is None else g.astype(np.float32).astype(np.float64)
    # dense form: every route through every expert, masked by the routing one-hot
    R = S * k
    src = np.repeat(Xf, k, axis=0) if gather_in else Xf[sparse_rows]   # src indexed by route i
    per_route = np.zeros((R, Dout))
    for e in range(E):
        mask = (te.reshape(-1) == e).astype(np.float64)[:, None]
        per_route += mask * (src @ Wf[e])
    if gf is not None:
        per_route *= gf.reshape(-1)[:, None]
    if scatter_out:
        ref = per_route.reshape(S, k, Dout).sum(axis=1)
    else:
        ref = per_route[sorted_rows]
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
