"""Pins of the oracle's ParallelLinear backward ("3. Fused Backward Pass Dynamics" of the ScatterMoE
guide: the input gradient scatters W-transposed products of the gated output gradient back to the
tokens, the weight gradient of expert e sums x^T times the gated output gradient over its tokens).

Each pin is independent of the backward's own loops:
  * adjoint identities: Y is linear in X, in W and in the gates, so <dY, Y> equals <dX, X>,
    <dW, W> and <dgates, gates> (a transposed operand, a wrong slot-to-token map or a dropped gate
    breaks one of them);
  * finite differences of L = <dY, Y> (exact for a linear map, with the step measured after fp32
    rounding of the perturbed input);
  * E = 1, k = 1 with the identity map reduces to dX = dY W^T and dW = X^T dY (numpy matmul).
"""
import numpy as np
import pytest

import moe_workloads as W

MODES = [(True, True), (False, True), (True, False), (False, False)]


def _case(S, k, E, Din, Dout, seed, gated):
    rng = np.random.default_rng(seed)
    te = W.make_top_experts(S, k, E, seed=seed, mode="uniform").numpy()
    X_tok = rng.standard_normal((S, Din)).astype(np.float32)
    Wt = (rng.standard_normal((E, Din, Dout)) * 0.3).astype(np.float32)
    g = rng.random(S * k).astype(np.float32) if gated else None
    return te, X_tok, Wt, g, rng


def _inputs(oracle_lib, S, k, E, Din, Dout, seed, gated, gather_in, scatter_out):
    te, X_tok, Wt, g, rng = _case(S, k, E, Din, Dout, seed, gated)
    counts, offsets, sparse_rows, sorted_rows = oracle_lib.sparse_map(te, E)
    X = X_tok if gather_in else rng.standard_normal((S * k, Din)).astype(np.float32)
    dY = rng.standard_normal((S if scatter_out else S * k, Dout)).astype(np.float32)
    return X, Wt, g, dY, sorted_rows, offsets


@pytest.mark.parametrize("gather_in,scatter_out", MODES)
@pytest.mark.parametrize("gated", [True, False])
def test_backward_adjoint_identities(oracle_lib, gather_in, scatter_out, gated):
    S, k, E, Din, Dout = 37, 3, 5, 11, 7
    X, Wt, g, dY, sorted_rows, offsets = _inputs(oracle_lib, S, k, E, Din, Dout, 5, gated,
                                                 gather_in, scatter_out)
    Y = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, g, gather_in=gather_in,
                                  scatter_out=scatter_out, S=S)
    grads = oracle_lib.scatter_linear_backward(X, Wt, dY, k, sorted_rows, offsets, g,
                                               gather_in=gather_in, scatter_out=scatter_out, S=S)
    lhs = float(np.sum(dY.astype(np.float64) * Y))
    assert grads["dX"].shape == X.shape and grads["dW"].shape == Wt.shape
    for name, inp in (("dX", X), ("dW", Wt)) + ((("dgates", g),) if gated else ()):
        rhs = float(np.sum(grads[name] * inp.astype(np.float64)))
        assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1.0), (name, lhs, rhs)


@pytest.mark.parametrize("gather_in,scatter_out", MODES)
def test_backward_finite_differences(oracle_lib, gather_in, scatter_out):
    S, k, E, Din, Dout = 5, 2, 3, 4, 3
    X, Wt, g, dY, sorted_rows, offsets = _inputs(oracle_lib, S, k, E, Din, Dout, 9, True,
                                                 gather_in, scatter_out)
    grads = oracle_lib.scatter_linear_backward(X, Wt, dY, k, sorted_rows, offsets, g,
                                               gather_in=gather_in, scatter_out=scatter_out, S=S)

    def loss(Xv, Wv, gv):
        Y = oracle_lib.scatter_linear(Xv, Wv, k, sorted_rows, offsets, gv, gather_in=gather_in,
                                      scatter_out=scatter_out, S=S)
        return float(np.sum(dY.astype(np.float64) * Y))

    def fd(arr, idx, build):
        up, dn = arr.copy(), arr.copy()
        up[idx] = np.float32(arr[idx] + np.float32(0.125))
        dn[idx] = np.float32(arr[idx] - np.float32(0.125))
        step = float(up[idx]) - float(dn[idx])   # the perturbation fp32 actually represents
        return (loss(*build(up)) - loss(*build(dn))) / step

    rng = np.random.default_rng(0)
    for _ in range(6):
        ix = tuple(int(rng.integers(0, n)) for n in X.shape)
        got = fd(X, ix, lambda a: (a, Wt, g))
        assert got == pytest.approx(grads["dX"][ix], rel=1e-9, abs=1e-9)
        iw = tuple(int(rng.integers(0, n)) for n in Wt.shape)
        got = fd(Wt, iw, lambda a: (X, a, g))
        assert got == pytest.approx(grads["dW"][iw], rel=1e-9, abs=1e-9)
        ig = (int(rng.integers(0, g.shape[0])),)
        got = fd(g, ig, lambda a: (X, Wt, a))
        assert got == pytest.approx(grads["dgates"][ig], rel=1e-9, abs=1e-9)


def test_backward_single_expert_is_matmul(oracle_lib):
    S, Din, Dout = 23, 9, 6
    rng = np.random.default_rng(3)
    X = rng.standard_normal((S, Din)).astype(np.float32)
    Wt = rng.standard_normal((1, Din, Dout)).astype(np.float32)
    dY = rng.standard_normal((S, Dout)).astype(np.float32)
    sorted_rows = np.arange(S, dtype=np.int32)
    offsets = np.array([0, S], dtype=np.int32)
    for gi, so in MODES:
        grads = oracle_lib.scatter_linear_backward(X, Wt, dY, 1, sorted_rows, offsets, None,
                                                   gather_in=gi, scatter_out=so, S=S)
        x64, w64, d64 = X.astype(np.float64), Wt[0].astype(np.float64), dY.astype(np.float64)
        np.testing.assert_allclose(grads["dX"], d64 @ w64.T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(grads["dW"][0], x64.T @ d64, rtol=1e-12, atol=1e-12)


def test_backward_empty_expert_has_zero_weight_gradient(oracle_lib):
    te = np.array([[0, 2], [2, 0], [0, 2]], dtype=np.int32)   # expert 1 of 3 gets no token
    counts, offsets, _, sorted_rows = oracle_lib.sparse_map(te, 3)
    rng = np.random.default_rng(4)
    X = rng.standard_normal((3, 4)).astype(np.float32)
    Wt = rng.standard_normal((3, 4, 5)).astype(np.float32)
    dY = rng.standard_normal((3, 5)).astype(np.float32)
    grads = oracle_lib.scatter_linear_backward(X, Wt, dY, 2, sorted_rows, offsets, None, S=3)
    assert counts[1] == 0
    assert np.all(grads["dW"][1] == 0.0)
    assert np.any(grads["dW"][0] != 0.0) and np.any(grads["dW"][2] != 0.0)
