"""Pins of the oracle's Mixture-of-Attention forward ("2. Generalization to Mixture of Attention
(MoA)" of the ScatterMoE guide): routed per-expert query and output projections around causal
attention over shared keys and values.

Independent of the oracle's loops:
  * the dense all-experts-then-mask formulation in torch float64, with the attention core from
    torch's scaled_dot_product_attention (causal), weighted by the top-k mask times the softmax
    of the selected logits (the routing taken from the oracle);
  * one token (S = 1): every query attends only to itself, so y = sum_j w_j (v_0 W_o[e_j]) in
    closed form, whatever the queries;
  * one expert, k = 1: plain causal multi-head attention with projections (through the same
    library attention core).
"""
import numpy as np
import pytest
import torch


def _inputs(S, D, H, dh, E, seed):
    g = torch.Generator().manual_seed(seed)
    HD = H * dh
    x = torch.randn(S, D, generator=g)
    wg = torch.randn(D, E, generator=g) / D ** 0.5
    wq = torch.randn(E, D, HD, generator=g) / D ** 0.5
    wk = torch.randn(D, HD, generator=g) / D ** 0.5
    wv = torch.randn(D, HD, generator=g) / D ** 0.5
    wo = torch.randn(E, HD, D, generator=g) / HD ** 0.5
    return x, wg, wq, wk, wv, wo


def _dense(x, wg, wq, wk, wv, wo, H, te):
    x64 = x.double()
    S = x.shape[0]
    E, D, HD = wq.shape
    dh = HD // H
    l = x64 @ wg.double()
    Jt = torch.from_numpy(te.astype(np.int64))
    w = torch.softmax(l.gather(1, Jt), dim=1)
    K = (x64 @ wk.double()).view(S, H, dh).transpose(0, 1)
    V = (x64 @ wv.double()).view(S, H, dh).transpose(0, 1)
    y = torch.zeros(S, D, dtype=torch.float64)
    for e in range(E):
        Q = (x64 @ wq[e].double()).view(S, H, dh).transpose(0, 1)
        O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
        Ye = O.transpose(0, 1).reshape(S, HD) @ wo[e].double()
        c = (w * (Jt == e).double()).sum(dim=1, keepdim=True)
        y = y + c * Ye
    return y.numpy()


@pytest.mark.parametrize("S,D,H,dh,E,k", [(17, 12, 2, 4, 4, 2), (9, 8, 1, 8, 3, 3), (24, 16, 4, 2, 6, 2)])
def test_moa_matches_dense_library_attention(oracle_lib, S, D, H, dh, E, k):
    x, wg, wq, wk, wv, wo = _inputs(S, D, H, dh, E, seed=S + E)
    out, te, tw = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, k, H)
    ref = _dense(x, wg, wq, wk, wv, wo, H, te)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(tw.sum(axis=1), 1.0, rtol=1e-12)


def test_moa_single_token_closed_form(oracle_lib):
    x, wg, wq, wk, wv, wo = _inputs(1, 10, 2, 3, 5, seed=2)
    out, te, tw = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, 2, 2)
    v0 = x.double().numpy() @ wv.double().numpy()            # [1, H*dh]
    ref = sum(tw[0, j] * (v0 @ wo[te[0, j]].double().numpy()) for j in range(2))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_moa_one_expert_is_causal_attention(oracle_lib):
    S, D, H, dh = 11, 8, 2, 4
    x, wg, wq, wk, wv, wo = _inputs(S, D, H, dh, 1, seed=5)
    out, te, tw = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, 1, H)
    assert np.all(te == 0) and np.allclose(tw, 1.0)
    x64 = x.double()
    Q = (x64 @ wq[0].double()).view(S, H, dh).transpose(0, 1)
    K = (x64 @ wk.double()).view(S, H, dh).transpose(0, 1)
    V = (x64 @ wv.double()).view(S, H, dh).transpose(0, 1)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    ref = (O.transpose(0, 1).reshape(S, H * dh) @ wo[0].double()).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_moa_query_token_subset_matches_full(oracle_lib):
    """A list of query tokens gives exactly the rows of the full forward, in list order (keys and
    values of every earlier token are still used), with and without a given routing."""
    S, D, H, dh, E, k = 23, 16, 2, 8, 4, 2
    x, wg, wq, wk, wv, wo = _inputs(S, D, H, dh, E, seed=12)
    full, te, tw = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, k, H)
    toks = np.array([22, 0, 7, 7, 15], dtype=np.int32)
    sub, tes, tws = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, k, H, tokens=toks)
    assert np.array_equal(sub, full[toks]) and np.array_equal(tes, te[toks])
    assert np.array_equal(tws, tw[toks])
    given = np.roll(te, 1, axis=1).astype(np.int32)
    full_g, _, _ = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, k, H, given_top_experts=given)
    sub_g, tes_g, _ = oracle_lib.moa_forward(x, wg, wq, wk, wv, wo, k, H, given_top_experts=given,
                                             tokens=toks)
    assert np.array_equal(sub_g, full_g[toks]) and np.array_equal(tes_g, given[toks])
