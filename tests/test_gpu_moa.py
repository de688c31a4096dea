"""Mixture of Attention forward on the GPU against the oracle ("2. Generalization to Mixture of
Attention (MoA)" of the ScatterMoE guide; the ScatterMoE abstract's MoA demonstration).

Every case checks, in order:
  * the GPU's routing against the oracle router (near-tie rule);
  * the sparse map of that routing, bit-exactly;
  * the output against the oracle's MoA forward run on the GPU's routing, within max-abs 2e-2 and
    relative Frobenius 1e-2.
The MoA output of token s depends only on tokens 0..s (causal attention), so at the full
Mixtral-shaped size the first tokens of the GPU's output are checked against the oracle run on
that prefix of the sequence, and 48 tokens spread over the whole sequence (key-block edges, the
last token, seeded random ones) against the oracle's forward for that list of query tokens.

Tolerance: q, K, V, the softmax weights and the attention output are each rounded once to bf16
(relative 2^-9). The output projection sums H*dh such terms with random signs, so the error is of
the same order as in the expert MLP's second GEMM (about 1e-3 relative).
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import MAX_ABS, REL_FROB, check_routing, rel_frob

pytestmark = pytest.mark.gpu

MW = W.MoaWorkload
SMALL = {
    # 5 query tiles, 5 key blocks with a ragged tail
    "moa_small": MW("moa_small", S=300, D=256, H=2, dh=128, E=8, k=2),
    "moa_dh64": MW("moa_dh64", S=513, D=128, H=3, dh=64, E=4, k=1),
    "moa_zipf": MW("moa_zipf", S=700, D=192, H=2, dh=64, E=16, k=4, router_std="1/sqrt(D)",
                   zipf_s=1.2),
    "moa_one_token": MW("moa_one_token", S=1, D=64, H=1, dh=128, E=8, k=8),
    "moa_e1": MW("moa_e1", S=260, D=64, H=2, dh=64, E=1, k=1),
    "moa_long": MW("moa_long", S=1500, D=256, H=2, dh=128, E=8, k=2),
}


def _run(moe, w, inp):
    ws = moe.MoaWorkspace(w.S, w.D, w.HD, w.E, w.k, inp["x"].device)
    out = moe.moa_forward(inp["x"], inp["w_gate"], inp["w_q"], inp["w_kv"], inp["w_o"], w.k, w.H,
                          logit_bias=inp["logit_bias"], ws=ws)
    moe.check_device_status(ws)
    views = {n: ws.view(n).cpu().numpy() for n in
             ("top_experts", "top_weights", "expert_counts", "expert_offsets", "sparse_rows",
              "sorted_rows")}
    return out, views


def _host(inp, S=None):
    cpu = {k: (t.float().cpu().numpy() if t is not None else None) for k, t in inp.items()}
    if S is not None:
        cpu["x"] = cpu["x"][:S]
    return cpu


def _oracle(oracle_lib, w, cpu, te):
    HD = w.HD
    return oracle_lib.moa_forward(cpu["x"], cpu["w_gate"], cpu["w_q"], cpu["w_kv"][:, :HD],
                                  cpu["w_kv"][:, HD:], cpu["w_o"], w.k, w.H,
                                  bias=cpu["logit_bias"], given_top_experts=te)


def _check(oracle_lib, w, out, v, cpu, S_check):
    te = v["top_experts"][:S_check]
    tokens = np.arange(S_check, dtype=np.int32)
    logits, absdot = oracle_lib.router_logits(cpu["x"], cpu["w_gate"], cpu["logit_bias"],
                                              tokens=tokens)
    ote, _ = oracle_lib.topk_softmax(logits, w.k)
    check_routing(te, ote, logits, absdot, w.D)
    y_ref, _, tw_ref = _oracle(oracle_lib, w, cpu, te)
    np.testing.assert_allclose(v["top_weights"][:S_check], tw_ref, atol=1e-5)
    y = out.cpu().numpy()[:S_check]
    assert np.all(np.isfinite(y))
    mx = float(np.abs(y - y_ref).max())
    rf = rel_frob(y, y_ref)
    assert mx < MAX_ABS, mx
    assert rf < REL_FROB, rf
    return mx, rf


@pytest.mark.parametrize("cta", ["0", "1"])
@pytest.mark.parametrize("name", list(SMALL))
def test_moa_small_all_tokens(oracle_lib, moe, monkeypatch, name, cta):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)  # one-CTA and CTA-pair grouped GEMMs
    w = SMALL[name]
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_moa_inputs(w).items()}
    out, v = _run(moe, w, inp)
    ref_map = oracle_lib.sparse_map(v["top_experts"], w.E)
    for name_, ref in zip(("expert_counts", "expert_offsets", "sparse_rows", "sorted_rows"),
                          ref_map):
        assert np.array_equal(v[name_], ref), name_
    _check(oracle_lib, w, out, v, _host(inp), w.S)


def test_moa_empty_sequence(moe):
    w = MW("moa_empty", S=0, D=64, H=1, dh=64, E=4, k=2)
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_moa_inputs(w).items()}
    out, v = _run(moe, w, inp)
    assert out.shape == (0, 64)
    assert v["expert_counts"].tolist() == [0] * 4


def test_moa_repeat_calls_identical(moe):
    w = SMALL["moa_zipf"]
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_moa_inputs(w).items()}
    out1, v1 = _run(moe, w, inp)
    out2, v2 = _run(moe, w, inp)
    for n in v1:
        assert np.array_equal(v1[n], v2[n]), n
    # the attention core and the GEMMs are deterministic; only the scatter-add order may differ
    assert float((out1 - out2).abs().max()) < 1e-5


def test_moa_unsupported_forms(moe):
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros(4, 64, 96, dtype=torch.bfloat16, device="cuda")   # dh = 96
    wkv = torch.zeros(64, 192, dtype=torch.bfloat16, device="cuda")
    wo = torch.zeros(4, 96, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moa_forward(x, wg, wq, wkv, wo, 2, 1)
    assert ei.value.code == -2


@pytest.mark.parametrize("name", list(W.MOA_WORKLOADS))
def test_moa_full_workload_prefix(oracle_lib, moe, name):
    """The launch configuration the bench times; tokens [0, 40) checked against the oracle run on
    that prefix (causality makes them independent of the later tokens), then 48 tokens spread over
    the whole sequence, the last one included, whose attention spans run up to every key."""
    w = W.MOA_WORKLOADS[name]
    inp = W.make_moa_inputs(w, device="cuda")
    out, v = _run(moe, w, inp)
    ref_map = oracle_lib.sparse_map(v["top_experts"], w.E)
    for name_, ref in zip(("expert_counts", "expert_offsets", "sparse_rows", "sorted_rows"),
                          ref_map):
        assert np.array_equal(v[name_], ref), name_
    S0 = 40
    _check(oracle_lib, w, out, v, _host(inp, S=S0), S0)
    assert bool(torch.isfinite(out).all())
    # sampled tokens across the sequence: block edges (multiples of 128 and one past), the last
    # token and seeded random ones; the oracle computes keys and values of every token
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([
        [127, 128, 129, 1023, 1024, 2047, 2048, w.S - 2, w.S - 1],
        rng.choice(w.S, size=39, replace=False)])).astype(np.int32)
    cpu = _host(inp)
    te = v["top_experts"]
    logits, absdot = oracle_lib.router_logits(cpu["x"], cpu["w_gate"], cpu["logit_bias"],
                                              tokens=toks)
    ote, _ = oracle_lib.topk_softmax(logits, w.k)
    check_routing(te[toks], ote, logits, absdot, w.D)
    HD = w.HD
    y_ref, _, tw_ref = oracle_lib.moa_forward(cpu["x"], cpu["w_gate"], cpu["w_q"],
                                              cpu["w_kv"][:, :HD], cpu["w_kv"][:, HD:],
                                              cpu["w_o"], w.k, w.H, bias=cpu["logit_bias"],
                                              given_top_experts=te, tokens=toks)
    np.testing.assert_allclose(v["top_weights"][toks], tw_ref, atol=1e-5)
    y = out.cpu().numpy()[toks]
    assert np.abs(y - y_ref).max() < MAX_ABS
    assert rel_frob(y, y_ref) < REL_FROB
