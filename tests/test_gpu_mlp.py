"""The whole MoE expert-MLP forward on the GPU against the oracle.

For every case: the GPU's routing is checked against the oracle's (near-tie rule), the sparse map
the GPU built from its own routing is compared bit-exactly with the oracle's map of that routing,
sampled rows of the intermediate h are compared with the oracle's expert hidden rows, and the
output of sampled tokens is compared with the oracle forward run on the GPU's routing, within
max-abs 2e-2 and relative Frobenius 1e-2. Small cases check every token; the full workloads (the
launch configuration the bench times) check 1024 seeded tokens plus every token routed to the three
least-loaded non-empty experts (where the schedule's partial tiles and any short-expert tile shape
sit), 256 sampled h rows, and the whole sparse map.

Sources: "ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs", "3. Assembling the ScatterMoE
FFN Block"; the router equation of "1. The Dynamic Routing Imbalance Dilemma".
"""
import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import MAX_ABS, REL_FROB, check_routing, rel_frob, sample_tokens

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "ragged_bf16": W.custom("ragged_bf16", S=700, D=200, F=328, E=3, k=2, dtype="bf16"),
    "ragged_f32": W.custom("ragged_f32", S=700, D=200, F=328, E=3, k=2, dtype="f32"),
    "zipf_small": W.custom("zipf_small", S=1000, D=256, F=384, E=16, k=4, dtype="bf16",
                           router_std="1/sqrt(D)", zipf_s=1.2),
    "dense_e1": W.custom("dense_e1", S=300, D=64, F=128, E=1, k=1, dtype="bf16"),
    "one_token": W.custom("one_token", S=1, D=128, F=256, E=8, k=8, dtype="bf16"),
    "e256": W.custom("e256", S=600, D=96, F=64, E=256, k=8, dtype="bf16",
                     router_std="1/sqrt(D)"),
    # 600 rows an expert, F = 2048: GEMM1 reads x rows copied to slot order (a K tail: D = 72)
    "pregather": W.custom("pregather", S=1200, D=72, F=2048, E=2, k=1, dtype="bf16"),
}

FULL_WORKLOADS = ["mixtral_prefill", "mixtral_decode", "e128", "zipf64"]
FULL_TOKENS = 1024
FULL_H_ROWS = 256


def _forward(moe, inp, w):
    dev = inp["x"].device
    ws = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
    out = moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                          inp["w_down"], w.k, logit_bias=inp["logit_bias"], ws=ws)
    moe.check_device_status(ws)
    views = {n: ws.view(n).cpu().numpy() for n in
             ("top_experts", "top_weights", "expert_counts", "expert_offsets", "sparse_rows",
              "sorted_rows")}
    return out, ws, views


def _check_case(oracle_lib, moe, w, inp_gpu, tokens, h_rows=64):
    out, ws, v = _forward(moe, inp_gpu, w)
    # one float32 host copy of every input (bf16 values are exact in float32)
    cpu = {k: (t.float().cpu().numpy() if t is not None else None) for k, t in inp_gpu.items()}
    te = v["top_experts"]
    # 1. routing (near-tie rule) on the sampled tokens
    logits, absdot = oracle_lib.router_logits(cpu["x"], cpu["w_gate"], cpu["logit_bias"],
                                              tokens=tokens)
    ote, _ = oracle_lib.topk_softmax(logits, w.k)
    check_routing(te[tokens], ote, logits, absdot, w.D)
    # 2. the map of the GPU's routing, bit-exact, on all routes
    ref_map = oracle_lib.sparse_map(te, w.E)
    for name, ref in zip(("expert_counts", "expert_offsets", "sparse_rows", "sorted_rows"),
                         ref_map):
        assert np.array_equal(v[name], ref), name
    # 3. sampled h rows (slot order) against the oracle's hidden row of (token, expert)
    h = ws.view("h")
    rng = np.random.default_rng(1)
    R = w.S * w.k
    if R > 0:
        slots = np.sort(rng.choice(R, size=min(h_rows, R), replace=False))
        routes = v["sorted_rows"][slots]
        ref = oracle_lib.expert_hidden_rows(cpu["x"], cpu["w_gate_e"], cpu["w_up"],
                                            routes // w.k, te.reshape(-1)[routes])
        got = h[torch.as_tensor(slots, device=h.device)].float().cpu().numpy()
        for j, p in enumerate(slots):
            assert rel_frob(got[j], ref[j]) < 1e-2, (int(p), rel_frob(got[j], ref[j]))
    # 4. the output on the GPU's routing
    y_ref, _, _ = oracle_lib.mlp_forward(cpu["x"], cpu["w_gate"], cpu["w_gate_e"], cpu["w_up"],
                                         cpu["w_down"], w.k, bias=cpu["logit_bias"],
                                         tokens=tokens, given_top_experts=te)
    y = out.cpu().numpy()[tokens]
    assert np.all(np.isfinite(y))
    mx = float(np.abs(y - y_ref).max())
    rf = rel_frob(y, y_ref)
    assert mx < MAX_ABS, mx
    assert rf < REL_FROB, rf
    return out, v, mx, rf


@pytest.mark.parametrize("cta", ["0", "1"])
@pytest.mark.parametrize("name", list(SMALL))
def test_mlp_small_all_tokens(oracle_lib, moe, monkeypatch, name, cta):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)  # one-CTA and CTA-pair grouped GEMMs
    w = SMALL[name]
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_inputs(w).items()}
    _check_case(oracle_lib, moe, w, inp, np.arange(w.S, dtype=np.int32))


@pytest.mark.parametrize("cta", ["0", "1"])
def test_mlp_slot_ordered_x_matches_gather_on_load(moe, monkeypatch, cta):
    """GEMM1 on x rows copied to slot order runs the same MMAs in the same K order as GEMM1
    gathering them on load: h and the output are bit-identical (MOE_PREGATHER=0 turns the copy
    off), and the copy is the x rows in slot order."""
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    w = SMALL["pregather"]
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_inputs(w).items()}
    out1, ws1, v1 = _forward(moe, inp, w)
    xs = ws1.view("x_sorted")
    routes = torch.from_numpy(v1["sorted_rows"].astype(np.int64)).cuda()
    assert torch.equal(xs, inp["x"][routes // w.k])
    monkeypatch.setenv("MOE_PREGATHER", "0")
    out0, ws0, v0 = _forward(moe, inp, w)
    assert torch.equal(ws0.view("h"), ws1.view("h"))
    assert torch.equal(out0, out1)


def test_mlp_empty_batch(moe):
    w = W.custom("empty", S=0, D=64, F=64, E=4, k=2, dtype="bf16")
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_inputs(w).items()}
    out, _, v = _forward(moe, inp, w)
    assert out.shape == (0, 64)
    assert v["expert_counts"].tolist() == [0] * 4


def test_mlp_repeat_calls_identical_map(oracle_lib, moe):
    w = SMALL["zipf_small"]
    inp = {k: (t.cuda() if t is not None else None) for k, t in W.make_inputs(w).items()}
    _, _, v1 = _forward(moe, inp, w)
    out2, _, v2 = _forward(moe, inp, w)
    for n in v1:
        assert np.array_equal(v1[n], v2[n]), n


@pytest.mark.parametrize("name", FULL_WORKLOADS)
def test_mlp_full_workload_sampled(oracle_lib, moe, name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, device="cuda")
    # every token of the three least-loaded non-empty experts, found from a first GPU routing
    # pass (the forward below routes the same way: the map comparison checks that bit-exactly)
    te, _ = moe.route_topk(inp["x"], inp["w_gate"], w.k, inp["logit_bias"])
    te = te.cpu().numpy()
    counts = np.bincount(te.reshape(-1), minlength=w.E)
    least = [e for e in np.argsort(counts, kind="stable") if counts[e] > 0][:3]
    must = np.nonzero(np.isin(te, least).any(axis=1))[0]
    assert len(must) >= max(1, counts[least].max())
    toks = sample_tokens(w.S, FULL_TOKENS, seed=0, must=must)
    _, v, _, _ = _check_case(oracle_lib, moe, w, inp, toks, h_rows=FULL_H_ROWS)
    assert np.array_equal(v["top_experts"], te)
