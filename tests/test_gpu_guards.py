"""Out-of-bounds write checks, standing in for a memory sanitizer (none is available where this
library is measured).

1. Guard regions (release build): the forward's output, its workspace and ParallelLinear's output
   sit inside larger buffers whose surrounding bytes, and the padding between the workspace's
   sections, hold a fill pattern. Small cases reach every tail of the tile schedule (an expert's
   rows not a multiple of the tile height, empty experts, fewer routes than one tile, ragged N and
   K), on the one-CTA and the CTA-pair kernels; afterwards every guard byte must be unchanged.
2. The debug build (libmoe_b200_debug.so, MOE_DEBUG=1): on valid inputs it reports nothing and
   gives the release build's map and h bit-identically. Given a slot table with route indices
   outside [0, S*k), or expert offsets past the slot count, its device bounds checks skip those
   accesses and report MOE_ERR_BAD_INDEX; the valid rows are still right and no guard byte moves.

Source of the index ranges: "ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs",
"2. Grouped Coordinate Indexing Without Padding" (an expert's slots lie in
[offsets[e], offsets[e+1]); a slot's route i gives token i / k).
"""
import contextlib

import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import rel_frob

pytestmark = pytest.mark.gpu

FILL_U8 = 0xA5
GUARD = 4096  # bytes of guard on each side (a multiple of 256 keeps the interior aligned)

CASES = {
    # ragged N and K, ~120 rows an expert (one tile each, none a multiple of 128)
    "tails_bf16": W.custom("tails_bf16", S=300, D=136, F=200, E=5, k=2, dtype="bf16"),
    # skew: empty experts and tiny ones
    "zipf_bf16": W.custom("zipf_bf16", S=257, D=64, F=72, E=16, k=3, dtype="bf16",
                          router_std="1/sqrt(D)", zipf_s=1.2),
    # fewer routes than one tile
    "few_routes": W.custom("few_routes", S=3, D=72, F=64, E=4, k=1, dtype="bf16"),
    # fp32 (tf32 MMAs), several tiles per expert with a short last tile
    "tails_f32": W.custom("tails_f32", S=700, D=200, F=328, E=3, k=2, dtype="f32"),
    # x rows copied to slot order before GEMM1 (experts of >= 384 rows, F >= 2048); ragged tiles
    "pregather": W.custom("pregather", S=1000, D=136, F=2056, E=2, k=1, dtype="bf16"),
}


@contextlib.contextmanager
def _using(moe, lib):
    old = moe._lib()
    moe._LIB = lib
    try:
        yield
    finally:
        moe._LIB = old


def _guarded(n_bytes, device):
    big = torch.full((GUARD + n_bytes + GUARD,), FILL_U8, dtype=torch.uint8, device=device)
    return big, big[GUARD:GUARD + n_bytes]


def _assert_untouched(u8, what):
    bad = (u8 != FILL_U8).nonzero()
    assert bad.numel() == 0, f"{what}: {bad.numel()} guard bytes changed, first at {bad[:4].tolist()}"


def _forward_guarded(moe, w, inp):
    dev = inp["x"].device
    ws = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, inp["x"].dtype, dev)
    n_ws = ws.buf.numel()
    ws_big, ws.buf = _guarded(n_ws, dev)
    out_big, out_u8 = _guarded(w.S * w.D * 4, dev)
    out = out_u8.view(torch.float32).view(w.S, w.D)
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k,
                    logit_bias=inp["logit_bias"], out=out, ws=ws)
    moe.check_device_status(ws)
    return ws, ws_big, out, out_big


def _check_forward_guards(moe, w, ws, ws_big, out_big):
    S, D, F, E, k = w.S, w.D, w.F, w.E, w.k
    n_ws = ws.buf.numel()
    _assert_untouched(ws_big[:GUARD], "before the workspace")
    _assert_untouched(ws_big[GUARD + n_ws:], "after the workspace")
    _assert_untouched(out_big[:GUARD], "before out")
    _assert_untouched(out_big[GUARD + S * D * 4:], "after out")
    # the status word is 4 bytes of a 256-byte area; every section's padding is untouched
    _assert_untouched(ws.buf[4:256], "status area")
    R = S * k
    hb = 2 if w.dtype == "bf16" else 4
    sections = [("top_experts", R * 4), ("top_weights", R * 4), ("expert_counts", E * 4),
                ("expert_offsets", (E + 1) * 4), ("sparse_rows", R * 4), ("sorted_rows", R * 4),
                ("h", R * F * hb)]
    code = moe.MOE_BF16 if w.dtype == "bf16" else moe.MOE_F32
    if moe.workspace_view("x_sorted", S, D, F, E, k, code) >= 0:
        sections.append(("x_sorted", R * D * hb))
    spans = sorted((moe.workspace_view(n, S, D, F, E, k, code), sz, n) for n, sz in sections)
    for (off, sz, name), nxt in zip(spans, spans[1:] + [(n_ws, 0, "end")]):
        if name == "sorted_rows":
            continue  # the map's scratch follows the slot table
        _assert_untouched(ws.buf[off + sz:nxt[0]], f"padding after {name}")


@pytest.mark.parametrize("cta", ["0", "1"])
@pytest.mark.parametrize("name", list(CASES))
def test_forward_writes_stay_inside_their_buffers(oracle_lib, moe, monkeypatch, name, cta):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    w = CASES[name]
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    ws, ws_big, out, out_big = _forward_guarded(moe, w, inp)
    torch.cuda.synchronize()
    _check_forward_guards(moe, w, ws, ws_big, out_big)
    # and the result is the forward's (the oracle on the GPU's routing)
    te = ws.view("top_experts").cpu().numpy()
    cpu = {n: (t.float().cpu().numpy() if t is not None else None) for n, t in inp.items()}
    ref, _, _ = oracle_lib.mlp_forward(cpu["x"], cpu["w_gate"], cpu["w_gate_e"], cpu["w_up"],
                                       cpu["w_down"], w.k, bias=cpu["logit_bias"],
                                       given_top_experts=te)
    assert rel_frob(out.cpu().numpy(), ref) < 1e-2


def _scatter_case(seed=3, S=300, k=2, E=7, Din=72, Dout=264):
    te = W.make_top_experts(S, k, E, seed=seed, mode="zipf")
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(S, Din, generator=gen).to(torch.bfloat16)
    Wt = (torch.randn(E, Din, Dout, generator=gen) * 0.05).to(torch.bfloat16)
    g = torch.rand(S * k, generator=gen)
    return te, X, Wt, g


def _scatter_guarded(moe, X, Wt, k, sorted_rows, offsets, g, S):
    Dout = Wt.shape[2]
    big, u8 = _guarded(S * Dout * 4, X.device)
    Y = u8.view(torch.float32).view(S, Dout)
    Y.zero_()
    ws = moe.alloc_workspace(256, X.device)
    moe.scatter_linear(X, Wt, k, sorted_rows, offsets, g, out=Y, ws=ws)
    return Y, big, ws


@pytest.mark.parametrize("cta", ["0", "1"])
def test_scatter_linear_writes_stay_inside_out(oracle_lib, moe, monkeypatch, cta):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    te, X, Wt, g = _scatter_case()
    S, k = te.shape
    E, _, Dout = Wt.shape
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    Y, big, ws = _scatter_guarded(moe, X.cuda(), Wt.cuda(), k, torch.from_numpy(sorted_rows).cuda(),
                                  torch.from_numpy(offsets).cuda(), g.cuda(), S)
    moe.check_device_status(ws)
    _assert_untouched(big[:GUARD], "before Y")
    _assert_untouched(big[GUARD + S * Dout * 4:], "after Y")
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, g, S=S)
    assert rel_frob(Y.cpu().numpy(), ref) < 2e-5


@pytest.mark.parametrize("cta", ["0", "1"])
def test_debug_build_matches_release_on_valid_inputs(moe, monkeypatch, cta):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    dbg = moe.debug_lib()
    assert dbg.moe_debug_build() == 1
    w = CASES["zipf_bf16"]
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    ws_r, _, out_r, _ = _forward_guarded(moe, w, inp)
    with _using(moe, dbg):
        ws_d, ws_big, out_d, out_big = _forward_guarded(moe, w, inp)  # raises on any flag
        torch.cuda.synchronize()
        _check_forward_guards(moe, w, ws_d, ws_big, out_big)
    for n in ("top_experts", "expert_counts", "expert_offsets", "sparse_rows", "sorted_rows", "h"):
        assert torch.equal(ws_r.view(n), ws_d.view(n)), n
    assert rel_frob(out_d.cpu().numpy(), out_r.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("cta", ["0", "1"])
def test_debug_build_flags_out_of_range_routes(oracle_lib, moe, monkeypatch, cta):
    """Slots whose route lies outside [0, S*k): the debug build neither reads their token row nor
    writes their output row, reports MOE_ERR_BAD_INDEX, and computes every other slot."""
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    te, X, Wt, g = _scatter_case(seed=9)
    S, k = te.shape
    E, _, Dout = Wt.shape
    R = S * k
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    bad_slots = [0, 5, R - 1]
    corrupt = sorted_rows.copy()
    corrupt[bad_slots] = [R + 1000, -7, 1 << 30]
    dbg = moe.debug_lib()
    with _using(moe, dbg):
        Y, big, ws = _scatter_guarded(moe, X.cuda(), Wt.cuda(), k,
                                      torch.from_numpy(corrupt).cuda(),
                                      torch.from_numpy(offsets).cuda(), g.cuda(), S)
        with pytest.raises(moe.MoeError) as ei:
            moe.check_device_status(ws)
    assert ei.value.code == -7  # MOE_ERR_BAD_INDEX
    _assert_untouched(big[:GUARD], "before Y")
    _assert_untouched(big[GUARD + S * Dout * 4:], "after Y")
    # the oracle with the corrupted slots left out
    keep = np.ones(R, bool)
    keep[bad_slots] = False
    dropped = sorted_rows[bad_slots]
    g_kept = g.clone()
    g_kept[torch.from_numpy(dropped.astype(np.int64))] = 0.0
    ref = oracle_lib.scatter_linear(X, Wt, k, sorted_rows, offsets, g_kept, S=S)
    assert rel_frob(Y.cpu().numpy(), ref) < 2e-5


def test_debug_build_rejects_offsets_past_the_slots(oracle_lib, moe):
    te, X, Wt, g = _scatter_case(seed=4)
    S, k = te.shape
    E = Wt.shape[0]
    _, offsets, _, sorted_rows = oracle_lib.sparse_map(te.numpy(), E)
    past = offsets.copy()
    past[E] = S * k + 64            # the last expert's range runs past the slot table
    decreasing = offsets.copy()
    decreasing[2], decreasing[3] = decreasing[3] + 1, decreasing[2]  # not monotone
    dbg = moe.debug_lib()
    for off in (past, decreasing):
        with _using(moe, dbg):
            Y, big, ws = _scatter_guarded(moe, X.cuda(), Wt.cuda(), k,
                                          torch.from_numpy(sorted_rows).cuda(),
                                          torch.from_numpy(off).cuda(), g.cuda(), S)
            with pytest.raises(moe.MoeError) as ei:
                moe.check_device_status(ws)
        assert ei.value.code == -7
        assert bool((Y == 0).all())  # the schedule was emptied: nothing written
        _assert_untouched(big[:GUARD], "before Y")
        _assert_untouched(big[GUARD + Y.numel() * 4:], "after Y")
