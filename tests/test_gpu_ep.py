"""Expert-parallel kernels on the GPU (ScatterMoE guide, "Combine with Tensor and Pipeline
Parallelism"): dispatch, the expert MLP on received rows, the combine, and whole forwards with
the ranks' exchanges emulated on one GPU.

* moe_ep_dispatch: the map of the routing, bit-exact against the oracle's; the send rows and
  ids exactly equal to x[sorted_rows / k] and top_experts[sorted_rows].
* moe_expert_mlp_forward: every row against the oracle's expert FFN of that row (max-abs 2e-2,
  relative Frobenius 1e-2), one-CTA and CTA-pair GEMMs, bf16 and fp32; an out-of-range id
  raises the device status.
* moe_ep_combine: against an fp64 weighted sum.
* Emulated ranks: n virtual ranks in one process, each with its own tokens and E/n experts. The
  all-to-alls are done with tensor slicing, which matches what NCCL's all_to_all_single moves.
  Every rank's output is compared with the oracle forward of its tokens over all E experts,
  on the GPU's routing.
* ep_mlp_forward over a real NCCL process group of one rank: the same result as mlp_forward.
"""
import os
import socket

import numpy as np
import pytest
import torch

import moe_workloads as W
from parity import MAX_ABS, REL_FROB, rel_frob

pytestmark = pytest.mark.gpu


def _te(S, k, E, seed, mode="uniform"):
    return W.make_top_experts(S, k, E, seed=seed, mode=mode).cuda()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("mode", ["uniform", "zipf"])
def test_ep_dispatch(oracle_lib, moe, dtype, mode):
    S, D, E, k = 300, 200, 16, 4
    x = torch.randn(S, D, generator=torch.Generator().manual_seed(1)).to(dtype).cuda()
    te = _te(S, k, E, 3, mode)
    d = moe.ep_dispatch(x, te, E)
    counts, offsets, sparse, srt = oracle_lib.sparse_map(te.cpu().numpy(), E)
    for name, ref in (("expert_counts", counts), ("expert_offsets", offsets),
                      ("sparse_rows", sparse), ("sorted_rows", srt)):
        assert np.array_equal(d[name].cpu().numpy(), ref), name
    idx = torch.from_numpy(srt.astype(np.int64)).cuda()
    assert torch.equal(d["send_x"], x[idx // k])
    assert torch.equal(d["send_e"], te.reshape(-1)[idx])


def _expert_ref(oracle_lib, xr, ids, base, wge, wup, wd):
    xn, wgn, wun = (t.float().cpu().numpy() for t in (xr, wge, wup))
    wdn = wd.float().cpu().numpy().astype(np.float64)
    ids = ids.cpu().numpy()
    y = np.zeros((xr.shape[0], xr.shape[1]))
    for i in range(xr.shape[0]):
        e = int(ids[i]) - base
        y[i] = oracle_lib.expert_hidden(xn, wgn, wun, i, e) @ wdn[e]
    return y


@pytest.mark.parametrize("cta", ["0", "1"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_expert_mlp_forward(oracle_lib, moe, monkeypatch, cta, dtype):
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    R, D, F, E, base = 700, 256, 384, 8, 8
    w = W.custom("ep_rows", S=R, D=D, F=F, E=E, k=1, dtype="bf16" if dtype == torch.bfloat16
                 else "f32")
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    ids = (_te(R, 1, E, 5, "zipf").reshape(-1) + base).contiguous()
    y = moe.expert_mlp_forward(inp["x"], ids, base, inp["w_gate_e"], inp["w_up"], inp["w_down"])
    ref = _expert_ref(oracle_lib, inp["x"], ids, base, inp["w_gate_e"], inp["w_up"],
                      inp["w_down"])
    got = y.cpu().numpy()
    assert np.abs(got - ref).max() < MAX_ABS
    assert rel_frob(got, ref) < REL_FROB


EDGE_COUNTS = [1, 64, 65, 128, 129, 256, 257, 384, 385, 0]


@pytest.mark.parametrize("cta", ["0", "1"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_expert_mlp_forward_tile_edges(oracle_lib, moe, monkeypatch, cta, dtype):
    """The fused gate+up GEMM (SwiGLU epilogue) and the scatter GEMM with experts whose row
    counts sit on every tile edge: 64 and 128 (an M=64 one-CTA tile, an M=128 pair tile), 256 (a
    full pair tile), one past each, 384 = 256 + an M=128 pair tile, and an empty expert. F = 328
    gives a ragged last N tile, so a half pair tile's second CTA sees only out-of-range columns."""
    monkeypatch.setenv("MOE_GEMM_2SM", cta)
    D, F, E, base = 136, 328, len(EDGE_COUNTS), 3
    owners = np.repeat(np.arange(E, dtype=np.int32), EDGE_COUNTS)
    owners = owners[np.random.default_rng(5).permutation(len(owners))]
    R = len(owners)
    w = W.custom("ep_edges", S=R, D=D, F=F, E=E, k=1,
                 dtype="bf16" if dtype == torch.bfloat16 else "f32")
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    ids = torch.from_numpy(owners + base).cuda()
    y = moe.expert_mlp_forward(inp["x"], ids, base, inp["w_gate_e"], inp["w_up"], inp["w_down"])
    ref = _expert_ref(oracle_lib, inp["x"], ids, base, inp["w_gate_e"], inp["w_up"],
                      inp["w_down"])
    got = y.cpu().numpy()
    assert np.abs(got - ref).max() < MAX_ABS
    assert rel_frob(got, ref) < REL_FROB


def test_expert_mlp_forward_bad_id(moe):
    R, D, F, E = 64, 64, 64, 4
    w = W.custom("ep_bad", S=R, D=D, F=F, E=E, k=1)
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    ids = torch.zeros(R, dtype=torch.int32, device="cuda")
    ids[5] = E  # outside [0, E)
    ws = moe.alloc_workspace(moe.workspace_size("expert_mlp_forward", R, D, F, E, 1,
                                                torch.bfloat16), torch.device("cuda"))
    y = moe.expert_mlp_forward(inp["x"], ids, 0, inp["w_gate_e"], inp["w_up"], inp["w_down"],
                               ws=ws)
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_status(ws)
    assert ei.value.code == -5  # MOE_ERR_BAD_EXPERT_ID
    assert bool((y[5] == 0).all())
    assert bool(torch.isfinite(y).all())


def test_ep_combine(moe):
    S, D, k = 257, 96, 3
    g = torch.Generator().manual_seed(2)
    ret = torch.randn(S * k, D, generator=g)
    perm = torch.randperm(S * k, generator=g).to(torch.int32)
    perm[7] = -1  # a route without a slot
    tw = torch.rand(S, k, generator=g)
    out = moe.ep_combine(ret.cuda(), perm.cuda(), tw.cuda())
    ref = np.zeros((S, D))
    pn, rn, wn = perm.numpy(), ret.numpy().astype(np.float64), tw.numpy().astype(np.float64)
    for i in range(S * k):
        if pn[i] >= 0:
            ref[i // k] += wn.reshape(-1)[i] * rn[pn[i]]
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=1e-5, atol=1e-5)


def _emulated_forward(moe, xs, w_gate, bias, wge, wup, wd, E, k):
    """n ranks' forwards with the all-to-alls done by slicing (what all_to_all_single moves)."""
    n = len(xs)
    el = E // n
    routes, disp, send = [], [], []
    for x in xs:
        te, tw = moe.route_topk(x, w_gate, k, bias)
        d = moe.ep_dispatch(x, te, E)
        off = d["expert_offsets"].cpu().tolist()
        routes.append((te, tw))
        disp.append(d)
        send.append([(off[q * el], off[(q + 1) * el]) for q in range(n)])
    ys = []
    for q in range(n):
        rx = torch.cat([disp[r]["send_x"][a:b] for r in range(n) for (a, b) in [send[r][q]]])
        re = torch.cat([disp[r]["send_e"][a:b] for r in range(n) for (a, b) in [send[r][q]]])
        sl = slice(q * el, (q + 1) * el)
        ys.append(moe.expert_mlp_forward(rx.contiguous(), re.contiguous(), q * el,
                                         wge[sl].contiguous(), wup[sl].contiguous(),
                                         wd[sl].contiguous()))
    outs = []
    for r in range(n):
        parts = []
        for q in range(n):
            start = sum(send[rr][q][1] - send[rr][q][0] for rr in range(r))
            a, b = send[r][q]
            parts.append(ys[q][start:start + (b - a)])
        ret = torch.cat(parts).contiguous()
        te, tw = routes[r]
        outs.append((moe.ep_combine(ret, disp[r]["sparse_rows"], tw), te))
    return outs


@pytest.mark.parametrize("n,E,k,zipf", [(2, 8, 2, 0.0), (4, 16, 4, 1.2), (8, 64, 6, 1.2)])
def test_ep_emulated_ranks(oracle_lib, moe, n, E, k, zipf):
    w = W.custom("ep_emul", S=n * 160, D=256, F=320, E=E, k=k,
                 router_std="1/sqrt(D)" if zipf else "0.02", zipf_s=zipf)
    inp = {nm: (t.cuda() if t is not None else None) for nm, t in W.make_inputs(w).items()}
    sizes = [160 + (17 if r % 2 else -17) for r in range(n)]  # uneven, summing to S
    xs = list(torch.split(inp["x"], sizes))
    xs = [x.contiguous() for x in xs]
    outs = _emulated_forward(moe, xs, inp["w_gate"], inp["logit_bias"], inp["w_gate_e"],
                             inp["w_up"], inp["w_down"], E, k)
    cpu = {nm: (t.float().cpu().numpy() if t is not None else None) for nm, t in inp.items()}
    for r, (out, te) in enumerate(outs):
        ref, _, _ = oracle_lib.mlp_forward(xs[r].float().cpu().numpy(), cpu["w_gate"],
                                           cpu["w_gate_e"], cpu["w_up"], cpu["w_down"], k,
                                           bias=cpu["logit_bias"],
                                           given_top_experts=te.cpu().numpy())
        got = out.cpu().numpy()
        assert np.abs(got - ref).max() < MAX_ABS, r
        assert rel_frob(got, ref) < REL_FROB, r


def test_ep_forward_nccl_one_rank(moe):
    """The real exchange path (torch.distributed over NCCL) with one rank: it must give the
    single-process forward's result."""
    import torch.distributed as dist
    from sparse_mixture_experts_02_b200.expert_parallel import ep_mlp_forward

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = W.custom("ep_one", S=512, D=256, F=384, E=8, k=2)
        inp = {nm: (t.cuda() if t is not None else None) for nm, t in W.make_inputs(w).items()}
        out, te, tw = ep_mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                                     inp["w_down"], w.E, w.k)
        ref = moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"],
                              inp["w_down"], w.k)
        torch.cuda.synchronize()
        assert float((out - ref).abs().max()) < 1e-3
    finally:
        dist.destroy_process_group()
