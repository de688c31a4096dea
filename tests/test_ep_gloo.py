"""Expert-parallel forward, host side: the exchange bookkeeping of `expert_parallel.ep_mlp_forward`
on 2 and 4 gloo ranks on the CPU (ScatterMoE guide, "Combine with Tensor and Pipeline
Parallelism").

The row kernels are replaced by oracle-based CPU stand-ins:
  * the routing comes from the oracle router;
  * the dispatch from the oracle's sparse map plus a row gather;
  * the experts from the oracle's hidden rows times W_down;
  * the combine from a weighted sum.
So this test checks what the host code decides: split sizes from the expert offsets, the count
exchange, the row / id / result all-to-alls and the expert base of each rank. Every rank's
output must equal the oracle's single-process forward of its tokens with all E experts. The CUDA
kernels themselves are covered by tests/test_gpu_ep.py.
"""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops(oracle):
    def route(x, w_gate, k, bias):
        logits, _ = oracle.router_logits(x.numpy(), w_gate.numpy(),
                                         None if bias is None else bias.numpy())
        te, tw = oracle.topk_softmax(logits, k)
        return torch.from_numpy(te), torch.from_numpy(tw.astype(np.float32))

    def dispatch(x, te, E):
        k = te.shape[1]
        counts, offsets, sparse, srt = oracle.sparse_map(te.numpy(), E)
        idx = torch.from_numpy(srt.astype(np.int64))
        return {"send_x": x[idx // k].contiguous(), "send_e": te.reshape(-1)[idx].contiguous(),
                "expert_counts": torch.from_numpy(counts),
                "expert_offsets": torch.from_numpy(offsets),
                "sparse_rows": torch.from_numpy(sparse), "sorted_rows": torch.from_numpy(srt)}

    def experts(xr, ids, base, wge, wup, wd):
        R, D = xr.shape
        y = np.zeros((R, D))
        xn, wgn, wun, wdn = xr.numpy(), wge.numpy(), wup.numpy(), wd.numpy().astype(np.float64)
        for i in range(R):
            e = int(ids[i]) - base
            assert 0 <= e < wge.shape[0], (e, base)
            y[i] = oracle.expert_hidden(xn, wgn, wun, i, e) @ wdn[e]
        return torch.from_numpy(y.astype(np.float32))

    def combine(ret, sparse, tw):
        S, k = tw.shape
        out = torch.zeros((S, ret.shape[1]), dtype=torch.float64)
        for i in range(S * k):
            p = int(sparse[i])
            if p >= 0:
                out[i // k] += float(tw.reshape(-1)[i]) * ret[p].double()
        return out

    return SimpleNamespace(route=route, dispatch=dispatch, experts=experts, combine=combine)


def _weights(E, D, F, skew):
    g = torch.Generator().manual_seed(7)
    w_gate = torch.randn(D, E, generator=g) / D ** 0.5
    wge = torch.randn(E, D, F, generator=g) * 0.1
    wup = torch.randn(E, D, F, generator=g) * 0.1
    wd = torch.randn(E, F, D, generator=g) * 0.1
    bias = None
    if skew:  # the first half of the experts are never chosen: some ranks receive no rows
        bias = torch.zeros(E)
        bias[: E // 2] = -1e4
    return w_gate, wge, wup, wd, bias


def _rank(rank, n, port, E, k, S, D, F, skew):
    import oracle
    from sparse_mixture_experts_02_b200.expert_parallel import ep_mlp_forward

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=n)
    try:
        w_gate, wge, wup, wd, bias = _weights(E, D, F, skew)
        el = E // n
        x = torch.randn(S + 3 * rank, D, generator=torch.Generator().manual_seed(100 + rank))
        out, te, tw = ep_mlp_forward(x, w_gate, wge[rank * el:(rank + 1) * el].contiguous(),
                                     wup[rank * el:(rank + 1) * el].contiguous(),
                                     wd[rank * el:(rank + 1) * el].contiguous(), E, k,
                                     logit_bias=bias, ops=_oracle_ops(oracle))
        ref, ote, _ = oracle.mlp_forward(x.numpy(), w_gate.numpy(), wge.numpy(), wup.numpy(),
                                         wd.numpy(), k, bias=None if bias is None else bias.numpy(),
                                         given_top_experts=te.numpy())
        err = np.abs(out.numpy() - ref).max() / max(np.abs(ref).max(), 1e-30)
        assert err < 1e-5, (rank, err)
        if skew:
            assert (te.numpy() >= E // 2).all()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,E,k,skew", [(2, 8, 2, False), (4, 8, 3, False), (2, 8, 2, True),
                                        (4, 16, 4, True)])
def test_ep_forward_matches_single_process(n, E, k, skew):
    mp.start_processes(_rank, args=(n, _free_port(), E, k, 24, 16, 24, skew), nprocs=n,
                       start_method="spawn")


def test_split_sizes():
    from sparse_mixture_experts_02_b200.expert_parallel import split_sizes
    off = [0, 3, 3, 7, 10, 10, 10, 12, 15]  # E = 8
    assert split_sizes(off, 8, 2) == [10, 5]
    assert split_sizes(off, 8, 4) == [3, 7, 0, 5]
    assert split_sizes(off, 8, 1) == [15]
