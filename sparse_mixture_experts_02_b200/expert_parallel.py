"""Expert-parallel MoE expert-MLP forward over torch.distributed ranks.

The experts are spread over the ranks of a process group: rank r owns experts
[r E/n, (r+1) E/n) and their weights; every rank holds its own tokens and the replicated router
(ScatterMoE guide, "Combine with Tensor and Pipeline Parallelism": expert weights distributed
over expert-parallel groups while ScatterMoE handles the local experts). A forward on every rank:

  1. route its tokens (moe_route_topk);
  2. dispatch: the sparse map and the routed rows in slot order (moe_ep_dispatch). Slots are
     grouped by expert, hence by destination rank;
  3. exchange the per-rank row counts, then the rows and their expert ids (all-to-all);
  4. run the local experts on the received rows (moe_expert_mlp_forward, fp32 outputs);
  5. send the outputs back (all-to-all with the splits reversed), into the send buffer's slots;
  6. combine: out[s] = sum_j w_{s,j} * y[slot of route (s, j)] (moe_ep_combine).

Every step that touches rows runs in the library's CUDA kernels; this module only computes split
sizes and calls torch.distributed (NCCL over NVLink on GPUs). The split sizes need the dispatch's
expert offsets on the host, which is the one host synchronisation of a forward.
"""
from __future__ import annotations

from types import SimpleNamespace
from typing import Optional

import torch
import torch.distributed as dist

from . import ep_combine, ep_dispatch, expert_mlp_forward, route_topk

CUDA_OPS = SimpleNamespace(route=route_topk, dispatch=ep_dispatch, experts=expert_mlp_forward,
                           combine=ep_combine)


def split_sizes(expert_offsets, E: int, n_ranks: int):
    """Rows sent to each rank: the slots of its contiguous expert range (host ints)."""
    off = [int(v) for v in expert_offsets]
    el = E // n_ranks
    return [off[(r + 1) * el] - off[r * el] for r in range(n_ranks)]


STAGES = ("route", "dispatch", "exchange", "experts", "return", "combine")


def ep_mlp_forward(x: torch.Tensor, w_gate: torch.Tensor, w_gate_e: torch.Tensor,
                   w_up: torch.Tensor, w_down: torch.Tensor, E: int, k: int,
                   group=None, logit_bias: Optional[torch.Tensor] = None, ops=None,
                   events=None):
    """Expert-parallel forward of this rank's tokens x [S, D]; w_gate [D, E] replicated;
    w_gate_e / w_up [E/n, D, F] and w_down [E/n, F, D] this rank's experts. Returns
    (out [S, D] float32, top_experts [S, k], top_weights [S, k]). Every rank of `group` must call
    it (the exchanges are collective). `ops` replaces the row kernels (tests only); `events`, 7
    torch.cuda.Event objects, are recorded on the current stream around the STAGES."""
    ops = CUDA_OPS if ops is None else ops

    def mark(i):
        if events is not None:
            events[i].record()

    mark(0)
    n = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if E % n != 0:
        raise ValueError(f"E={E} experts do not split evenly over {n} ranks")
    el = E // n
    if w_gate_e.shape[0] != el or w_up.shape[0] != el or w_down.shape[0] != el:
        raise ValueError(f"each rank holds E/n = {el} experts")
    S, D = x.shape
    dev = x.device
    top_e, top_w = ops.route(x, w_gate, k, logit_bias)
    mark(1)
    d = ops.dispatch(x, top_e, E)
    mark(2)
    off = d["expert_offsets"].to("cpu")
    send = split_sizes(off.tolist(), E, n)
    n_send = int(off[E])
    # counts first, then rows and expert ids
    send_t = torch.tensor(send, dtype=torch.int64, device=dev)
    recv_t = torch.empty_like(send_t)
    dist.all_to_all_single(recv_t, send_t, group=group)
    recv = [int(v) for v in recv_t.to("cpu").tolist()]
    n_recv = sum(recv)
    recv_x = torch.empty((n_recv, D), dtype=x.dtype, device=dev)
    recv_e = torch.empty(n_recv, dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_x, d["send_x"][:n_send], recv, send, group=group)
    dist.all_to_all_single(recv_e, d["send_e"][:n_send], recv, send, group=group)
    mark(3)
    y = ops.experts(recv_x, recv_e, rank * el, w_gate_e, w_up, w_down)
    mark(4)
    # expert outputs back into the slots they were sent from (slots past n_send carry routes
    # with an out-of-range id, which the combine skips)
    ret = torch.empty((S * k, D), dtype=torch.float32, device=dev)
    dist.all_to_all_single(ret[:n_send], y, send, recv, group=group)
    mark(5)
    out = ops.combine(ret, d["sparse_rows"], top_w)
    mark(6)
    return out, top_e, top_w
