"""Device-side error reporting without faulting the GPU: a bounded wait that nothing satisfies
returns MOE_ERR_DEVICE_TIMEOUT through the status word and leaves the context usable; a bad
expert id is reported (see test_gpu_map); argument errors never reach the device."""
import pytest
import torch

import moe_workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(moe):
    ws = moe.alloc_workspace(256, torch.device("cuda"))
    moe.debug_wait_timeout(2_000_000, ws)  # 2 ms limit on a barrier nobody arrives at
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_status(ws)
    assert ei.value.code == -6
    # the context still works: a normal forward runs and the status is clean
    w = W.custom("after", S=64, D=64, F=64, E=4, k=2)
    inp = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w).items()}
    wsf = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, torch.bfloat16, torch.device("cuda"))
    out = moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"],
                          w.k, ws=wsf)
    moe.check_device_status(wsf)
    assert torch.isfinite(out).all()


def test_python_argument_errors(moe):
    x = torch.zeros(8, 60, dtype=torch.bfloat16, device="cuda")  # D not a multiple of 8
    wg = torch.zeros(60, 4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.route_topk(x, wg, 2)
    assert ei.value.code == -1
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.route_topk(x, wg, 5)  # k > E
    with pytest.raises(TypeError):
        moe.route_topk(x.half(), wg.half(), 2)


def test_launch_counts(moe):
    w = W.custom("cnt", S=100, D=64, F=64, E=4, k=2)
    inp = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w).items()}
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k)
    # route, one-block map (S*k <= 16384 routes), GEMM1 (also zeroes out), GEMM2
    assert moe.last_launch_count() == 4
    w = W.custom("cnt2", S=9000, D=64, F=64, E=4, k=2)
    inp = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w).items()}
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k)
    # route, map count / scan / assign, GEMM1, GEMM2
    assert moe.last_launch_count() == 6


@pytest.mark.parametrize("S,E", [(100, 4), (3000, 64), (600, 96)])
def test_forward_clears_a_stale_status(moe, S, E):
    # the forward's first kernel (whichever router runs) clears the status word in the workspace
    w = W.custom("stale", S=S, D=64, F=64, E=E, k=2, router_std="1/sqrt(D)")
    inp = {k: (v.cuda() if v is not None else None) for k, v in W.make_inputs(w).items()}
    wsf = moe.ForwardWorkspace(w.S, w.D, w.F, w.E, w.k, torch.bfloat16, torch.device("cuda"))
    wsf.buf[:4].view(torch.int32).fill_(2)  # a timeout flag left over from an earlier call
    moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"], w.k,
                    ws=wsf)
    moe.check_device_status(wsf)
