"""The optional fp32 -> bf16 cast of the forward's output (moe_cast_bf16) against the oracle's
round-to-nearest-even, bit for bit (ScatterMoE guide, "3. Assembling the ScatterMoE FFN Block":
the layer returns the input's dtype)."""
import numpy as np
import pytest
import torch

import moe_workloads as W

pytestmark = pytest.mark.gpu


def test_cast_bits(oracle_lib, moe):
    g = np.random.default_rng(1)
    x = (g.standard_normal(1 << 20) * np.exp2(g.integers(-140, 120, 1 << 20))).astype(np.float32)
    ties = np.array([0x3F808000, 0x3F818000, 0x7F7FFFFF, 0xFF7FFFFF, 0x7F7F7FFF, 0x000116C2,
                     0x80000000, 0x7F800000], dtype=np.uint32).view(np.float32)
    x[: ties.size] = ties
    got = moe.cast_bf16(torch.from_numpy(x).cuda()).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, oracle_lib.to_bf16_bits(x))


def test_cast_forward_output(oracle_lib, moe):
    w = W.custom("cast_fwd", S=300, D=256, F=384, E=8, k=2)
    inp = {n: (t.cuda() if t is not None else None) for n, t in W.make_inputs(w).items()}
    out = moe.mlp_forward(inp["x"], inp["w_gate"], inp["w_gate_e"], inp["w_up"], inp["w_down"],
                          w.k)
    ob = moe.cast_bf16(out)
    assert ob.shape == out.shape and ob.dtype == torch.bfloat16
    got = ob.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, oracle_lib.to_bf16_bits(out.cpu().numpy()))


def test_cast_argument_errors(moe):
    with pytest.raises(moe.MoeError):
        moe.cast_bf16(torch.zeros(12, device="cuda"))  # not a multiple of 8
    assert moe.cast_bf16(torch.zeros(0, device="cuda")).numel() == 0
