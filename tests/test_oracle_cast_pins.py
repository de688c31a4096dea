"""Pins of the oracle's float32 -> bfloat16 rounding (the optional cast of the forward's output;
ScatterMoE guide, "3. Assembling the ScatterMoE FFN Block": the layer returns the input's dtype).

Hand-worked bit patterns (round to nearest, ties to even, overflow to infinity), and agreement with
torch's CPU conversion on random values of every magnitude.
"""
import numpy as np
import torch


def _bits(v):
    return np.array([v], dtype=np.uint32).view(np.float32)


def test_hand_worked_patterns(oracle_lib):
    cases = [
        (0x3F800000, 0x3F80),  # 1.0
        (0x3F808000, 0x3F80),  # 1 + 2^-8: a tie, the kept part is even -> down
        (0x3F818000, 0x3F82),  # 1 + 3*2^-8: a tie, the kept part is odd -> up
        (0x3F808001, 0x3F81),  # just above the tie -> up
        (0x3F807FFF, 0x3F80),  # just below the tie -> down
        (0xC0200000, 0xC020),  # -2.5
        (0x7F7FFFFF, 0x7F80),  # the largest float rounds to +inf
        (0xFF7FFFFF, 0xFF80),  # ... and its negative to -inf
        (0x7F7F7FFF, 0x7F7F),  # below the tie at the top: the largest finite bf16
        (0x00000000, 0x0000),
        (0x80000000, 0x8000),  # -0
        (0x000116C2, 0x0001),  # a subnormal rounds like any other pattern
        (0x7F800000, 0x7F80),  # +inf stays
    ]
    for src, want in cases:
        got = int(oracle_lib.to_bf16_bits(_bits(src))[0])
        assert got == want, (hex(src), hex(got), hex(want))
    nan = oracle_lib.to_bf16_bits(np.array([np.nan, -np.nan], dtype=np.float32))
    assert (nan & 0x7FFF).tolist() == [0x7FC0, 0x7FC0]


def test_matches_torch_rounding(oracle_lib):
    g = np.random.default_rng(0)
    x = (g.standard_normal(200000) * np.exp2(g.integers(-140, 120, 200000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_lib.to_bf16_bits(x), want)
