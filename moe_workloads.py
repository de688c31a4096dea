"""Seeded synthetic inputs for the dropless MoE expert-MLP forward.

This module only draws random numbers. It holds none of the method's arithmetic (no routing, no
map, no matmul), so both the CPU oracle's tests and the CUDA path's tests and bench can take their
inputs from here without sharing any computation.

Recipe (one generator per workload, seed 0, fixed draw order x, W_gate, W_gate_e, W_up, W_down,
then the popularity permutation when the workload has one):

* every tensor is drawn as float32 standard normals and scaled by its std;
* bf16 workloads round the draws to bfloat16 (round-to-nearest-even) once; fp32 workloads keep them;
* x ~ N(0, 1); expert weights ~ N(0, 0.02^2);
* router W_gate ~ N(0, 0.02^2) ("gaussian router", near-uniform load) or N(0, 1/D) ("logits N(0,1)");
* the skewed workload adds a per-expert logit bias  b[pi(r)] = -s * ln(r + 1)  for popularity rank
  r = 0..E-1, with s = 1.2 and pi a seeded permutation, so that expert popularity follows a
  Zipf(s) mass that is not tied to the expert id.

The shapes follow the Mixtral-8x7B layer (S=4096, D=4096, E=8, top-2) of the ScatterMoE guide's
benchmark ("Benchmark Comparison", table 1), the 128-expert / top-4 GPT-OSS case of the Fast-LLM
scalable sparse-map pull request ("3. GPT-OSS Specific Config") and the Zipf-skew regime named in the
TritonMoE abstract.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    S: int
    D: int
    F: int
    E: int
    k: int
    dtype: str            # "f32" or "bf16"
    router_std: str       # "0.02" or "1/sqrt(D)"
    zipf_s: float = 0.0   # 0 = no popularity bias
    expert_std: float = 0.02

    @property
    def R(self) -> int:
        return self.S * self.k

    def describe(self) -> dict:
        return dataclasses.asdict(self)


WORKLOADS = {
    "tiny": Workload("tiny", S=512, D=256, F=512, E=8, k=2, dtype="f32", router_std="0.02"),
    "mixtral_prefill": Workload("mixtral_prefill", S=4096, D=4096, F=14336, E=8, k=2,
                                dtype="bf16", router_std="0.02"),
    "mixtral_decode": Workload("mixtral_decode", S=128, D=4096, F=14336, E=8, k=2,
                               dtype="bf16", router_std="0.02"),
    "e128": Workload("e128", S=8192, D=2880, F=2880, E=128, k=4, dtype="bf16",
                     router_std="1/sqrt(D)"),
    "zipf64": Workload("zipf64", S=16384, D=2048, F=1408, E=64, k=6, dtype="bf16",
                       router_std="1/sqrt(D)", zipf_s=1.2),
}

# A smaller prefill-shaped case for detailed profiler captures (1.4 GB of weights, 4 M tiles per
# expert): same kernels and regime as the Mixtral prefill layer, a fraction of its size.
PROFILE_WORKLOADS = {
    "prefill_profile": Workload("prefill_profile", S=2048, D=4096, F=7168, E=8, k=2,
                                dtype="bf16", router_std="0.02"),
    # the 128-expert layer's tiles (about 256 rows per expert, D = F = 2880, one-CTA GEMMs) with
    # a quarter of its experts and tokens: 1.6 GB of weights
    "e128_profile": Workload("e128_profile", S=2048, D=2880, F=2880, E=32, k=4, dtype="bf16",
                             router_std="1/sqrt(D)"),
    # the routers and sparse maps of the Mixtral prefill and the 128-expert layers (same S, D, E,
    # k, so the same kernels and launch shapes) with a small F: 50 MB and 566 MB of weights
    "router_e8_profile": Workload("router_e8_profile", S=4096, D=4096, F=256, E=8, k=2,
                                  dtype="bf16", router_std="0.02"),
    "router_e128_profile": Workload("router_e128_profile", S=8192, D=2880, F=256, E=128, k=4,
                                    dtype="bf16", router_std="1/sqrt(D)"),
}


def custom(name, S, D, F, E, k, dtype="bf16", router_std="0.02", zipf_s=0.0) -> Workload:
    return Workload(name, S=S, D=D, F=F, E=E, k=k, dtype=dtype, router_std=router_std,
                    zipf_s=zipf_s)


def _torch_dtype(w: Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def _draw(gen, shape, std, dtype, device, chunk_dim0=True):
    """N(0, std^2) float32 draws rounded once to `dtype`; drawn slab by slab along dim 0 so that a
    multi-GB weight never needs a float32 copy of the whole tensor."""
    out = torch.empty(shape, dtype=dtype, device=device)
    if len(shape) == 3 and chunk_dim0:
        for e in range(shape[0]):
            t = torch.randn(shape[1:], generator=gen, dtype=torch.float32, device=device)
            out[e].copy_(t.mul_(std))
            del t
    else:
        t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
        out.copy_(t.mul_(std))
    return out


def make_inputs(w: Workload, device="cpu", seed: int = 0) -> dict:
    """Returns a dict with x [S,D], w_gate [D,E], w_gate_e [E,D,F], w_up [E,D,F], w_down [E,F,D]
    (all in the workload's dtype) and logit_bias [E] float32 or None."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = _torch_dtype(w)
    rstd = 0.02 if w.router_std == "0.02" else 1.0 / math.sqrt(w.D)
    x = _draw(gen, (w.S, w.D), 1.0, dt, device)
    w_gate = _draw(gen, (w.D, w.E), rstd, dt, device)
    w_gate_e = _draw(gen, (w.E, w.D, w.F), w.expert_std, dt, device)
    w_up = _draw(gen, (w.E, w.D, w.F), w.expert_std, dt, device)
    w_down = _draw(gen, (w.E, w.F, w.D), w.expert_std, dt, device)
    bias: Optional[torch.Tensor] = None
    if w.zipf_s > 0:
        perm = torch.randperm(w.E, generator=gen, device=device)
        ranks = torch.arange(w.E, dtype=torch.float64)
        vals = (-w.zipf_s * torch.log(ranks + 1.0)).to(torch.float32).to(device)
        bias = torch.empty(w.E, dtype=torch.float32, device=device)
        bias[perm] = vals
    return dict(x=x, w_gate=w_gate, w_gate_e=w_gate_e, w_up=w_up, w_down=w_down, logit_bias=bias)


@dataclasses.dataclass(frozen=True)
class MoaWorkload:
    """A Mixture-of-Attention layer: E attention experts with H heads of dh columns each (own
    query and output projections), keys and values shared, one causal sequence of S tokens."""
    name: str
    S: int
    D: int
    H: int
    dh: int
    E: int
    k: int
    router_std: str = "0.02"
    zipf_s: float = 0.0
    weight_std: float = 0.02

    @property
    def R(self) -> int:
        return self.S * self.k

    @property
    def HD(self) -> int:
        return self.H * self.dh

    def describe(self) -> dict:
        return dataclasses.asdict(self)


# The MoA layer at the Mixtral-8x7B prefill shape: 8 attention experts of 8 heads x 128 (each
# token's k = 2 experts give 16 query heads, half of a 32-head dense layer), one 4096-token sequence.
MOA_WORKLOADS = {
    "moa_prefill": MoaWorkload("moa_prefill", S=4096, D=4096, H=8, dh=128, E=8, k=2),
}


def make_moa_inputs(w: MoaWorkload, device="cpu", seed: int = 0) -> dict:
    """bf16 x [S,D] ~ N(0,1), w_gate [D,E], w_q [E,D,HD], w_kv [D,2HD] (key columns first),
    w_o [E,HD,D] ~ N(0, weight_std^2); router std as for the MLP workloads; logit_bias [E] float32
    (Zipf popularity, as for the MLP workloads) or None. Draw order x, w_gate, w_q, w_kv, w_o,
    then the popularity permutation."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = torch.bfloat16
    rstd = 0.02 if w.router_std == "0.02" else 1.0 / math.sqrt(w.D)
    x = _draw(gen, (w.S, w.D), 1.0, dt, device)
    w_gate = _draw(gen, (w.D, w.E), rstd, dt, device)
    w_q = _draw(gen, (w.E, w.D, w.HD), w.weight_std, dt, device)
    w_kv = _draw(gen, (w.D, 2 * w.HD), w.weight_std, dt, device)
    w_o = _draw(gen, (w.E, w.HD, w.D), w.weight_std, dt, device)
    bias: Optional[torch.Tensor] = None
    if w.zipf_s > 0:
        perm = torch.randperm(w.E, generator=gen, device=device)
        ranks = torch.arange(w.E, dtype=torch.float64)
        vals = (-w.zipf_s * torch.log(ranks + 1.0)).to(torch.float32).to(device)
        bias = torch.empty(w.E, dtype=torch.float32, device=device)
        bias[perm] = vals
    return dict(x=x, w_gate=w_gate, w_q=w_q, w_kv=w_kv, w_o=w_o, logit_bias=bias)


def make_top_experts(S: int, k: int, E: int, seed: int = 0, mode: str = "uniform",
                     device="cpu") -> torch.Tensor:
    """Seeded routing tables [S,k] int32 for the sparse-map tests, without any router.

    mode "uniform": each row holds k distinct experts drawn uniformly (a random permutation prefix).
    mode "zipf":    distinct experts drawn by Zipf(1.2) popularity (Gumbel top-k of log-masses).
    mode "one":     every route of every row is expert 0 (rows are then not distinct: a stress case).
    mode "any":     k independent uniform draws (repeats allowed inside a row).
    mode "stride":  row s holds (b_s + j*c_s) mod E for j < k, with b_s uniform and c_s uniform among
                    the residues coprime to E: k distinct experts, uniform marginals, drawn on
                    `device` without an S x E key matrix (for route counts up to 2^26).
    """
    if mode == "stride":
        g2 = torch.Generator(device=device)
        g2.manual_seed(seed)
        units = torch.tensor([c for c in range(1, E) if math.gcd(c, E) == 1] or [1],
                             dtype=torch.int64, device=device)
        b = torch.randint(0, E, (S, 1), generator=g2, device=device)
        c = units[torch.randint(0, units.numel(), (S, 1), generator=g2, device=device)]
        j = torch.arange(k, dtype=torch.int64, device=device)[None, :]
        return ((b + j * c) % E).to(torch.int32).contiguous()
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    if mode == "one":
        t = torch.zeros((S, k), dtype=torch.int32)
    elif mode == "any":
        t = torch.randint(0, E, (S, k), generator=gen, dtype=torch.int64).to(torch.int32)
    elif mode in ("uniform", "zipf"):
        keys = torch.rand((S, E), generator=gen, dtype=torch.float64)
        g = -torch.log(-torch.log(keys.clamp_min(1e-300)))
        if mode == "zipf":
            g = g + (-1.2 * torch.log(torch.arange(E, dtype=torch.float64) + 1.0))[None, :]
        t = torch.topk(g, k, dim=1).indices.to(torch.int32)
    else:
        raise ValueError(mode)
    return t.contiguous().to(device)
