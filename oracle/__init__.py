"""ctypes binding of the CPU oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the package entry's smoke check and the bench's CPU baseline
leg are the only callers. The CUDA product path never imports this package, and this package never
imports the product. Inputs are numpy arrays (float32 for tensors that are bf16 or fp32 on the GPU:
bf16 values are exact in float32); results come back as float64 / int32 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_OUT = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_OUT) or os.path.getmtime(_OUT) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_OUT), exist_ok=True)
        tmp = _OUT + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _OUT)
    return _OUT


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_router_logits.argtypes = [P, P, P, i64, i32, P, i64, P, P]
        L.oracle_topk_softmax.argtypes = [P, i64, i32, i32, P, P]
        L.oracle_weights_for.argtypes = [P, P, i64, i32, i32, P]
        L.oracle_sparse_map.argtypes = [P, i64, i32, P, P, P, P]
        L.oracle_sparse_map.restype = ctypes.c_int
        L.oracle_expert_hidden.argtypes = [P, P, P, i64, i64, i32, i32, P]
        L.oracle_expert_hidden_rows.argtypes = [P, P, P, i64, i64, P, P, i64, P]
        L.oracle_mlp_forward.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, P, i64, P, P, P, P]
        L.oracle_scatter_linear.argtypes = [P, P, i64, i64, i64, i32, i32, P, P, P, ctypes.c_int,
                                            ctypes.c_int, P]
        L.oracle_scatter_linear_backward.argtypes = [P, P, P, i64, i64, i64, i32, i32, P, P, P,
                                                     ctypes.c_int, ctypes.c_int, P, P, P]
        L.oracle_mlp_backward.argtypes = [P, P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P,
                                          P, P, P]
        L.oracle_moa_forward.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i32, i32, P, P,
                                         P, P]
        L.oracle_moa_forward_tokens.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i32, i32,
                                                P, P, i64, P, P, P]
    return _lib


def _f32(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().oracle_num_threads()


def router_logits(x, w_gate, bias=None, tokens=None):
    """fp64 logits [n, E] and magnitude sums sum_d |x_d W[d,e]| [n, E] for the listed tokens."""
    x, w_gate, bias = _f32(x), _f32(w_gate), _f32(bias)
    S, D = x.shape
    E = w_gate.shape[1]
    tokens = np.arange(S, dtype=np.int32) if tokens is None else _i32(tokens)
    n = tokens.shape[0]
    logits = np.zeros((n, E), dtype=np.float64)
    absdot = np.zeros((n, E), dtype=np.float64)
    lib().oracle_router_logits(_p(x), _p(w_gate), _p(bias), D, E, _p(tokens), n, _p(logits),
                               _p(absdot))
    return logits, absdot


def topk_softmax(logits, k):
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    n, E = logits.shape
    te = np.zeros((n, k), dtype=np.int32)
    tw = np.zeros((n, k), dtype=np.float64)
    lib().oracle_topk_softmax(_p(logits), n, E, k, _p(te), _p(tw))
    return te, tw


def weights_for(logits, top_experts):
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    te = _i32(top_experts)
    n, E = logits.shape
    k = te.shape[1]
    tw = np.zeros((n, k), dtype=np.float64)
    lib().oracle_weights_for(_p(logits), _p(te), n, E, k, _p(tw))
    return tw


def route(x, w_gate, k, bias=None):
    logits, _ = router_logits(x, w_gate, bias)
    return topk_softmax(logits, k)


def sparse_map(top_experts, E):
    """Returns (counts [E], offsets [E+1], sparse_rows [R], sorted_rows [R]) or raises ValueError
    on an expert id outside [0, E)."""
    te = _i32(top_experts).reshape(-1)
    R = te.shape[0]
    counts = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    sparse_rows = np.zeros(R, dtype=np.int32)
    sorted_rows = np.zeros(R, dtype=np.int32)
    rc = lib().oracle_sparse_map(_p(te), R, E, _p(counts), _p(offsets), _p(sparse_rows),
                                 _p(sorted_rows))
    if rc != 0:
        raise ValueError("expert id outside [0, E)")
    return counts, offsets, sparse_rows, sorted_rows


def expert_hidden(x, w_gate_e, w_up, token, expert):
    x, wge, wu = _f32(x), _f32(w_gate_e), _f32(w_up)
    D = x.shape[1]
    F = wge.shape[2]
    h = np.zeros(F, dtype=np.float64)
    lib().oracle_expert_hidden(_p(x), _p(wge), _p(wu), D, F, int(token), int(expert), _p(h))
    return h


def expert_hidden_rows(x, w_gate_e, w_up, tokens, experts):
    """expert_hidden for n (token, expert) pairs at once (rows in parallel): h [n, F]."""
    x, wge, wu = _f32(x), _f32(w_gate_e), _f32(w_up)
    tokens, experts = _i32(tokens).reshape(-1), _i32(experts).reshape(-1)
    assert tokens.shape == experts.shape
    D = x.shape[1]
    F = wge.shape[2]
    h = np.zeros((tokens.shape[0], F), dtype=np.float64)
    lib().oracle_expert_hidden_rows(_p(x), _p(wge), _p(wu), D, F, _p(tokens), _p(experts),
                                    tokens.shape[0], _p(h))
    return h


def mlp_forward(x, w_gate, w_gate_e, w_up, w_down, k, bias=None, tokens=None,
                given_top_experts=None):
    """fp64 y [n, D] for the listed tokens (all tokens by default), plus the oracle's (or the
    given) top experts [n, k] and weights [n, k]."""
    x, w_gate, bias = _f32(x), _f32(w_gate), _f32(bias)
    wge, wu, wd = _f32(w_gate_e), _f32(w_up), _f32(w_down)
    S, D = x.shape
    E = w_gate.shape[1]
    F = wge.shape[2]
    tokens = np.arange(S, dtype=np.int32) if tokens is None else _i32(tokens)
    given = _i32(given_top_experts)
    n = tokens.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    te = np.zeros((n, k), dtype=np.int32)
    tw = np.zeros((n, k), dtype=np.float64)
    lib().oracle_mlp_forward(_p(x), _p(w_gate), _p(bias), _p(wge), _p(wu), _p(wd), D, F, E, k,
                             _p(tokens), n, _p(given), _p(out), _p(te), _p(tw))
    return out, te, tw


def scatter_linear(X, W, k, sorted_rows, offsets, gates=None, gather_in=True, scatter_out=True,
                   S=None):
    """ParallelLinear(X, W, I, G) in fp64: grouped rows [R, Dout] or the token-order sum [S, Dout]."""
    X, W, gates = _f32(X), _f32(W), _f32(gates)
    sorted_rows, offsets = _i32(sorted_rows), _i32(offsets)
    E, Din, Dout = W.shape
    if S is None:
        S = X.shape[0] if gather_in else (sorted_rows.shape[0] // k)
    P = int(offsets[E])
    rows = S if scatter_out else max(P, 0)
    Y = np.zeros((rows, Dout), dtype=np.float64)
    lib().oracle_scatter_linear(_p(X), _p(W), S, Din, Dout, E, k, _p(sorted_rows), _p(offsets),
                                _p(gates.reshape(-1) if gates is not None else None),
                                int(bool(gather_in)), int(bool(scatter_out)), _p(Y))
    return Y


def scatter_linear_backward(X, W, dY, k, sorted_rows, offsets, gates=None, gather_in=True,
                            scatter_out=True, S=None):
    """Backward of ParallelLinear in fp64: {"dX", "dW", "dgates"} (dgates only with gates).
    dY has Y's shape: [S, Dout] when scatter_out, else [R, Dout]; dX has X's shape."""
    X, W, dY, gates = _f32(X), _f32(W), _f32(dY), _f32(gates)
    sorted_rows, offsets = _i32(sorted_rows), _i32(offsets)
    E, Din, Dout = W.shape
    if S is None:
        S = X.shape[0] if gather_in else (sorted_rows.shape[0] // k)
    P = int(offsets[E])
    dX = np.zeros((S if gather_in else max(P, 0), Din), dtype=np.float64)
    dW = np.zeros((E, Din, Dout), dtype=np.float64)
    dg = np.zeros(S * k, dtype=np.float64) if gates is not None else None
    lib().oracle_scatter_linear_backward(
        _p(X), _p(W), _p(dY), S, Din, Dout, E, k, _p(sorted_rows), _p(offsets),
        _p(gates.reshape(-1) if gates is not None else None), int(bool(gather_in)),
        int(bool(scatter_out)), _p(dX), _p(dW), _p(dg))
    out = {"dX": dX, "dW": dW}
    if dg is not None:
        out["dgates"] = dg
    return out


def mlp_backward(x, w_gate, w_gate_e, w_up, w_down, dout, k, bias=None, given_top_experts=None,
                 want=("dx", "dw_gate", "dw_gate_e", "dw_up", "dw_down")):
    """Backward of mlp_forward over all tokens in fp64, given dout [S, D]: a dict with the
    requested ones of "dx", "dw_gate", "dw_gate_e", "dw_up", "dw_down" (dx is always computed).
    given_top_experts [S, k] fixes the routing. Without weight gradients the tokens run in
    parallel (dx of a token depends on that token alone)."""
    x, wg, wge, wu, wd = _f32(x), _f32(w_gate), _f32(w_gate_e), _f32(w_up), _f32(w_down)
    dout, bias = _f32(dout), _f32(bias)
    S, D = x.shape
    E, _, F = wge.shape
    given = _i32(given_top_experts) if given_top_experts is not None else None
    shapes = {"dx": (S, D), "dw_gate": (D, E), "dw_gate_e": (E, D, F), "dw_up": (E, D, F),
              "dw_down": (E, F, D)}
    out = {n: np.zeros(sh) for n, sh in shapes.items() if n == "dx" or n in want}
    lib().oracle_mlp_backward(_p(x), _p(wg), _p(bias), _p(wge), _p(wu), _p(wd), _p(dout), S, D,
                              F, E, k, _p(given), _p(out["dx"]), _p(out.get("dw_gate")),
                              _p(out.get("dw_gate_e")), _p(out.get("dw_up")),
                              _p(out.get("dw_down")))
    return out


def moa_forward(x, w_gate, w_q, w_k, w_v, w_o, k, heads, bias=None, given_top_experts=None,
                tokens=None):
    """Mixture of Attention forward in fp64: (out [S, D], top_experts [S, k], top_weights [S, k]).
    w_q [E, D, H*dh], w_k and w_v [D, H*dh], w_o [E, H*dh, D]; causal attention per head. With
    `tokens`, only those query tokens (rows of the results in list order; keys and values of every
    token up to the largest listed one)."""
    x, wg, wq, wk, wv, wo = (_f32(a) for a in (x, w_gate, w_q, w_k, w_v, w_o))
    bias = _f32(bias)
    S, D = x.shape
    E, _, HD = wq.shape
    dh = HD // heads
    given = _i32(given_top_experts) if given_top_experts is not None else None
    if tokens is not None:
        tok = _i32(tokens).reshape(-1)
        n = tok.shape[0]
        out = np.zeros((n, D))
        te = np.zeros((n, k), dtype=np.int32)
        tw = np.zeros((n, k))
        lib().oracle_moa_forward_tokens(_p(x), _p(wg), _p(bias), _p(wq), _p(wk), _p(wv), _p(wo),
                                        S, D, heads, dh, E, k, _p(given), _p(tok), n, _p(out),
                                        _p(te), _p(tw))
        return out, te, tw
    out = np.zeros((S, D))
    te = np.zeros((S, k), dtype=np.int32)
    tw = np.zeros((S, k))
    lib().oracle_moa_forward(_p(x), _p(wg), _p(bias), _p(wq), _p(wk), _p(wv), _p(wo), S, D, heads,
                             dh, E, k, _p(given), _p(out), _p(te), _p(tw))
    return out, te, tw


def to_bf16_bits(x):
    """The optional last step of the forward: float32 -> bfloat16 with round-to-nearest-even
    (ScatterMoE guide, "3. Assembling the ScatterMoE FFN Block": the layer returns the input's
    dtype). Plain definition on the bit pattern: keep the top 16 bits after adding half an ulp of
    the kept part minus one, plus the kept part's lowest bit (ties go to the even pattern);
    overflow carries into the exponent and yields infinity. NaN becomes the quiet NaN 0x7FC0 (sign
    kept). Returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    nan = np.isnan(np.ascontiguousarray(x, dtype=np.float32))
    qnan = ((u >> 16) & 0x8000) | 0x7FC0
    return np.where(nan, qnan, rounded).astype(np.uint16)
