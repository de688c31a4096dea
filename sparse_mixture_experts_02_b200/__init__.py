"""Python binding of the B200 dropless sparse-MoE expert-MLP library (libmoe_b200.so).

This module only marshals arguments: it checks tensor shapes, dtypes and devices, allocates the
outputs and the workspace with torch (device memory and streams are torch's), and calls the C ABI
declared in include/moe.h on the current CUDA stream. Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback. The compiled library is loaded on
first use (so that the build module can be imported before it exists); if it is missing, that
first use raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_b200.so")
# the same library built with MOE_DEBUG=1: device bounds checks on every index read from inputs
DEBUG_LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_b200_debug.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED",
                -3: "MOE_ERR_WORKSPACE", -4: "MOE_ERR_CUDA", -5: "MOE_ERR_BAD_EXPERT_ID",
                -6: "MOE_ERR_DEVICE_TIMEOUT", -7: "MOE_ERR_BAD_INDEX"}

EXPORTS = ["moe_route_topk", "moe_sparse_map", "moe_sparse_map_noalloc", "moe_scatter_linear",
           "moe_scatter_linear_backward", "moe_mlp_forward", "moe_mlp_backward",
           "moe_moa_forward", "moe_ep_dispatch", "moe_expert_mlp_forward", "moe_ep_combine",
           "moe_cast_bf16", "moe_workspace_size", "moe_workspace_view", "moe_last_error",
           "moe_check_device_status", "moe_profile_events", "moe_debug_wait_timeout",
           "moe_last_launch_count", "moe_debug_build"]


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def _load(path: str = None):
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m sparse_mixture_experts_02_b200.build`"
            " (the library has no fallback path)")
    lib = ctypes.CDLL(path)
    P, i64, i32, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    lib.moe_route_topk.argtypes = [P, P, P, i64, i64, i32, i32, c_int, P, P, P]
    lib.moe_sparse_map.argtypes = [P, i64, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_sparse_map_noalloc.argtypes = [P, i64, i32, i32, P, P, P, P, P]
    lib.moe_scatter_linear.argtypes = [P, P, i64, i64, i64, i32, i32, P, P, P, c_int, c_int,
                                       c_int, P, P, ctypes.c_size_t, P]
    lib.moe_scatter_linear_backward.argtypes = [P, P, P, i64, i64, i64, i32, i32, P, P, P, c_int,
                                                c_int, c_int, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_mlp_forward.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, c_int, P, P,
                                    ctypes.c_size_t, P]
    lib.moe_moa_forward.argtypes = [P, P, P, P, P, P, i64, i64, i32, i32, i32, i32, c_int, P, P,
                                    ctypes.c_size_t, P]
    lib.moe_ep_dispatch.argtypes = [P, P, i64, i64, i32, i32, c_int, P, P, P, P, P, P, P,
                                    ctypes.c_size_t, P]
    lib.moe_expert_mlp_forward.argtypes = [P, P, i32, i64, i64, i64, i32, P, P, P, c_int, P, P,
                                           ctypes.c_size_t, P]
    lib.moe_ep_combine.argtypes = [P, P, P, i64, i64, i32, P, P]
    lib.moe_cast_bf16.argtypes = [P, i64, P, P]
    lib.moe_mlp_backward.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, c_int, P,
                                     ctypes.c_size_t, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_workspace_size.argtypes = [ctypes.c_char_p, i64, i64, i64, i32, i32, c_int]
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_workspace_view.argtypes = [ctypes.c_char_p, i64, i64, i64, i32, i32, c_int]
    lib.moe_workspace_view.restype = ctypes.c_int64
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_check_device_status.argtypes = [P, P]
    lib.moe_profile_events.argtypes = [P, c_int]
    lib.moe_debug_wait_timeout.argtypes = [i64, P, ctypes.c_size_t, P]
    for name in ("moe_route_topk", "moe_sparse_map", "moe_sparse_map_noalloc",
                 "moe_scatter_linear", "moe_scatter_linear_backward", "moe_mlp_forward",
                 "moe_mlp_backward", "moe_moa_forward", "moe_ep_dispatch",
                 "moe_expert_mlp_forward", "moe_ep_combine", "moe_cast_bf16",
                 "moe_check_device_status", "moe_profile_events", "moe_debug_wait_timeout",
                 "moe_last_launch_count", "moe_debug_build"):
        getattr(lib, name).restype = c_int
    return lib


def debug_lib():
    """The debug build (libmoe_b200_debug.so) as a separate ctypes handle with the same entry
    points: every index its kernels read from their inputs is bounds-checked on the device, and
    one outside its range is skipped and reported as MOE_ERR_BAD_INDEX by
    moe_check_device_status. The module's own calls keep using the release build."""
    return _load(DEBUG_LIB_PATH)


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def _check(rc: int):
    if rc != 0:
        raise MoeError(rc, _lib().moe_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or float32)")


def _req(t, name, dtype=None, dim=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def workspace_size(op: str, S: int, D: int, F: int, E: int, k: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (MOE_BF16 if dtype == torch.bfloat16 else MOE_F32)
    return int(_lib().moe_workspace_size(op.encode(), S, D, F, E, k, code))


def workspace_view(which: str, S: int, D: int, F: int, E: int, k: int, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (MOE_BF16 if dtype == torch.bfloat16 else MOE_F32)
    return int(_lib().moe_workspace_view(which.encode(), S, D, F, E, k, code))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def route_topk(x: torch.Tensor, w_gate: torch.Tensor, k: int,
               logit_bias: Optional[torch.Tensor] = None):
    """Top-k experts [S,k] int32 and softmax weights [S,k] float32 (moe_route_topk)."""
    _req(x, "x", dim=2)
    _req(w_gate, "w_gate", dtype=x.dtype, dim=2, device=x.device)
    S, D = x.shape
    E = w_gate.shape[1]
    if w_gate.shape[0] != D:
        raise ValueError("w_gate must be [D, E]")
    if logit_bias is not None:
        _req(logit_bias, "logit_bias", dtype=torch.float32, dim=1, device=x.device)
    te = torch.empty((S, k), dtype=torch.int32, device=x.device)
    tw = torch.empty((S, k), dtype=torch.float32, device=x.device)
    _check(_lib().moe_route_topk(_ptr(x), _ptr(w_gate), _ptr(logit_bias), S, D, E, k,
                              _dtype_code(x), _ptr(te), _ptr(tw), _stream(x.device)))
    return te, tw


def sparse_map(top_experts: torch.Tensor, E: int, ws: Optional[torch.Tensor] = None):
    """(counts [E], offsets [E+1], sparse_rows [S*k], sorted_rows [S*k]) int32 (moe_sparse_map)."""
    _req(top_experts, "top_experts", dtype=torch.int32, dim=2)
    S, k = top_experts.shape
    dev = top_experts.device
    need = workspace_size("sparse_map", S, 0, 0, E, k, MOE_BF16)
    if need == 0:
        raise ValueError("sizes outside the library's limits")
    if ws is None:
        ws = alloc_workspace(need, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sparse_rows = torch.empty(S * k, dtype=torch.int32, device=dev)
    sorted_rows = torch.empty(S * k, dtype=torch.int32, device=dev)
    _check(_lib().moe_sparse_map(_ptr(top_experts), S, k, E, _ptr(counts), _ptr(offsets),
                              _ptr(sparse_rows), _ptr(sorted_rows), _ptr(ws), ws.numel(),
                              _stream(dev)))
    return counts, offsets, sparse_rows, sorted_rows


def scatter_linear(X: torch.Tensor, W: torch.Tensor, k: int, sorted_rows: torch.Tensor,
                   expert_offsets: torch.Tensor, gates: Optional[torch.Tensor] = None,
                   gather_in: bool = True, scatter_out: bool = True, S: Optional[int] = None,
                   out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """ParallelLinear(X, W, I, G) (moe_scatter_linear). Returns Y: [S, Dout] float32 when
    scatter_out (accumulated into `out` if given, else into a fresh zero tensor), otherwise
    [S*k, Dout] in X's dtype."""
    _req(X, "X", dim=2)
    _req(W, "W", dtype=X.dtype, dim=3, device=X.device)
    _req(sorted_rows, "sorted_rows", dtype=torch.int32, dim=1, device=X.device)
    _req(expert_offsets, "expert_offsets", dtype=torch.int32, dim=1, device=X.device)
    E, Din, Dout = W.shape
    if X.shape[1] != Din:
        raise ValueError("X and W disagree on Din")
    R = sorted_rows.shape[0]
    if S is None:
        S = X.shape[0] if gather_in else R // k
    if S * k != R:
        raise ValueError("sorted_rows must hold S*k entries")
    if not gather_in and X.shape[0] != R:
        raise ValueError("grouped X must have S*k rows")
    if gates is not None:
        _req(gates, "gates", dtype=torch.float32, device=X.device)
        if gates.numel() != R:
            raise ValueError("gates must hold S*k entries")
    dev = X.device
    if scatter_out:
        Y = torch.zeros((S, Dout), dtype=torch.float32, device=dev) if out is None else out
        _req(Y, "out", dtype=torch.float32, dim=2, device=dev)
    else:
        Y = torch.empty((R, Dout), dtype=X.dtype, device=dev) if out is None else out
        _req(Y, "out", dtype=X.dtype, dim=2, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_size("scatter_linear", S, Din, Dout, E, k, X.dtype), dev)
    _check(_lib().moe_scatter_linear(_ptr(X), _ptr(W), S, Din, Dout, E, k, _ptr(sorted_rows),
                                  _ptr(expert_offsets), _ptr(gates), int(bool(gather_in)),
                                  int(bool(scatter_out)), _dtype_code(X), _ptr(Y), _ptr(ws),
                                  ws.numel(), _stream(dev)))
    return Y


def scatter_linear_backward(X: torch.Tensor, W: torch.Tensor, dY: torch.Tensor, k: int,
                            sorted_rows: torch.Tensor, expert_offsets: torch.Tensor,
                            gates: Optional[torch.Tensor] = None, gather_in: bool = True,
                            scatter_out: bool = True, S: Optional[int] = None,
                            need=("dX", "dW", "dgates"), ws: Optional[torch.Tensor] = None):
    """Backward of scatter_linear (moe_scatter_linear_backward), bf16 inputs. dY has the forward
    output's shape and dtype (float32 [S, Dout] when scatter_out, else X's dtype [S*k, Dout]).
    Returns {"dX", "dW", "dgates"} for the names in `need` (dgates only with gates): dX float32
    [S, Din] when gather_in, else [S*k, Din] in X's dtype; dW float32 [E, Din, Dout]; dgates
    float32 [S*k]."""
    _req(X, "X", dim=2)
    _req(W, "W", dtype=X.dtype, dim=3, device=X.device)
    _req(sorted_rows, "sorted_rows", dtype=torch.int32, dim=1, device=X.device)
    _req(expert_offsets, "expert_offsets", dtype=torch.int32, dim=1, device=X.device)
    E, Din, Dout = W.shape
    R = sorted_rows.shape[0]
    if S is None:
        S = X.shape[0] if gather_in else R // k
    if S * k != R or X.shape[1] != Din:
        raise ValueError("shapes of X, W and sorted_rows disagree")
    _req(dY, "dY", dtype=torch.float32 if scatter_out else X.dtype, dim=2, device=X.device)
    if dY.shape != ((S if scatter_out else R), Dout):
        raise ValueError("dY must have the forward output's shape")
    if gates is not None:
        _req(gates, "gates", dtype=torch.float32, device=X.device)
    dev = X.device
    out = {}
    dX = dW = dg = None
    if "dX" in need:
        dX = torch.empty((S, Din), dtype=torch.float32, device=dev) if gather_in else \
            torch.empty((R, Din), dtype=X.dtype, device=dev)
        out["dX"] = dX
    if "dW" in need:
        dW = torch.empty((E, Din, Dout), dtype=torch.float32, device=dev)
        out["dW"] = dW
    if "dgates" in need and gates is not None:
        dg = torch.empty(R, dtype=torch.float32, device=dev)
        out["dgates"] = dg
    if ws is None:
        ws = alloc_workspace(workspace_size("scatter_linear_backward", S, Din, Dout, E, k, X.dtype),
                             dev)
    _check(_lib().moe_scatter_linear_backward(
        _ptr(X), _ptr(W), _ptr(dY), S, Din, Dout, E, k, _ptr(sorted_rows), _ptr(expert_offsets),
        _ptr(gates), int(bool(gather_in)), int(bool(scatter_out)), _dtype_code(X), _ptr(dX),
        _ptr(dW), _ptr(dg), _ptr(ws), ws.numel(), _stream(dev)))
    return out


class ForwardWorkspace:
    """A workspace for mlp_forward plus typed views of what the forward leaves in it."""

    def __init__(self, S, D, F, E, k, dtype, device):
        self.shape = (S, D, F, E, k)
        self.dtype = dtype
        code = _dtype_code(torch.empty(0, dtype=dtype))
        self.code = code
        n = workspace_size("mlp_forward", S, D, F, E, k, code)
        if n == 0:
            raise ValueError("sizes outside the library's limits")
        self.buf = alloc_workspace(n, device)

    def view(self, which: str) -> torch.Tensor:
        S, D, F, E, k = self.shape
        off = workspace_view(which, S, D, F, E, k, self.code)
        if off < 0:
            raise KeyError(which)
        R = S * k
        n, dt, shape = {
            "top_experts": (R, torch.int32, (S, k)),
            "top_weights": (R, torch.float32, (S, k)),
            "expert_counts": (E, torch.int32, (E,)),
            "expert_offsets": (E + 1, torch.int32, (E + 1,)),
            "sparse_rows": (R, torch.int32, (R,)),
            "sorted_rows": (R, torch.int32, (R,)),
            "h": (R * F, self.dtype, (R, F)),
            "x_sorted": (R * D, self.dtype, (R, D)),
        }[which]
        nbytes = n * torch.empty(0, dtype=dt).element_size()
        return self.buf[off:off + nbytes].view(dt).view(shape)


def mlp_forward(x: torch.Tensor, w_gate: torch.Tensor, w_gate_e: torch.Tensor,
                w_up: torch.Tensor, w_down: torch.Tensor, k: int,
                logit_bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                ws: Optional[ForwardWorkspace] = None) -> torch.Tensor:
    """The whole MoE expert-MLP forward (moe_mlp_forward); returns out [S, D] float32."""
    _req(x, "x", dim=2)
    dev = x.device
    for t, n, d in ((w_gate, "w_gate", 2), (w_gate_e, "w_gate_e", 3), (w_up, "w_up", 3),
                    (w_down, "w_down", 3)):
        _req(t, n, dtype=x.dtype, dim=d, device=dev)
    S, D = x.shape
    E = w_gate.shape[1]
    F = w_gate_e.shape[2]
    if w_gate.shape[0] != D or tuple(w_gate_e.shape) != (E, D, F) or \
            tuple(w_up.shape) != (E, D, F) or tuple(w_down.shape) != (E, F, D):
        raise ValueError("expected w_gate [D,E], w_gate_e/w_up [E,D,F], w_down [E,F,D]")
    if logit_bias is not None:
        _req(logit_bias, "logit_bias", dtype=torch.float32, dim=1, device=dev)
    if out is None:
        out = torch.empty((S, D), dtype=torch.float32, device=dev)
    _req(out, "out", dtype=torch.float32, dim=2, device=dev)
    if ws is None:
        ws = ForwardWorkspace(S, D, F, E, k, x.dtype, dev)
    _check(_lib().moe_mlp_forward(_ptr(x), _ptr(w_gate), _ptr(logit_bias), _ptr(w_gate_e),
                               _ptr(w_up), _ptr(w_down), S, D, F, E, k, _dtype_code(x),
                               _ptr(out), _ptr(ws.buf), ws.buf.numel(), _stream(dev)))
    return out


class MoaWorkspace:
    """A workspace for moa_forward plus views of the routing it leaves there."""

    def __init__(self, S, D, HD, E, k, device):
        self.shape = (S, D, HD, E, k)
        code = _dtype_code(torch.empty(0, dtype=torch.bfloat16))
        self.code = code
        n = workspace_size("moa_forward", S, D, HD, E, k, code)
        if n == 0:
            raise ValueError("sizes outside the library's limits")
        self.buf = alloc_workspace(n, device)

    def view(self, which: str) -> torch.Tensor:
        S, D, HD, E, k = self.shape
        R = S * k
        shapes = {
            "top_experts": (R, torch.int32, (S, k)),
            "top_weights": (R, torch.float32, (S, k)),
            "expert_counts": (E, torch.int32, (E,)),
            "expert_offsets": (E + 1, torch.int32, (E + 1,)),
            "sparse_rows": (R, torch.int32, (R,)),
            "sorted_rows": (R, torch.int32, (R,)),
        }
        if which not in shapes:
            raise KeyError(which)
        # the routing sits at the same offsets as in an mlp_forward workspace (F is irrelevant)
        off = workspace_view(which, S, D, 0, E, k, self.code)
        n, dt, shape = shapes[which]
        nbytes = n * torch.empty(0, dtype=dt).element_size()
        return self.buf[off:off + nbytes].view(dt).view(shape)


def moa_forward(x: torch.Tensor, w_gate: torch.Tensor, w_q: torch.Tensor, w_kv: torch.Tensor,
                w_o: torch.Tensor, k: int, heads: int, logit_bias: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None,
                ws: Optional[MoaWorkspace] = None) -> torch.Tensor:
    """Mixture of Attention forward (moe_moa_forward), bf16; returns out [S, D] float32.
    w_gate [D,E], w_q [E,D,H*dh], w_kv [D,2*H*dh] (key columns first), w_o [E,H*dh,D]."""
    _req(x, "x", dim=2)
    dev = x.device
    for t, n, d in ((w_gate, "w_gate", 2), (w_q, "w_q", 3), (w_kv, "w_kv", 2), (w_o, "w_o", 3)):
        _req(t, n, dtype=x.dtype, dim=d, device=dev)
    S, D = x.shape
    E = w_gate.shape[1]
    HD = w_q.shape[2]
    if heads < 1 or HD % heads != 0:
        raise ValueError("w_q's last dimension must be heads * dh")
    if w_gate.shape[0] != D or tuple(w_q.shape) != (E, D, HD) or \
            tuple(w_kv.shape) != (D, 2 * HD) or tuple(w_o.shape) != (E, HD, D):
        raise ValueError("expected w_gate [D,E], w_q [E,D,HD], w_kv [D,2HD], w_o [E,HD,D]")
    if logit_bias is not None:
        _req(logit_bias, "logit_bias", dtype=torch.float32, dim=1, device=dev)
    if out is None:
        out = torch.empty((S, D), dtype=torch.float32, device=dev)
    _req(out, "out", dtype=torch.float32, dim=2, device=dev)
    if ws is None:
        ws = MoaWorkspace(S, D, HD, E, k, dev)
    _check(_lib().moe_moa_forward(_ptr(x), _ptr(w_gate), _ptr(logit_bias), _ptr(w_q),
                               _ptr(w_kv), _ptr(w_o), S, D, heads, HD // heads, E, k,
                               _dtype_code(x), _ptr(out), _ptr(ws.buf), ws.buf.numel(),
                               _stream(dev)))
    return out


def ep_dispatch(x: torch.Tensor, top_experts: torch.Tensor, E: int,
                ws: Optional[torch.Tensor] = None) -> dict:
    """Sending side of expert parallelism (moe_ep_dispatch): the sparse map of top_experts
    [S, k] and the routed rows in slot order. Returns a dict with send_x [S*k, D] (x's dtype),
    send_e [S*k] int32, expert_counts [E], expert_offsets [E+1], sparse_rows and sorted_rows
    [S*k]."""
    _req(x, "x", dim=2)
    dev = x.device
    _req(top_experts, "top_experts", dtype=torch.int32, dim=2, device=dev)
    S, D = x.shape
    k = top_experts.shape[1]
    if top_experts.shape[0] != S:
        raise ValueError("top_experts must be [S, k]")
    R = S * k
    out = {
        "send_x": torch.empty((R, D), dtype=x.dtype, device=dev),
        "send_e": torch.empty(R, dtype=torch.int32, device=dev),
        "expert_counts": torch.empty(E, dtype=torch.int32, device=dev),
        "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "sparse_rows": torch.empty(R, dtype=torch.int32, device=dev),
        "sorted_rows": torch.empty(R, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = alloc_workspace(workspace_size("ep_dispatch", S, D, 0, E, k, _dtype_code(x)), dev)
    _check(_lib().moe_ep_dispatch(
        _ptr(x), _ptr(top_experts), S, D, E, k, _dtype_code(x), _ptr(out["expert_counts"]),
        _ptr(out["expert_offsets"]), _ptr(out["sparse_rows"]), _ptr(out["sorted_rows"]),
        _ptr(out["send_x"]), _ptr(out["send_e"]), _ptr(ws), ws.numel(), _stream(dev)))
    return out


def expert_mlp_forward(x_rows: torch.Tensor, expert_ids: torch.Tensor, expert_base: int,
                       w_gate_e: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                       y: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Expert MLP on rows with given expert ids (moe_expert_mlp_forward): row i goes through
    expert expert_ids[i] - expert_base of the given weights, unweighted; returns y [R, D] float32."""
    _req(x_rows, "x_rows", dim=2)
    dev = x_rows.device
    _req(expert_ids, "expert_ids", dtype=torch.int32, dim=1, device=dev)
    for t, n in ((w_gate_e, "w_gate_e"), (w_up, "w_up"), (w_down, "w_down")):
        _req(t, n, dtype=x_rows.dtype, dim=3, device=dev)
    R, D = x_rows.shape
    E, _, F = w_gate_e.shape
    if expert_ids.shape[0] != R or tuple(w_gate_e.shape) != (E, D, F) or \
            tuple(w_up.shape) != (E, D, F) or tuple(w_down.shape) != (E, F, D):
        raise ValueError("expected expert_ids [R], w_gate_e/w_up [E,D,F], w_down [E,F,D]")
    if y is None:
        y = torch.empty((R, D), dtype=torch.float32, device=dev)
    _req(y, "y", dtype=torch.float32, dim=2, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_size("expert_mlp_forward", R, D, F, E, 1,
                                            _dtype_code(x_rows)), dev)
    _check(_lib().moe_expert_mlp_forward(
        _ptr(x_rows), _ptr(expert_ids), int(expert_base), R, D, F, E, _ptr(w_gate_e), _ptr(w_up),
        _ptr(w_down), _dtype_code(x_rows), _ptr(y), _ptr(ws), ws.numel(), _stream(dev)))
    return y


def ep_combine(y_ret: torch.Tensor, sparse_rows: torch.Tensor, top_weights: torch.Tensor,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Expert-parallel combine (moe_ep_combine): out[s] = sum_j w[s, j] * y_ret[sparse_rows[s k + j]];
    returns out [S, D] float32."""
    _req(y_ret, "y_ret", dtype=torch.float32, dim=2)
    dev = y_ret.device
    _req(top_weights, "top_weights", dtype=torch.float32, dim=2, device=dev)
    _req(sparse_rows, "sparse_rows", dtype=torch.int32, dim=1, device=dev)
    S, k = top_weights.shape
    D = y_ret.shape[1]
    if sparse_rows.shape[0] != S * k or y_ret.shape[0] != S * k:
        raise ValueError("expected y_ret [S*k, D] and sparse_rows [S*k] for top_weights [S, k]")
    if out is None:
        out = torch.empty((S, D), dtype=torch.float32, device=dev)
    _req(out, "out", dtype=torch.float32, dim=2, device=dev)
    _check(_lib().moe_ep_combine(_ptr(y_ret), _ptr(sparse_rows), _ptr(top_weights), S, D, k,
                                 _ptr(out), _stream(dev)))
    return out


def cast_bf16(src: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """fp32 -> bf16, round-to-nearest-even (moe_cast_bf16); src's element count a multiple of 8."""
    _req(src, "src", dtype=torch.float32)
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    _req(out, "out", dtype=torch.bfloat16, device=src.device)
    if out.numel() != src.numel():
        raise ValueError("out must have src's element count")
    _check(_lib().moe_cast_bf16(_ptr(src), src.numel(), _ptr(out), _stream(src.device)))
    return out


def mlp_backward(x: torch.Tensor, w_gate: torch.Tensor, w_gate_e: torch.Tensor,
                 w_up: torch.Tensor, w_down: torch.Tensor, k: int, dout: torch.Tensor,
                 fwd_ws: ForwardWorkspace, ws: Optional[torch.Tensor] = None) -> dict:
    """Backward of mlp_forward (moe_mlp_backward), bf16: given dout [S, D] float32 and the
    workspace of the forward call on the same inputs (its routing, map and h), returns float32
    {"dx" [S, D], "dw_gate" [D, E], "dw_gate_e" [E, D, F], "dw_up" [E, D, F],
    "dw_down" [E, F, D]}."""
    _req(x, "x", dim=2)
    dev = x.device
    S, D = x.shape
    E, F = w_gate.shape[1], w_gate_e.shape[2]
    if fwd_ws.shape != (S, D, F, E, k):
        raise ValueError("the forward workspace was made for other sizes")
    _req(dout, "dout", dtype=torch.float32, dim=2, device=dev)
    out = {"dx": torch.empty((S, D), dtype=torch.float32, device=dev),
           "dw_gate": torch.empty((D, E), dtype=torch.float32, device=dev),
           "dw_gate_e": torch.empty((E, D, F), dtype=torch.float32, device=dev),
           "dw_up": torch.empty((E, D, F), dtype=torch.float32, device=dev),
           "dw_down": torch.empty((E, F, D), dtype=torch.float32, device=dev)}
    if ws is None:
        ws = alloc_workspace(workspace_size("mlp_backward", S, D, F, E, k, x.dtype), dev)
    _check(_lib().moe_mlp_backward(
        _ptr(x), _ptr(w_gate), _ptr(w_gate_e), _ptr(w_up), _ptr(w_down), _ptr(dout), S, D, F, E,
        k, _dtype_code(x), _ptr(fwd_ws.buf), fwd_ws.buf.numel(), _ptr(out["dx"]),
        _ptr(out["dw_gate"]), _ptr(out["dw_gate_e"]), _ptr(out["dw_up"]), _ptr(out["dw_down"]),
        _ptr(ws), ws.numel(), _stream(dev)))
    return out


def check_device_status(ws: torch.Tensor):
    """Synchronises and raises MoeError if the device flagged a bad expert id or a timeout."""
    buf = ws.buf if isinstance(ws, (ForwardWorkspace, MoaWorkspace)) else ws
    _check(_lib().moe_check_device_status(_ptr(buf), _stream(buf.device)))


def profile_events(events):
    """Registers torch.cuda.Event objects (>= 5) for the next mlp_forward, mlp_backward or
    moa_forward on this thread."""
    if not events:
        _check(_lib().moe_profile_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib().moe_profile_events(arr, len(events)))


def debug_wait_timeout(limit_ns: int, ws: torch.Tensor):
    _check(_lib().moe_debug_wait_timeout(limit_ns, _ptr(ws), ws.numel(), _stream(ws.device)))


def last_launch_count() -> int:
    return int(_lib().moe_last_launch_count())
