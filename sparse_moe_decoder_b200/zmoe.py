"""ctypes binding of libzmoe (argument marshalling only).

Every ``zmoe_*`` function here takes torch CUDA tensors, checks shapes and dtypes,
allocates outputs with torch (device memory is the only thing torch provides) and
calls the C entry point of the same name on the current torch stream.  Every step
of the computation runs in libzmoe's CUDA kernels; there is no CPU or PyTorch
fallback: if the shared library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzmoe.so")

ZMOE_F32 = 0
ZMOE_BF16 = 1

STATUS_NAMES = {0: "ZMOE_OK", 1: "ZMOE_ERR_INVALID_ARG", 2: "ZMOE_ERR_UNSUPPORTED", 3: "ZMOE_ERR_CUDA",
                4: "ZMOE_ERR_WORKSPACE_TOO_SMALL", 5: "ZMOE_ERR_DEVICE_CHECK", 6: "ZMOE_ERR_TIMEOUT"}

# name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
SIGNATURES = {
    "zmoe_version": (_I, []),
    "zmoe_status_string": (ctypes.c_char_p, [_I]),
    "zmoe_last_error": (ctypes.c_char_p, []),
    "zmoe_delay_shear": (_I, [_P, _P, _I, _I, _I, ctypes.c_int32, _P]),
    "zmoe_delay_unshear": (_I, [_P, _P, _I, _I, _I, _P]),
    "zmoe_embed_sum_rmsnorm": (_I, [_P, _P, _I, _P, _F, _I, _I, _I, _I, _P, _I, _P]),
    "zmoe_rmsnorm": (_I, [_P, _I, _P, _F, _I, _I, _P, _I, _P]),
    "zmoe_route": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P]),
    "zmoe_permute_workspace_size": (_S, [_I, _I, _I]),
    "zmoe_permute": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _S, _P]),
    "zmoe_permute_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "zmoe_grouped_swiglu_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "zmoe_grouped_swiglu": (_I, [_P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _S, _P]),
    "zmoe_combine": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "zmoe_moe_layer_workspace_size": (_S, [_I, _I, _I, _I, _I, _I]),
    "zmoe_output_heads_workspace_size": (_S, [_I, _I]),
    "zmoe_moe_layer_fp8_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "zmoe_moe_layer_fp8": (_I, [_P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P,
                                _P, _P, _P, _S, _P]),
    "zmoe_speaker_prefix": (_I, [_P, _P, _I, _P, _I, _I, _I, _P, _P]),
    "zmoe_output_heads": (_I, [_P, _P, _F, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _S, _P]),
    "zmoe_moe_layer": (_I, [_P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                            _P, _S, _P]),
    "zmoe_get_device_errors": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "zmoe_debug_inject_timeout": (_I, [ctypes.c_uint32, ctypes.c_uint64]),
    "zmoe_decode_stack_workspace_size": (_S, [_I, _I, _I, _I]),
    "zmoe_prepare_w_down_f16": (_I, [_P, _I, _I, _I, _P, _P, _P, _S, _P]),
    "zmoe_grouped_swiglu_f16h": (_I, [_P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "zmoe_moe_layer_f16h_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "zmoe_moe_layer_w8a8_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "zmoe_moe_layer_w8a8_workspace_layout": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t), _I]),
    "zmoe_moe_layer_w8a8": (_I, [_P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P,
                                 _P, _P, _P, _S, _P]),
    "zmoe_moe_layer_f16h": (_I, [_P, _P, _P, _F, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                 _P, _S, _P]),
    "zmoe_decode_stack": (_I, [_P, _I, _I, _I, _F, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _S, _P]),
}


class StackLayer(ctypes.Structure):
    """zmoe_stack_layer (include/zmoe.h)."""
    _fields_ = [("w_router", _P), ("logit_bias", _P), ("sel_bias", _P), ("gamma", _P), ("w_gate", _P),
                ("w_up", _P), ("w_down", _P), ("E", _I), ("k", _I)]


class ZmoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}" + (f" ({detail})" if detail else ""))


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libzmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libzmoe.so not found at {LIB_PATH}; build it with "
                              "`python -m sparse_moe_decoder_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        detail = lib().zmoe_last_error().decode(errors="replace")
        raise ZmoeError(status, where, detail)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return ZMOE_F32
    if dt == torch.bfloat16:
        return ZMOE_BF16
    raise TypeError(f"libzmoe computes in float32 or bfloat16, got {dt}")


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")


# ---------------------------------------------------------------------------------------------
# the C-ABI calls
# ---------------------------------------------------------------------------------------------

def zmoe_version() -> int:
    return lib().zmoe_version()


def zmoe_delay_shear(X: torch.Tensor, pad: int = 1024, out: Optional[torch.Tensor] = None, stream=None):
    """Y[b, t, j] = X[b, t - j, j] (pad outside), X int32 [B, T, N] or [T, N]."""
    _need(X, "X", torch.int32)
    squeeze = X.dim() == 2
    X3 = X.unsqueeze(0) if squeeze else X
    B, T, N = X3.shape
    Y = out if out is not None else torch.empty((B, T + N - 1, N), dtype=torch.int32, device=X.device)
    _check(lib().zmoe_delay_shear(_ptr(X3), _ptr(Y), B, T, N, int(pad), _stream(stream)), "zmoe_delay_shear")
    return Y[0] if squeeze and out is None else Y


def zmoe_delay_unshear(Y: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """X_hat[b, t, j] = Y[b, t + j, j], Y int32 [B, Ty, N] or [Ty, N]."""
    _need(Y, "Y", torch.int32)
    squeeze = Y.dim() == 2
    Y3 = Y.unsqueeze(0) if squeeze else Y
    B, Ty, N = Y3.shape
    X = out if out is not None else torch.empty((B, max(Ty - N + 1, 0), N), dtype=torch.int32, device=Y.device)
    _check(lib().zmoe_delay_unshear(_ptr(Y3), _ptr(X), B, Ty, N, _stream(stream)), "zmoe_delay_unshear")
    return X[0] if squeeze and out is None else X


def zmoe_embed_sum_rmsnorm(ids: torch.Tensor, tables: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                           out_dtype: Optional[torch.dtype] = None, out: Optional[torch.Tensor] = None, stream=None):
    """RMSNorm(sum_j tables[j, ids[:, j]]) * gamma.  ids int32 [T, N], tables [N, V, d]."""
    _need(ids, "ids", torch.int32, 2)
    _need(tables, "tables", None, 3)
    _need(gamma, "gamma", torch.float32, 1)
    T, N = ids.shape
    Nt, V, d = tables.shape
    if Nt != N or gamma.shape[0] != d:
        raise ValueError("ids / tables / gamma shapes disagree")
    od = out_dtype or tables.dtype
    o = out if out is not None else torch.empty((T, d), dtype=od, device=ids.device)
    _check(lib().zmoe_embed_sum_rmsnorm(_ptr(ids), _ptr(tables), _dtype_code(tables.dtype), _ptr(gamma), float(eps),
                                        T, N, V, d, _ptr(o), _dtype_code(o.dtype), _stream(stream)),
           "zmoe_embed_sum_rmsnorm")
    return o


def zmoe_rmsnorm(h: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6, out_dtype: Optional[torch.dtype] = None,
                 out: Optional[torch.Tensor] = None, stream=None):
    _need(h, "h", None, 2)
    _need(gamma, "gamma", torch.float32, 1)
    T, d = h.shape
    o = out if out is not None else torch.empty((T, d), dtype=out_dtype or h.dtype, device=h.device)
    _check(lib().zmoe_rmsnorm(_ptr(h), _dtype_code(h.dtype), _ptr(gamma), float(eps), T, d, _ptr(o),
                              _dtype_code(o.dtype), _stream(stream)), "zmoe_rmsnorm")
    return o


def zmoe_route(x: torch.Tensor, w_router: Optional[torch.Tensor], k: int, logit_bias: Optional[torch.Tensor] = None,
               sel_bias: Optional[torch.Tensor] = None, margin: bool = True, outs=None, stream=None):
    """Returns (expert_idx int32 [T, k], gates f32 [T, k], margin f32 [T] or None).

    w_router None means one expert without a router (a dense FFN layer): expert 0, gate 1."""
    _need(x, "x", None, 2)
    if w_router is not None:
        _need(w_router, "w_router", x.dtype, 2)
    for t, n in ((logit_bias, "logit_bias"), (sel_bias, "sel_bias")):
        if t is not None:
            _need(t, n, torch.float32, 1)
    T, d = x.shape
    E = w_router.shape[0] if w_router is not None else 1
    if outs is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        g = torch.empty((T, k), dtype=torch.float32, device=x.device)
        mg = torch.empty((T,), dtype=torch.float32, device=x.device) if margin else None
    else:
        idx, g, mg = outs
    _check(lib().zmoe_route(_ptr(x), _ptr(w_router), _dtype_code(x.dtype), _ptr(logit_bias), _ptr(sel_bias), T, d, E,
                            k, _ptr(idx), _ptr(g), _ptr(mg), _stream(stream)), "zmoe_route")
    return idx, g, mg


def zmoe_permute_workspace_size(T: int, E: int, k: int) -> int:
    return int(lib().zmoe_permute_workspace_size(T, E, k))


def zmoe_permute(expert_idx: torch.Tensor, x: torch.Tensor, E: int, outs: Optional[dict] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """counts, offsets, perm, inv_perm, x_perm of a [T, k] expert assignment."""
    _need(expert_idx, "expert_idx", torch.int32, 2)
    _need(x, "x", None, 2)
    T, k = expert_idx.shape
    d = x.shape[1]
    dev = x.device
    if outs is None:
        outs = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
                    offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                    perm=torch.empty(T * k, dtype=torch.int32, device=dev),
                    inv_perm=torch.empty((T, k), dtype=torch.int32, device=dev),
                    x_perm=torch.empty((T * k, d), dtype=x.dtype, device=dev))
    ws_bytes = zmoe_permute_workspace_size(T, E, k)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _check(lib().zmoe_permute(_ptr(expert_idx), _ptr(x), _dtype_code(x.dtype), T, d, E, k, _ptr(outs["counts"]),
                              _ptr(outs["offsets"]), _ptr(outs["perm"]), _ptr(outs["inv_perm"]),
                              _ptr(outs["x_perm"]), _ptr(workspace), workspace.numel(), _stream(stream)),
           "zmoe_permute")
    return outs


def zmoe_grouped_swiglu_workspace_size(M_total: int, E: int, d: int, f: int, dtype: torch.dtype) -> int:
    return int(lib().zmoe_grouped_swiglu_workspace_size(M_total, E, d, f, _dtype_code(dtype)))


def hidden_cols(f: int, dtype: torch.dtype) -> int:
    """Columns of the h scratch of zmoe_grouped_swiglu: 2f (h_hi | h_lo) for bf16, f for f32."""
    return 2 * f if dtype == torch.bfloat16 else f


def zmoe_grouped_swiglu(x_perm: torch.Tensor, offsets: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
                        w_down: torch.Tensor, h: Optional[torch.Tensor] = None, y_perm: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None):
    """Returns (h, y_perm f32 [M, d]).  h is bf16 [M, 2f] = [h_hi | h_lo] for bf16 inputs
    (h ~= h_hi + h_lo), f32 [M, f] for f32 inputs."""
    _need(x_perm, "x_perm", None, 2)
    _need(offsets, "offsets", torch.int32, 1)
    for t, n in ((w_gate, "w_gate"), (w_up, "w_up"), (w_down, "w_down")):
        _need(t, n, x_perm.dtype, 3)
    M, d = x_perm.shape
    E, f, _ = w_gate.shape
    dev = x_perm.device
    if h is None:
        h = torch.empty((M, hidden_cols(f, x_perm.dtype)), dtype=x_perm.dtype, device=dev)
    if y_perm is None:
        y_perm = torch.empty((M, d), dtype=torch.float32, device=dev)
    ws_bytes = zmoe_grouped_swiglu_workspace_size(M, E, d, f, x_perm.dtype)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _check(lib().zmoe_grouped_swiglu(_ptr(x_perm), _ptr(offsets), M, _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                     _dtype_code(x_perm.dtype), E, d, f, _ptr(h), _ptr(y_perm), _ptr(workspace),
                                     workspace.numel(), _stream(stream)), "zmoe_grouped_swiglu")
    return h, y_perm


def zmoe_combine(y_perm: torch.Tensor, inv_perm: torch.Tensor, gates: torch.Tensor,
                 residual: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    """y[t] = residual[t] + sum_i gates[t, i] * y_perm[inv_perm[t, i]], all f32."""
    _need(y_perm, "y_perm", torch.float32, 2)
    _need(inv_perm, "inv_perm", torch.int32, 2)
    _need(gates, "gates", torch.float32, 2)
    T, k = inv_perm.shape
    d = y_perm.shape[1]
    if residual is not None:
        _need(residual, "residual", torch.float32, 2)
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=y_perm.device)
    _check(lib().zmoe_combine(_ptr(y_perm), _ptr(inv_perm), _ptr(gates), _ptr(residual), T, d, k, _ptr(y),
                              _stream(stream)), "zmoe_combine")
    return y


def zmoe_moe_layer_workspace_size(T: int, d: int, f: int, E: int, k: int, dtype: torch.dtype) -> int:
    return int(lib().zmoe_moe_layer_workspace_size(T, d, f, E, k, _dtype_code(dtype)))


def zmoe_moe_layer(w_router: Optional[torch.Tensor], w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, k: int,
                   x: Optional[torch.Tensor] = None, h: Optional[torch.Tensor] = None,
                   gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                   logit_bias: Optional[torch.Tensor] = None, sel_bias: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, outs: Optional[dict] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = h + MoE(x), or with gamma y = h + MoE(RMSNorm(h) * gamma); f32 [T, d].

    ``outs`` may hold preallocated ``expert_idx`` int32 [T, k], ``gates`` f32 [T, k], ``margin`` f32 [T]
    and ``x_norm`` [T, d] tensors to receive those intermediates.
    """
    src = h if gamma is not None else x
    if src is None:
        raise ValueError("zmoe_moe_layer: needs x, or h with gamma")
    T, d = src.shape
    E, f = w_gate.shape[0], w_gate.shape[1]
    dt = w_gate.dtype
    if x is not None:
        _need(x, "x", dt, 2)
    if h is not None:
        _need(h, "h", torch.float32, 2)
    outs = outs or {}
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=src.device)
    ws_bytes = zmoe_moe_layer_workspace_size(T, d, f, E, k, dt)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=src.device)
    _check(lib().zmoe_moe_layer(_ptr(x), _ptr(h), _ptr(gamma), float(eps), _ptr(w_router), _ptr(logit_bias),
                                _ptr(sel_bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _dtype_code(dt), T, d, f, E,
                                k, _ptr(y), _ptr(outs.get("expert_idx")), _ptr(outs.get("gates")),
                                _ptr(outs.get("margin")), _ptr(outs.get("x_norm")), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)), "zmoe_moe_layer")
    return y


def zmoe_moe_layer_fp8(w_router: Optional[torch.Tensor], q_gate: torch.Tensor, s_gate: torch.Tensor,
                       q_up: torch.Tensor, s_up: torch.Tensor, q_down: torch.Tensor, s_down: torch.Tensor, k: int,
                       x: Optional[torch.Tensor] = None, h: Optional[torch.Tensor] = None,
                       gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                       logit_bias: Optional[torch.Tensor] = None, sel_bias: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, outs: Optional[dict] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """zmoe_moe_layer with fp8 expert weights: q_* uint8 E4M3 codes, s_* f32 row scales (w = code * scale)."""
    src = h if gamma is not None else x
    if src is None:
        raise ValueError("zmoe_moe_layer_fp8: needs x, or h with gamma")
    T, d = src.shape
    E, f = q_gate.shape[0], q_gate.shape[1]
    for t, n in ((q_gate, "q_gate"), (q_up, "q_up"), (q_down, "q_down")):
        _need(t, n, torch.uint8, 3)
    for t, n in ((s_gate, "s_gate"), (s_up, "s_up"), (s_down, "s_down")):
        _need(t, n, torch.float32, 2)
    if h is not None:
        _need(h, "h", torch.float32, 2)
    outs = outs or {}
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=src.device)
    ws_bytes = int(lib().zmoe_moe_layer_fp8_workspace_size(T, d, f, E, k))
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=src.device)
    _check(lib().zmoe_moe_layer_fp8(_ptr(x), _ptr(h), _ptr(gamma), float(eps), _ptr(w_router), _ptr(logit_bias),
                                    _ptr(sel_bias), _ptr(q_gate), _ptr(s_gate), _ptr(q_up), _ptr(s_up), _ptr(q_down),
                                    _ptr(s_down), T, d, f, E, k, _ptr(y), _ptr(outs.get("expert_idx")),
                                    _ptr(outs.get("gates")), _ptr(outs.get("margin")), _ptr(outs.get("x_norm")),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "zmoe_moe_layer_fp8")
    return y


def zmoe_output_heads(h: torch.Tensor, w_heads: torch.Tensor, gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                      want_logits: bool = False, want_x: bool = False, outs: Optional[dict] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """The codebook heads on the final hidden state h (f32 [T, d]) and the greedy next frame.

    Returns dict(ids=int32 [T, N], logits=f32 [T, N, V] or None, x=[T, d] or None); ``outs`` may hold
    preallocated tensors under the same names."""
    _need(h, "h", torch.float32, 2)
    _need(w_heads, "w_heads", None, 3)
    T, d = h.shape
    N, V = w_heads.shape[0], w_heads.shape[1]
    outs = dict(outs or {})
    ids = outs.get("ids")
    if ids is None:
        ids = torch.empty((T, N), dtype=torch.int32, device=h.device)
    lg = outs.get("logits")
    if lg is None and want_logits:
        lg = torch.empty((T, N, V), dtype=torch.float32, device=h.device)
    x = outs.get("x")
    if x is None and want_x:
        x = torch.empty((T, d), dtype=w_heads.dtype, device=h.device)
    ws_bytes = int(lib().zmoe_output_heads_workspace_size(T, N))
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=h.device)
    _check(lib().zmoe_output_heads(_ptr(h), _ptr(gamma), float(eps), _ptr(w_heads), _dtype_code(w_heads.dtype), T, N,
                                   V, d, _ptr(ids), _ptr(lg), _ptr(x), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "zmoe_output_heads")
    return dict(ids=ids, logits=lg, x=x)


def zmoe_speaker_prefix(e: torch.Tensor, w_spk: torch.Tensor, b_spk: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """h_spk = W_spk e + b_spk: e f32 [B, n_in], W_spk [d, n_in] -> f32 [B, d]."""
    _need(e, "e", torch.float32, 2)
    _need(w_spk, "w_spk", None, 2)
    if b_spk is not None:
        _need(b_spk, "b_spk", torch.float32, 1)
    B, n_in = e.shape
    d = w_spk.shape[0]
    y = out if out is not None else torch.empty((B, d), dtype=torch.float32, device=e.device)
    _check(lib().zmoe_speaker_prefix(_ptr(e), _ptr(w_spk), _dtype_code(w_spk.dtype), _ptr(b_spk), B, d, n_in, _ptr(y),
                                     _stream(stream)), "zmoe_speaker_prefix")
    return y


def zmoe_prepare_w_down_f16(w_down: torch.Tensor, out: Optional[torch.Tensor] = None,
                            scale: Optional[torch.Tensor] = None, stream=None):
    """The f16 copy of bf16 W_down [E, d, f] (each expert scaled by a power of two) and its per-expert
    factors down_scale [E] f32 (w_down = w_down_f16 * down_scale, exact)."""
    _need(w_down, "w_down", torch.bfloat16, 3)
    E, d, f = w_down.shape
    out = out if out is not None else torch.empty((E, d, f), dtype=torch.float16, device=w_down.device)
    scale = scale if scale is not None else torch.empty((E,), dtype=torch.float32, device=w_down.device)
    ws = torch.empty(max(4 * E, 16), dtype=torch.uint8, device=w_down.device)
    _check(lib().zmoe_prepare_w_down_f16(_ptr(w_down), E, d, f, _ptr(out), _ptr(scale), _ptr(ws), ws.numel(),
                                         _stream(stream)), "zmoe_prepare_w_down_f16")
    return out, scale


def zmoe_grouped_swiglu_f16h(x_perm: torch.Tensor, offsets: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
                             w_down_f16: torch.Tensor, down_scale: torch.Tensor, h: Optional[torch.Tensor] = None,
                             y_perm: Optional[torch.Tensor] = None, stream=None):
    """Prefill grouped SwiGLU with h in f16 and the prepared down weights.  Returns (h f16 [M, f], y_perm f32)."""
    _need(x_perm, "x_perm", torch.bfloat16, 2)
    _need(w_down_f16, "w_down_f16", torch.float16, 3)
    M, d = x_perm.shape
    E, f = w_gate.shape[0], w_gate.shape[1]
    h = h if h is not None else torch.empty((M, f), dtype=torch.float16, device=x_perm.device)
    y_perm = y_perm if y_perm is not None else torch.empty((M, d), dtype=torch.float32, device=x_perm.device)
    _check(lib().zmoe_grouped_swiglu_f16h(_ptr(x_perm), _ptr(offsets), M, _ptr(w_gate), _ptr(w_up), _ptr(w_down_f16),
                                          _ptr(down_scale), E, d, f, _ptr(h), _ptr(y_perm), _stream(stream)),
           "zmoe_grouped_swiglu_f16h")
    return h, y_perm


def zmoe_moe_layer_f16h(w_router: Optional[torch.Tensor], w_gate: torch.Tensor, w_up: torch.Tensor,
                        w_down_f16: torch.Tensor, down_scale: torch.Tensor, k: int, x: Optional[torch.Tensor] = None,
                        h: Optional[torch.Tensor] = None, gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                        logit_bias: Optional[torch.Tensor] = None, sel_bias: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, outs: Optional[dict] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """zmoe_moe_layer with the prepared f16 down weights (prefill sizes); f32 [T, d]."""
    src = h if gamma is not None else x
    if src is None:
        raise ValueError("zmoe_moe_layer_f16h: needs x, or h with gamma")
    T, d = src.shape
    E, f = w_gate.shape[0], w_gate.shape[1]
    if x is not None:
        _need(x, "x", torch.bfloat16, 2)
    outs = outs or {}
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=src.device)
    ws_bytes = int(lib().zmoe_moe_layer_f16h_workspace_size(T, d, f, E, k))
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=src.device)
    _check(lib().zmoe_moe_layer_f16h(_ptr(x), _ptr(h), _ptr(gamma), float(eps), _ptr(w_router), _ptr(logit_bias),
                                     _ptr(sel_bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down_f16), _ptr(down_scale), T,
                                     d, f, E, k, _ptr(y), _ptr(outs.get("expert_idx")), _ptr(outs.get("gates")),
                                     _ptr(outs.get("margin")), _ptr(outs.get("x_norm")), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "zmoe_moe_layer_f16h")
    return y


def zmoe_moe_layer_w8a8(w_router: Optional[torch.Tensor], q_gate: torch.Tensor, s_gate: torch.Tensor,
                        q_up: torch.Tensor, s_up: torch.Tensor, q_down: torch.Tensor, s_down: torch.Tensor, k: int,
                        x: Optional[torch.Tensor] = None, h: Optional[torch.Tensor] = None,
                        gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                        logit_bias: Optional[torch.Tensor] = None, sel_bias: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, outs: Optional[dict] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The W8A8 fp8 layer (prefill sizes); f32 [T, d].  Weights: uint8 E4M3 codes [E, f, d] / [E, d, f]
    with f32 row scales [E, f] / [E, d]."""
    src = h if gamma is not None else x
    if src is None:
        raise ValueError("zmoe_moe_layer_w8a8: needs x, or h with gamma")
    T, d = src.shape
    E, f = q_gate.shape[0], q_gate.shape[1]
    for t, n in ((q_gate, "q_gate"), (q_up, "q_up"), (q_down, "q_down")):
        _need(t, n, torch.uint8, 3)
    outs = outs or {}
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=src.device)
    ws_bytes = int(lib().zmoe_moe_layer_w8a8_workspace_size(T, d, f, E, k))
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=src.device)
    _check(lib().zmoe_moe_layer_w8a8(_ptr(x), _ptr(h), _ptr(gamma), float(eps), _ptr(w_router), _ptr(logit_bias),
                                     _ptr(sel_bias), _ptr(q_gate), _ptr(s_gate), _ptr(q_up), _ptr(s_up), _ptr(q_down),
                                     _ptr(s_down), T, d, f, E, k, _ptr(y), _ptr(outs.get("expert_idx")),
                                     _ptr(outs.get("gates")), _ptr(outs.get("margin")), _ptr(outs.get("x_norm")),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "zmoe_moe_layer_w8a8")
    return y


def w8a8_intermediates(workspace: torch.Tensor, T: int, d: int, f: int, E: int, k: int) -> dict:
    """Views of zmoe_moe_layer_w8a8's intermediates inside its workspace (after the call)."""
    o = (ctypes.c_size_t * 10)()
    _check(lib().zmoe_moe_layer_w8a8_workspace_layout(T, d, f, E, k, o, 10), "zmoe_moe_layer_w8a8_workspace_layout")
    M = T * k
    shapes = (("counts", torch.int32, (E,)), ("offsets", torch.int32, (E + 1,)), ("perm", torch.int32, (M,)),
              ("inv_perm", torch.int32, (T, k)), ("xq", torch.uint8, (M, d)), ("sx", torch.float32, (M,)),
              ("h16", torch.float16, (M, f)), ("hq", torch.uint8, (M, f)), ("sh", torch.float32, (M,)),
              ("y_perm", torch.float32, (M, d)))
    out = {}
    for i, (name, dt, shape) in enumerate(shapes):
        n = 1
        for v in shape:
            n *= v
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        out[name] = workspace[o[i]:o[i] + nbytes].view(dt).view(shape)
    return out


def zmoe_decode_stack_workspace_size(n_layers: int, d: int, f: int, E_max: int) -> int:
    """Bytes of workspace for zmoe_decode_stack; 0 when these sizes are not supported."""
    return int(lib().zmoe_decode_stack_workspace_size(n_layers, d, f, E_max))


def stack_layers(layers) -> ctypes.Array:
    """The zmoe_stack_layer array of a list of MoEWeights-like objects (w_router, logit_bias, sel_bias,
    gamma, w_gate, w_up, w_down, k).  The tensors must stay alive while the array is used."""
    arr = (StackLayer * len(layers))()
    for i, L in enumerate(layers):
        for name in ("w_gate", "w_up", "w_down"):
            _need(getattr(L, name), name, torch.bfloat16, 3)
        _need(L.gamma, "gamma", torch.float32, 1)
        arr[i] = StackLayer(_ptr(L.w_router), _ptr(L.logit_bias), _ptr(L.sel_bias), _ptr(L.gamma), _ptr(L.w_gate),
                            _ptr(L.w_up), _ptr(L.w_down), L.w_gate.shape[0], L.k)
    return arr


def zmoe_decode_stack(layers, h: torch.Tensor, eps: float = 1e-6, ids: Optional[torch.Tensor] = None,
                      tables: Optional[torch.Tensor] = None, gamma0: Optional[torch.Tensor] = None,
                      outs: Optional[dict] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                      layer_array: Optional[ctypes.Array] = None) -> torch.Tensor:
    """The batch-1 stack in one call: h [1, d] (or [d]) f32 in place; with ``ids`` [N] / [1, N] the
    stack input is the embedding sum + RMSNorm of ``tables`` [N, V, d] with ``gamma0``.

    ``outs`` may hold ``layer_idx`` int32 [L, 2], ``layer_gates`` f32 [L, 2], ``layer_h`` f32 [L, d] and
    ``layer_x`` bf16 [L, d].  ``layer_array`` (from ``stack_layers``) skips rebuilding the descriptors.
    """
    _need(h, "h", torch.float32)
    d = h.shape[-1]
    n = len(layers)
    f = layers[0].w_gate.shape[1]
    outs = outs or {}
    arr = layer_array if layer_array is not None else stack_layers(layers)
    N = V = 0
    if ids is not None:
        _need(ids, "ids", torch.int32)
        _need(tables, "tables", torch.bfloat16, 3)
        N, V = tables.shape[0], tables.shape[1]
    ws_bytes = zmoe_decode_stack_workspace_size(n, d, f, max(L.w_gate.shape[0] for L in layers))
    if ws_bytes == 0:
        raise ZmoeError(2, "zmoe_decode_stack", "these sizes are not supported")
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=h.device)
    _check(lib().zmoe_decode_stack(ctypes.cast(arr, _P), n, d, f, float(eps), _ptr(ids), _ptr(tables), _ptr(gamma0),
                                   N, V, _ptr(h), _ptr(outs.get("layer_idx")), _ptr(outs.get("layer_gates")),
                                   _ptr(outs.get("layer_h")), _ptr(outs.get("layer_x")), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "zmoe_decode_stack")
    return h


def zmoe_get_device_errors(stream=None) -> int:
    """Reads and clears the device error counter (synchronises the stream)."""
    c = ctypes.c_uint32(0)
    st = lib().zmoe_get_device_errors(_stream(stream), ctypes.byref(c))
    if st not in (0, 5, 6):
        _check(st, "zmoe_get_device_errors")
    return int(c.value)
