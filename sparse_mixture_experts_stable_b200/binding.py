"""Thin ctypes binding of ``libmoe.so`` (declared in ``include/moe.h``).

Every function here has the name of the C entry point it calls and does only
argument marshalling: it checks shapes and dtypes, allocates missing output and
workspace tensors with PyTorch on the current CUDA device, and passes raw
pointers plus the current stream.  All arithmetic runs in the CUDA library.
There is no fallback: if ``libmoe.so`` is missing or fails to load, importing
this module's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_BAD_INDEX = 4
MOE_ERR_NONFINITE = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_WORKSPACE = 7

MOE_F32, MOE_BF16 = 0, 1
BASE = {"zero": 0, "input": 1, "tensor": 2}
FFN = {"linear": 0, "gelu_mlp": 1, "swiglu": 2}
ROUTER_LAYOUT = {"DE": 0, "ED": 1}

EXPORTED = [
    "moe_status_string", "moe_version", "moe_capacity", "moe_route_workspace_size", "moe_route",
    "moe_dispatch_workspace_size", "moe_dispatch", "moe_expert_ffn_workspace_size", "moe_expert_ffn",
    "moe_combine", "moe_aux_stats", "moe_backward_workspace_size", "moe_backward", "moe_transpose_weights",
    "moe_clear_status", "moe_read_status", "moe_dispatch_static_max_state_bytes", "moe_dispatch_static",
    "moe_route_ex", "moe_renormalize_kept_gates", "moe_expert_ffn_gathered", "moe_backward_swiglu_workspace_size",
    "moe_backward_swiglu", "moe_router_backward_workspace_size", "moe_router_backward",
    "moe_backward_gelu_workspace_size", "moe_backward_gelu", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_combine",
    "moe_ipc_export", "moe_ipc_import", "moe_ipc_close", "moe_expert_ffn_save", "moe_wait_probe",
    "moe_swiglu_layer_workspace_size", "moe_swiglu_layer_forward",
]
IPC_HANDLE_BYTES = 64
SCORING = {"softmax": 0, "sigmoid": 1}


class SwiGLULayerDesc(ctypes.Structure):
    """``moe_swiglu_layer`` of include/moe.h (sizes and device weight pointers)."""

    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("F", ctypes.c_int64), ("F_shared", ctypes.c_int64),
                ("C", ctypes.c_int64), ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("aux_coef", ctypes.c_float),
                ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
                ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


_lib = None
_vp, _i64, _i32, _sz, _f32, _f64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t,
                                     ctypes.c_float, ctypes.c_double)


def lib():
    """Load ``libmoe.so`` (raises OSError/FileNotFoundError when it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(
                f"{LIB_PATH} is not built; run `python -m sparse_mixture_experts_stable_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_version.restype = ctypes.c_int
        L.moe_capacity.argtypes = [_i64, _i32, _i32, _f64, ctypes.POINTER(_i64)]
        L.moe_route_workspace_size.restype = _sz
        L.moe_route_workspace_size.argtypes = [_i64, _i64, _i32, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.moe_route.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, ctypes.c_int, _i32, _vp, _i32, _vp, _vp,
                                _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_route_ex.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _vp, ctypes.c_int, _i32, _vp, _i32,
                                   ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_renormalize_kept_gates.argtypes = [_vp, _vp, _i64, _i32, _vp, _vp]
        L.moe_dispatch_workspace_size.restype = _sz
        L.moe_dispatch_workspace_size.argtypes = [_i64, _i32, _i32]
        L.moe_dispatch.argtypes = [_vp, _i64, _i32, _i32, _i64, _vp, ctypes.c_int, _i64, _i64, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_dispatch_static_max_state_bytes.restype = _sz
        L.moe_dispatch_static_max_state_bytes.argtypes = []
        L.moe_dispatch_static.argtypes = [_vp, _i64, _i32, _i32, _i64, _vp, ctypes.c_int, _i64, _i64, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _vp, _vp]
        L.moe_expert_ffn_workspace_size.restype = _sz
        L.moe_expert_ffn_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, _i32, _i64, _i64, _i64, _i64]
        L.moe_expert_ffn.argtypes = [ctypes.c_int, ctypes.c_int, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _vp,
                                     _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_expert_ffn_gathered.argtypes = [ctypes.c_int, ctypes.c_int, _vp, _i64, _i64, _vp, _vp, _i32, _i64,
                                              _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_combine.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, _i64, _i32, _i32, _i64, _i64, ctypes.c_int,
                                  _vp, _i64, _vp, _i64, ctypes.c_int, _vp, _vp]
        L.moe_aux_stats.argtypes = [_vp, _vp, _i64, _i32, _i32, ctypes.c_int, _f32, _vp, _vp, ctypes.c_int, _vp,
                                    _vp]
        L.moe_router_backward_workspace_size.restype = _sz
        L.moe_router_backward_workspace_size.argtypes = [_i64, _i64, _i32, ctypes.c_int, ctypes.c_int]
        L.moe_router_backward.argtypes = [ctypes.c_int, _vp, _i64, _i64, _i64, _vp, ctypes.c_int, _i32, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_backward_swiglu_workspace_size.restype = _sz
        L.moe_backward_swiglu_workspace_size.argtypes = [_i32, _i64, _i64, _i64]
        L.moe_expert_ffn_save.argtypes = [_vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _sz, _vp]
        L.moe_backward_swiglu.argtypes = [ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _i64,
                                          _i32, _i32, _i64, _i64, _i64, ctypes.c_int, _f32, ctypes.c_int, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_backward_gelu_workspace_size.restype = _sz
        L.moe_backward_gelu_workspace_size.argtypes = [_i32, _i64, _i64, _i64, _i64]
        L.moe_backward_gelu.argtypes = [ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                        _i32, _i32, _i64, _i64, _i64, _i64, ctypes.c_int, _f32, ctypes.c_int, _vp,
                                        _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_backward_workspace_size.restype = _sz
        L.moe_backward_workspace_size.argtypes = [_i32, _i64, _i64, _i64]
        L.moe_backward.argtypes = [ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _i64, _i32, _i32, _i64, _i64, _i64, ctypes.c_int, _f32, ctypes.c_int, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_ep_plan.argtypes = [_vp, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp]
        L.moe_ep_dispatch.argtypes = [_vp, _i64, _i32, _i32, _i64, _vp, _i64, _vp, ctypes.c_int, _i64, _i64, _vp,
                                      _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.moe_ep_combine.argtypes = [_vp, _i32, _vp, _vp, _vp, ctypes.c_int, _i64, _i32, _i32, _i64, _i64,
                                     ctypes.c_int, _vp, _i64, _vp, _i64, ctypes.c_int, _vp, _vp]
        L.moe_ipc_export.argtypes = [_vp, _vp, ctypes.POINTER(_i64)]
        L.moe_ipc_import.argtypes = [_vp, ctypes.POINTER(_vp)]
        L.moe_ipc_close.argtypes = [_vp]
        L.moe_transpose_weights.argtypes = [_vp, _vp, _i32, _i64, _i64, ctypes.c_int, _vp]
        L.moe_wait_probe.argtypes = [_vp, _i64, _vp, _vp]
        L.moe_swiglu_layer_workspace_size.restype = _sz
        L.moe_swiglu_layer_workspace_size.argtypes = [ctypes.POINTER(SwiGLULayerDesc)]
        L.moe_swiglu_layer_forward.argtypes = [ctypes.POINTER(SwiGLULayerDesc), _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                               _vp, _vp, _vp, _vp, _vp]
        L.moe_clear_status.argtypes = [_vp, _vp]
        L.moe_read_status.argtypes = [_vp, _vp, ctypes.POINTER(_i32)]
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _tdt(code: int):
    return torch.float32 if code == MOE_F32 else torch.bfloat16


def _dev(t: torch.Tensor):
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    return t.device


def _rowstride(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]):
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace holds {ws.numel() * ws.element_size()} bytes, needs {nbytes}")
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


# ------------------------------------------------------------------------------
def moe_capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    c = _i64(0)
    _check("moe_capacity", lib().moe_capacity(T, k, E, float(capacity_factor), ctypes.byref(c)))
    return int(c.value)


def moe_route_workspace_size(T, D, E, dtype: int, has_router_weight: bool, layout: str = "ED") -> int:
    return int(lib().moe_route_workspace_size(T, D, E, dtype, int(has_router_weight), ROUTER_LAYOUT[layout]))


def moe_route(x: torch.Tensor, k: int, w_router: Optional[torch.Tensor] = None, layout: str = "ED",
              E: Optional[int] = None, logit_bias: Optional[torch.Tensor] = None, want_logits: bool = False,
              out: Optional[dict] = None, dev_status: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, stream=None, scoring: str = "softmax",
              selection_bias: Optional[torch.Tensor] = None, want_z_loss: bool = False) -> dict:
    """Router scores, clean scores (softmax or sigmoid), stable top-k, gates, counts, score sums.

    ``x`` is (T, D) activations with ``w_router`` given in ``layout`` ("ED" =
    nn.Linear (E, D), "DE" = (D, E)), or (T, E) logits when ``w_router`` is None.
    ``selection_bias`` (E) moves the selection only.  Calls ``moe_route_ex``
    (``moe_route`` is its softmax, no-bias case).  Returns a dict of device
    tensors: selected, gates (x dtype), gates_f32, counts, prob_sum (and logits,
    z_loss when requested).
    """
    dev = _dev(x)
    dt = _dt(x)
    T = x.shape[0]
    if w_router is not None:
        if w_router.dtype != x.dtype:
            raise TypeError("w_router must have x's dtype")
        D = x.shape[1]
        E = w_router.shape[0] if layout == "ED" else w_router.shape[1]
        w_router = w_router.contiguous()
    else:
        D = 0
        E = x.shape[1]
    o = dict(out or {})
    o.setdefault("selected", torch.empty(T, k, dtype=torch.int64, device=dev))
    o.setdefault("gates", torch.empty(T, k, dtype=x.dtype, device=dev))
    o.setdefault("gates_f32", torch.empty(T, k, dtype=torch.float32, device=dev))
    o.setdefault("counts", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("prob_sum", torch.empty(E, dtype=torch.float32, device=dev))
    if want_logits:
        o.setdefault("logits", torch.empty(T, E, dtype=torch.float32, device=dev))
    if want_z_loss:
        o.setdefault("z_loss", torch.empty(1, dtype=torch.float32, device=dev))
    ws = _workspace(moe_route_workspace_size(T, D, E, dt, w_router is not None, layout), dev, workspace)
    bias = None if logit_bias is None else logit_bias.to(torch.float32).contiguous()
    sb = None if selection_bias is None else selection_bias.to(torch.float32).contiguous()
    rc = lib().moe_route_ex(_p(x), dt, T, D, _rowstride(x), _p(w_router), ROUTER_LAYOUT[layout], E, _p(bias), k,
                            SCORING[scoring], _p(sb), _p(o.get("logits")), _p(o["selected"]), _p(o["gates"]),
                            _p(o["gates_f32"]), _p(o["counts"]), _p(o["prob_sum"]), _p(o.get("z_loss")),
                            _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_route_ex", rc)
    return o


def moe_renormalize_kept_gates(gates_f32: torch.Tensor, slot: torch.Tensor, stream=None) -> torch.Tensor:
    """Kept gates divided by their per-token sum; dropped assignments and fully dropped tokens get 0."""
    T, k = gates_f32.shape
    out = torch.empty_like(gates_f32)
    rc = lib().moe_renormalize_kept_gates(_p(gates_f32.contiguous()), _p(slot.contiguous()), T, k, _p(out),
                                          _stream(stream))
    _check("moe_renormalize_kept_gates", rc)
    return out


def moe_dispatch_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_dispatch_workspace_size(T, k, E))


def moe_dispatch(selected: torch.Tensor, E: int, C: int, x: Optional[torch.Tensor] = None,
                 out: Optional[dict] = None, dev_status: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Greedy position-priority slots (+ gather of x into xbuf (E, C, D) when x is given)."""
    dev = _dev(selected)
    if selected.dtype != torch.int64:
        raise TypeError("selected must be int64")
    sel = selected.reshape(selected.shape[0], -1).contiguous()
    T, k = sel.shape
    o = dict(out or {})
    o.setdefault("slot", torch.empty(T, k, dtype=torch.int64, device=dev))
    o.setdefault("kept", torch.empty(T, k, dtype=torch.uint8, device=dev))
    o.setdefault("used", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("overflow", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("drops", torch.empty(T, dtype=torch.int32, device=dev))
    o.setdefault("token_of_slot", torch.empty(E, max(C, 0), dtype=torch.int32, device=dev))
    dt, D, ldx = MOE_F32, 0, 0
    if x is not None:
        dt, D, ldx = _dt(x), x.shape[1], _rowstride(x)
        o.setdefault("xbuf", torch.empty(E, C, D, dtype=x.dtype, device=dev))
    ws = _workspace(moe_dispatch_workspace_size(T, k, E), dev, workspace)
    rc = lib().moe_dispatch(_p(sel), T, k, E, C, _p(x), dt, D, ldx, _p(o["slot"]), _p(o["kept"]), _p(o["used"]),
                            _p(o["overflow"]), _p(o["drops"]), _p(o["token_of_slot"]), _p(o.get("xbuf")),
                            _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_dispatch", rc)
    return o


def moe_dispatch_static(selected: torch.Tensor, E: int, C: int, x: Optional[torch.Tensor] = None,
                        out: Optional[dict] = None, dev_status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """moe_dispatch without a workspace: the scan state is a fixed device array in the library.

    For callers that may not allocate device memory; the outputs here are still
    allocated by PyTorch when ``out`` does not provide them.
    """
    dev = _dev(selected)
    if selected.dtype != torch.int64:
        raise TypeError("selected must be int64")
    sel = selected.reshape(selected.shape[0], -1).contiguous()
    T, k = sel.shape
    o = dict(out or {})
    o.setdefault("slot", torch.empty(T, k, dtype=torch.int64, device=dev))
    o.setdefault("kept", torch.empty(T, k, dtype=torch.uint8, device=dev))
    o.setdefault("used", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("overflow", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("drops", torch.empty(T, dtype=torch.int32, device=dev))
    o.setdefault("token_of_slot", torch.empty(E, max(C, 0), dtype=torch.int32, device=dev))
    dt, D, ldx = MOE_F32, 0, 0
    if x is not None:
        dt, D, ldx = _dt(x), x.shape[1], _rowstride(x)
        o.setdefault("xbuf", torch.empty(E, C, D, dtype=x.dtype, device=dev))
    rc = lib().moe_dispatch_static(_p(sel), T, k, E, C, _p(x), dt, D, ldx, _p(o["slot"]), _p(o["kept"]),
                                   _p(o["used"]), _p(o["overflow"]), _p(o["drops"]), _p(o["token_of_slot"]),
                                   _p(o.get("xbuf")), _p(dev_status), _stream(stream))
    _check("moe_dispatch_static", rc)
    return o


def moe_expert_ffn_workspace_size(kind: str, dtype: int, E: int, C: int, D: int, F: int, Dout: int) -> int:
    return int(lib().moe_expert_ffn_workspace_size(FFN[kind], dtype, E, C, D, F, Dout))


def moe_expert_ffn(kind: str, xbuf: torch.Tensor, used: Optional[torch.Tensor], w1: torch.Tensor,
                   b1: Optional[torch.Tensor] = None, w2: Optional[torch.Tensor] = None,
                   b2: Optional[torch.Tensor] = None, w3: Optional[torch.Tensor] = None,
                   ybuf: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Grouped expert FFN over an expert-major buffer xbuf (E, C, D); weights in (out, in) layout."""
    dev = _dev(xbuf)
    dt = _dt(xbuf)
    E, C, D = xbuf.shape
    if kind == "linear":
        F, Dout = 0, w1.shape[1]
    else:
        F, Dout = w1.shape[1], w2.shape[1]
    for w in (w1, b1, w2, b2, w3):
        if w is not None and (w.dtype != xbuf.dtype or not w.is_contiguous()):
            raise TypeError("weights must be contiguous and share xbuf's dtype")
    if not xbuf.is_contiguous():
        raise ValueError("xbuf must be contiguous")
    if ybuf is None:
        ybuf = torch.empty(E, C, Dout, dtype=xbuf.dtype, device=dev)
    ws = _workspace(moe_expert_ffn_workspace_size(kind, dt, E, C, D, max(F, 1), Dout), dev, workspace)
    rc = lib().moe_expert_ffn(FFN[kind], dt, _p(xbuf), _p(used), E, C, D, F, Dout, _p(w1), _p(b1), _p(w2), _p(b2),
                              _p(w3), _p(ybuf), _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_expert_ffn", rc)
    return ybuf


def moe_expert_ffn_gathered(x: torch.Tensor, token_of_slot: torch.Tensor, used: torch.Tensor, w_gate: torch.Tensor,
                            w_down: torch.Tensor, w_up: torch.Tensor, ybuf: Optional[torch.Tensor] = None,
                            dev_status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """SwiGLU experts on the rows token_of_slot picks from x (no expert-major copy of x), bf16.

    x (T, D); token_of_slot (E, C) int32 and used (E) int32 from moe_dispatch;
    w_gate/w_up (E, F, D), w_down (E, Dout, F).  Returns ybuf (E, C, Dout).
    """
    dev = _dev(x)
    dt = _dt(x)
    T, D = x.shape
    E, C = token_of_slot.shape
    F, Dout = w_gate.shape[1], w_down.shape[1]
    for w in (w_gate, w_up, w_down):
        if w.dtype != x.dtype or not w.is_contiguous():
            raise TypeError("weights must be contiguous and share x's dtype")
    if token_of_slot.dtype != torch.int32 or used.dtype != torch.int32:
        raise TypeError("token_of_slot and used must be int32")
    if ybuf is None:
        ybuf = torch.empty(E, C, Dout, dtype=x.dtype, device=dev)
    ws = _workspace(moe_expert_ffn_workspace_size("swiglu", dt, E, C, D, F, Dout), dev, workspace)
    rc = lib().moe_expert_ffn_gathered(FFN["swiglu"], dt, _p(x), T, _rowstride(x), _p(token_of_slot.contiguous()),
                                       _p(used), E, C, D, F, Dout, _p(w_gate), _p(w_down), _p(w_up), _p(ybuf),
                                       _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_expert_ffn_gathered", rc)
    return ybuf


def moe_expert_ffn_save(xbuf: torch.Tensor, used: torch.Tensor, w_gate: torch.Tensor, w_down: torch.Tensor,
                        w_up: torch.Tensor, saved_ab: Optional[torch.Tensor] = None, ybuf: Optional[torch.Tensor] = None,
                        dev_status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream=None):
    """bf16 SwiGLU experts that also keep the gate/up pre-activations [a | b] (E, C, 2F) for the backward.

    Returns (ybuf, saved_ab).
    """
    dev = _dev(xbuf)
    E, C, D = xbuf.shape
    F, Dout = w_gate.shape[1], w_down.shape[1]
    if ybuf is None:
        ybuf = torch.empty(E, C, Dout, dtype=xbuf.dtype, device=dev)
    if saved_ab is None:
        saved_ab = torch.empty(E, C, 2 * F, dtype=xbuf.dtype, device=dev)
    ws = _workspace(moe_expert_ffn_workspace_size("swiglu", MOE_BF16, E, C, D, F, Dout), dev, workspace)
    rc = lib().moe_expert_ffn_save(_p(xbuf), _p(used), E, C, D, F, Dout, _p(w_gate), _p(w_down), _p(w_up), _p(ybuf),
                                   _p(saved_ab), _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_expert_ffn_save", rc)
    return ybuf, saved_ab


def moe_combine(ybuf: torch.Tensor, selected: torch.Tensor, slot: torch.Tensor, gates: Optional[torch.Tensor],
                base_kind: str = "zero", base: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = base + sum over kept assignments of gate * ybuf[e, slot] (fixed j order, fp32 accumulation)."""
    dev = _dev(ybuf)
    dt = _dt(ybuf)
    E, C, N = ybuf.shape
    sel = selected.reshape(selected.shape[0], -1).contiguous()
    T, k = sel.shape
    sl = slot.reshape(T, k).contiguous()
    g = None if gates is None else gates.reshape(T, k).contiguous()
    gdt = MOE_F32 if g is None else _dt(g)
    if y is None:
        y = torch.empty(T, N, dtype=ybuf.dtype, device=dev)
    ldb = _rowstride(base) if base is not None else 0
    rc = lib().moe_combine(_p(ybuf), _p(sel), _p(sl), _p(g), gdt, T, k, E, C, N, BASE[base_kind], _p(base), ldb,
                           _p(y), _rowstride(y), dt, _p(dev_status), _stream(stream))
    _check("moe_combine", rc)
    return y


def moe_aux_stats(counts: torch.Tensor, prob_sum: torch.Tensor, T: int, k: int, normalize_by_k: bool = True,
                  aux_coef: float = 0.0, out_dtype=torch.float32, stream=None):
    """(f, P, aux) with aux = tensor([aux, aux_coef * aux])."""
    dev = _dev(counts)
    E = counts.shape[0]
    f = torch.empty(E, dtype=out_dtype, device=dev)
    P = torch.empty(E, dtype=out_dtype, device=dev)
    aux = torch.empty(2, dtype=torch.float32, device=dev)
    rc = lib().moe_aux_stats(_p(counts), _p(prob_sum), T, E, k, int(bool(normalize_by_k)), float(aux_coef), _p(f),
                             _p(P), MOE_BF16 if out_dtype == torch.bfloat16 else MOE_F32, _p(aux), _stream(stream))
    _check("moe_aux_stats", rc)
    return f, P, aux


def moe_backward_workspace_size(E: int, C: int, D: int, Dout: int) -> int:
    return int(lib().moe_backward_workspace_size(E, C, D, Dout))


def moe_backward(dy, x, logits, selected, gates_f32, slot, used, token_of_slot, xbuf, ybuf, W, C: int,
                 use_residual: bool = True, aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None,
                 dev_status=None, workspace=None, stream=None):
    """Backward of the fp32 linear-expert layer.  Returns (dx, dW, dlogits, dgate)."""
    dev = _dev(dy)
    T, Dout = dy.shape
    E, _, D = xbuf.shape
    k = selected.shape[1]
    dx = torch.empty(T, D, dtype=dy.dtype, device=dev)
    dW = torch.empty(E, Dout, D, dtype=dy.dtype, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)
    dg = torch.empty(T, k, dtype=torch.float32, device=dev)
    ws = _workspace(moe_backward_workspace_size(E, C, D, Dout), dev, workspace)
    rc = lib().moe_backward(FFN["linear"], _dt(dy), _p(dy), _p(x), _p(logits), _p(selected), _p(gates_f32), _p(slot),
                            _p(used), _p(token_of_slot), _p(xbuf), _p(ybuf), _p(W), T, k, E, C, D, Dout,
                            int(bool(use_residual)), float(aux_coef), int(bool(normalize_by_k)), _p(counts), _p(dx),
                            _p(dW), _p(dl), _p(dg), _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_backward", rc)
    return dx, dW, dl, dg


def moe_router_backward(x: torch.Tensor, w_router: torch.Tensor, dlogits: torch.Tensor, layout: str = "ED",
                        dev_status=None, workspace=None, stream=None):
    """Gradients of s = x W (+ b) for dL/ds: returns (dx_router fp32 (T,D), dw_router fp32 in W's layout, db fp32 (E))."""
    dev = _dev(x)
    T, D = x.shape
    E = dlogits.shape[1]
    if w_router.dtype != x.dtype:
        raise TypeError("w_router must have x's dtype")
    dx = torch.empty(T, D, dtype=torch.float32, device=dev)
    dw = torch.empty(tuple(w_router.shape), dtype=torch.float32, device=dev)
    db = torch.empty(E, dtype=torch.float32, device=dev)
    dt = _dt(x)
    ws = _workspace(int(lib().moe_router_backward_workspace_size(T, D, E, dt, ROUTER_LAYOUT[layout])), dev, workspace)
    rc = lib().moe_router_backward(dt, _p(x), T, D, _rowstride(x), _p(w_router.contiguous()), ROUTER_LAYOUT[layout], E,
                                   _p(dlogits.to(torch.float32).contiguous()), _p(dx), _p(dw), _p(db),
                                   _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_router_backward", rc)
    return dx, dw, db


def moe_backward_swiglu_workspace_size(E: int, C: int, H: int, F: int) -> int:
    return int(lib().moe_backward_swiglu_workspace_size(E, C, H, F))


def moe_backward_swiglu(dy, logits, selected, gates_f32, slot, used, xbuf, ybuf, w_gate, w_up, w_down, C: int,
                        use_residual: bool = False, aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None,
                        dev_status=None, workspace=None, stream=None, saved_ab=None):
    """Backward of the bf16 SwiGLU-expert layer.

    Returns (dx bf16 (T,H), dw_gate fp32 (E,F,H), dw_up fp32 (E,F,H), dw_down fp32 (E,H,F),
    dlogits fp32 (T,E), dgate fp32 (T,k)).
    """
    dev = _dev(dy)
    T, H = dy.shape
    E, F = w_gate.shape[0], w_gate.shape[1]
    k = selected.shape[1]
    dx = torch.empty(T, H, dtype=dy.dtype, device=dev)
    dwg = torch.empty(E, F, H, dtype=torch.float32, device=dev)
    dwu = torch.empty(E, F, H, dtype=torch.float32, device=dev)
    dwd = torch.empty(E, H, F, dtype=torch.float32, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)
    dg = torch.empty(T, k, dtype=torch.float32, device=dev)
    ws = _workspace(moe_backward_swiglu_workspace_size(E, C, H, F), dev, workspace)
    rc = lib().moe_backward_swiglu(_dt(dy), _p(dy), _p(logits), _p(selected), _p(gates_f32), _p(slot), _p(used),
                                   _p(xbuf), _p(ybuf), _p(saved_ab), _p(w_gate), _p(w_up), _p(w_down), T, k, E, C, H, F,
                                   int(bool(use_residual)), float(aux_coef), int(bool(normalize_by_k)), _p(counts),
                                   _p(dx), _p(dwg), _p(dwu), _p(dwd), _p(dl), _p(dg), _p(dev_status), _p(ws),
                                   ws.numel(), _stream(stream))
    _check("moe_backward_swiglu", rc)
    return dx, dwg, dwu, dwd, dl, dg


def moe_backward_gelu_workspace_size(E: int, C: int, D: int, F: int, Dout: int) -> int:
    return int(lib().moe_backward_gelu_workspace_size(E, C, D, F, Dout))


def moe_backward_gelu(dy, logits, selected, gates_f32, slot, used, xbuf, ybuf, w1, b1, w2, C: int,
                      use_residual: bool = False, aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None,
                      dev_status=None, workspace=None, stream=None):
    """Backward of the fp32 GELU-MLP-expert layer (weights in the (out, in) layout:
    w1 (E,F,D), b1 (E,F), w2 (E,Dout,F)).

    Returns (dx (T,D), dw1 (E,F,D), db1 (E,F), dw2 (E,Dout,F), db2 (E,Dout),
    dlogits (T,E), dgate (T,k)), all fp32.
    """
    dev = _dev(dy)
    T, Dout = dy.shape
    E, F, D = w1.shape
    k = selected.shape[1]
    dx = torch.empty(T, D, dtype=torch.float32, device=dev)
    dw1 = torch.empty(E, F, D, dtype=torch.float32, device=dev)
    db1 = torch.empty(E, F, dtype=torch.float32, device=dev)
    dw2 = torch.empty(E, Dout, F, dtype=torch.float32, device=dev)
    db2 = torch.empty(E, Dout, dtype=torch.float32, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)
    dg = torch.empty(T, k, dtype=torch.float32, device=dev)
    ws = _workspace(moe_backward_gelu_workspace_size(E, C, D, F, Dout), dev, workspace)
    rc = lib().moe_backward_gelu(_dt(dy), _p(dy), _p(logits), _p(selected), _p(gates_f32), _p(slot), _p(used),
                                 _p(xbuf), _p(ybuf), _p(w1), _p(b1), _p(w2), T, k, E, C, D, F, Dout,
                                 int(bool(use_residual)), float(aux_coef), int(bool(normalize_by_k)), _p(counts),
                                 _p(dx), _p(dw1), _p(db1), _p(dw2), _p(db2), _p(dl), _p(dg), _p(dev_status),
                                 _p(ws), ws.numel(), _stream(stream))
    _check("moe_backward_gelu", rc)
    return dx, dw1, db1, dw2, db2, dl, dg


def _ptr_table(bufs):
    """Host array of device pointers from tensors or integer addresses."""
    addrs = [b.data_ptr() if isinstance(b, torch.Tensor) else int(b) for b in bufs]
    return (ctypes.c_void_p * len(addrs))(*addrs), len(addrs)


def moe_ep_plan(counts_all: torch.Tensor, rank: int, C: int, out: Optional[dict] = None, stream=None) -> dict:
    """This rank's per-expert slot base and the global used/overflow/counts from every rank's counts (R, E)."""
    dev = _dev(counts_all)
    R, E = counts_all.shape
    ca = counts_all.to(torch.int32).contiguous()
    o = dict(out or {})
    for key in ("rank_base", "used", "overflow", "counts_total"):
        o.setdefault(key, torch.empty(E, dtype=torch.int32, device=dev))
    rc = lib().moe_ep_plan(_p(ca), R, rank, E, C, _p(o["rank_base"]), _p(o["used"]), _p(o["overflow"]),
                           _p(o["counts_total"]), _stream(stream))
    _check("moe_ep_plan", rc)
    return o


def moe_ep_dispatch(selected: torch.Tensor, E: int, C: int, rank_base: torch.Tensor, token_base: int,
                    x: Optional[torch.Tensor], xbuf_ranks, out: Optional[dict] = None,
                    dev_status: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> dict:
    """Slots from this rank's base and the rows written into the owner ranks' buffers (list, one per rank)."""
    dev = _dev(selected)
    if selected.dtype != torch.int64:
        raise TypeError("selected must be int64")
    sel = selected.reshape(selected.shape[0], -1).contiguous()
    T, k = sel.shape
    o = dict(out or {})
    o.setdefault("slot", torch.empty(T, k, dtype=torch.int64, device=dev))
    o.setdefault("kept", torch.empty(T, k, dtype=torch.uint8, device=dev))
    o.setdefault("drops", torch.empty(T, dtype=torch.int32, device=dev))
    o.setdefault("token_of_slot", torch.empty(E, max(C, 0), dtype=torch.int32, device=dev))
    dt, D, ldx = MOE_F32, 0, 0
    if x is not None:
        dt, D, ldx = _dt(x), x.shape[1], _rowstride(x)
    tab, R = _ptr_table(xbuf_ranks)
    ws = _workspace(moe_dispatch_workspace_size(T, k, E), dev, workspace)
    rc = lib().moe_ep_dispatch(_p(sel), T, k, E, C, _p(rank_base), int(token_base), _p(x), dt, D, ldx, tab, R,
                               _p(o["slot"]), _p(o["kept"]), _p(o["drops"]), _p(o["token_of_slot"]),
                               _p(dev_status), _p(ws), ws.numel(), _stream(stream))
    _check("moe_ep_dispatch", rc)
    return o


def moe_ep_combine(ybuf_ranks, selected: torch.Tensor, slot: torch.Tensor, gates: Optional[torch.Tensor], E: int,
                   C: int, N: int, dtype: torch.dtype, base_kind: str = "zero", base: Optional[torch.Tensor] = None,
                   y: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """moe_combine reading every kept row from its owner rank's output buffer (list, one per rank)."""
    dev = _dev(selected)
    sel = selected.reshape(selected.shape[0], -1).contiguous()
    T, k = sel.shape
    sl = slot.reshape(T, k).contiguous()
    g = None if gates is None else gates.reshape(T, k).contiguous()
    gdt = MOE_F32 if g is None else _dt(g)
    if y is None:
        y = torch.empty(T, N, dtype=dtype, device=dev)
    tab, R = _ptr_table(ybuf_ranks)
    ldb = _rowstride(base) if base is not None else 0
    rc = lib().moe_ep_combine(tab, R, _p(sel), _p(sl), _p(g), gdt, T, k, E, C, N, BASE[base_kind], _p(base), ldb,
                              _p(y), _rowstride(y), _dt(y), _p(dev_status), _stream(stream))
    _check("moe_ep_combine", rc)
    return y


def moe_ipc_export(t: torch.Tensor):
    """(handle bytes, byte offset) of the device allocation holding ``t``."""
    h = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = _i64(0)
    _check("moe_ipc_export", lib().moe_ipc_export(_p(t), h, ctypes.byref(off)))
    return h.raw, int(off.value)


def moe_ipc_import(handle: bytes) -> int:
    """Maps another process's allocation; returns the mapping's device address."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be %d bytes" % IPC_HANDLE_BYTES)
    m = _vp(0)
    _check("moe_ipc_import", lib().moe_ipc_import(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES),
                                                  ctypes.byref(m)))
    return int(m.value)


def moe_ipc_close(mapping: int):
    _check("moe_ipc_close", lib().moe_ipc_close(_vp(mapping)))


def moe_transpose_weights(src: torch.Tensor, stream=None) -> torch.Tensor:
    """(E, K_in, N_out) x@W matrices -> (E, N_out, K_in) (out, in) layout."""
    E, K, N = src.shape
    dst = torch.empty(E, N, K, dtype=src.dtype, device=src.device)
    rc = lib().moe_transpose_weights(_p(src.contiguous()), _p(dst), E, K, N, _dt(src), _stream(stream))
    _check("moe_transpose_weights", rc)
    return dst


def moe_swiglu_layer_workspace_size(desc: SwiGLULayerDesc) -> int:
    return int(lib().moe_swiglu_layer_workspace_size(ctypes.byref(desc)))


def moe_swiglu_layer_forward(desc: SwiGLULayerDesc, x: torch.Tensor, y: torch.Tensor, aux: Optional[torch.Tensor],
                             workspace: torch.Tensor, dev_status: Optional[torch.Tensor] = None, stream=None,
                             side_stream=None, copy_in_stream=None, copy_out_stream=None,
                             x_free: Optional[torch.cuda.Event] = None, y_free: Optional[torch.cuda.Event] = None):
    """The whole SwiGLU layer forward in one C call; x, y and aux may be host (pinned) or device tensors."""
    if x.dtype != torch.bfloat16 or y.dtype != torch.bfloat16 or not x.is_contiguous() or not y.is_contiguous():
        raise TypeError("x and y must be contiguous bf16")
    if tuple(x.shape) != (desc.T, desc.H) or tuple(y.shape) != (desc.T, desc.H):
        raise ValueError("x and y must be (T, H)")
    if aux is not None and (aux.dtype != torch.float32 or aux.numel() < 2):
        raise TypeError("aux must hold two fp32 values")
    nbytes = workspace.numel() * workspace.element_size()

    def st(s):
        return None if s is None else ctypes.c_void_p(s.cuda_stream)

    def ev(e):
        if e is None:
            return None
        if not e.cuda_event:  # PyTorch creates the CUDA event at its first record
            e.record()
        return ctypes.c_void_p(e.cuda_event)

    rc = lib().moe_swiglu_layer_forward(ctypes.byref(desc), _p(x), _p(y), _p(aux), _p(dev_status), _p(workspace),
                                        nbytes, _stream(stream), st(side_stream), st(copy_in_stream),
                                        st(copy_out_stream), ev(x_free), ev(y_free))
    _check("moe_swiglu_layer_forward", rc)
    return y


def moe_wait_probe(flag: torch.Tensor, limit_ns: int, dev_status: torch.Tensor, stream=None):
    """Bounded device wait on ``flag`` (int32, device): MOE_ERR_TIMEOUT in dev_status after limit_ns."""
    _check("moe_wait_probe", lib().moe_wait_probe(_p(flag), int(limit_ns), _p(dev_status), _stream(stream)))


def moe_clear_status(dev_status: torch.Tensor, stream=None):
    _check("moe_clear_status", lib().moe_clear_status(_p(dev_status), _stream(stream)))


def moe_read_status(dev_status: torch.Tensor, stream=None) -> int:
    h = _i32(0)
    _check("moe_read_status", lib().moe_read_status(_p(dev_status), _stream(stream), ctypes.byref(h)))
    return int(h.value)
