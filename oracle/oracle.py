"""Python face of the fp64 CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product package never imports this module, and this module
imports nothing from the product package.

The functions take and return numpy arrays.  Floating inputs are converted to
float64 (exact for fp32 and bf16 storage values) before the C code sees them.
Expert weights are passed in the pages' ``x @ W`` layout, shape
``(E, K_in, N_out)``.

Each function names the page passage it follows; the arithmetic itself is in
``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` into ``liboracle.so`` with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.oracle_capacity.restype = i64
        lib.oracle_capacity.argtypes = [i64, i32, i32, dbl]
        lib.oracle_router_logits.argtypes = [_D, _D, _D, i64, i64, i32, _D]
        lib.oracle_route.argtypes = [_D, i64, i32, i32, _D, _I64, _D, _I64, _D]
        lib.oracle_dispatch.restype = ctypes.c_int
        lib.oracle_dispatch.argtypes = [_I64, i64, i32, i32, i64, _I64, _U8, _I64, _I64, _I64, _I64]
        lib.oracle_layer_rows.argtypes = [ctypes.c_int, _D, i64, i64, _I64, _U8, _D, i32, _D, _D, _D,
                                          _D, _D, i64, i64, ctypes.c_int, _D, _I64, i64, _D]
        lib.oracle_expert_rows.argtypes = [ctypes.c_int, _D, i64, _I64, _I64, i64, _D, _D, _D, _D, _D,
                                           i64, i64, _D]
        lib.oracle_aux.argtypes = [_I64, _D, i64, i32, i32, ctypes.c_int, _D, _D, _D]
        lib.oracle_z_loss.restype = dbl
        lib.oracle_z_loss.argtypes = [_D, i64, i32]
        lib.oracle_backward_linear.argtypes = [_D, _D, _D, _I64, _U8, _D, _D, i64, i32, i32, i64, i64,
                                               ctypes.c_int, dbl, ctypes.c_int, _I64, _D, _D, _D, _D]
        lib.oracle_backward_swiglu.argtypes = [_D, _D, _D, _I64, _U8, _D, _D, _D, _D, i64, i32, i32, i64, i64,
                                               i64, ctypes.c_int, dbl, ctypes.c_int, _I64, _D, _D, _D, _D, _D, _D]
        lib.oracle_backward_gelu.argtypes = [_D, _D, _D, _I64, _U8, _D, _D, _D, _D, _D, i64, i32, i32, i64, i64,
                                             i64, ctypes.c_int, dbl, ctypes.c_int, _I64, _D, _D, _D, _D, _D, _D,
                                             _D]
        lib.oracle_router_backward.argtypes = [_D, _D, _D, i64, i64, i32, _D, _D, _D]
        lib.oracle_combine_precomputed.argtypes = [_D, i64, i32, i64, _I64, _U8, _D, i32, ctypes.c_int,
                                                   _D, _D]
        lib.oracle_combine_slots.argtypes = [_D, i64, i32, i64, i64, _I64, _I64, _U8, _D, i32,
                                             ctypes.c_int, _D, _D]
        lib.oracle_route_variant.argtypes = [_D, i64, i32, i32, ctypes.c_int, _D, _D, _I64, _D, _I64]
        lib.oracle_renormalize_kept.argtypes = [_D, _U8, i64, i32, _D]
        lib.oracle_dense_linear.argtypes = [_D, _I64, _I64, _U8, _D, _D, i64, i32, i32, i64, i64, i64,
                                            ctypes.c_int, _U8, _D, _D]
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def _p(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    return a.ctypes.data_as(typ)


KIND = {"linear": 0, "gelu_mlp": 1, "swiglu": 2}
BASE = {"zero": 0, "input": 1, "tensor": 2}


def capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    """``ceil(capacity_factor * T * k / E)``, floor 1 (module-7 ``expert_capacity``)."""
    c = _load().oracle_capacity(int(T), int(k), int(E), float(capacity_factor))
    if c < 0:
        raise ValueError("invalid capacity arguments")
    return int(c)


def router_logits(x, w_router, bias=None) -> np.ndarray:
    """Router scores ``s = x @ w_router (+ b)``; w_router is (D, E) as on the router page."""
    x, w = _f64(x), _f64(w_router)
    T, D = x.shape
    D2, E = w.shape
    assert D == D2
    b = None if bias is None else _f64(bias)
    s = np.empty((T, E), np.float64)
    _load().oracle_router_logits(_p(x, _D), _p(w, _D), _p(b, _D), T, D, E, _p(s, _D))
    return s


def router_backward(x, w_router, dlogits):
    """``(dx, dw_router, db)`` of ``s = x @ w_router + b`` for the gradient ``dlogits`` (w_router is (D, E))."""
    x, w, g = _f64(x), _f64(w_router), _f64(dlogits)
    T, D = x.shape
    E = w.shape[1]
    dx = np.empty((T, D), np.float64)
    dw = np.empty((D, E), np.float64)
    db = np.empty(E, np.float64)
    _load().oracle_router_backward(_p(x, _D), _p(w, _D), _p(g, _D), T, D, E, _p(dx, _D), _p(dw, _D), _p(db, _D))
    return dx, dw, db


def route(s, k: int):
    """Softmax, stable top-k, renormalised gates, pre-drop counts, probability sums.

    Returns ``(probs (T,E), selected (T,k) int64, gates (T,k), counts (E) int64,
    prob_sum (E))``.
    """
    s = _f64(s)
    T, E = s.shape
    if not (1 <= k <= E):
        raise ValueError("k must lie in [1, E]")
    if not np.all(np.isfinite(s)):
        raise ValueError("logits must be finite")
    probs = np.empty((T, E), np.float64)
    sel = np.empty((T, k), np.int64)
    gates = np.empty((T, k), np.float64)
    counts = np.empty(E, np.int64)
    psum = np.empty(E, np.float64)
    _load().oracle_route(_p(s, _D), T, E, k, _p(probs, _D), _p(sel, _I64), _p(gates, _D),
                         _p(counts, _I64), _p(psum, _D))
    return probs, sel, gates, counts, psum


SCORING = {"softmax": 0, "sigmoid": 1}


def route_variant(s, k: int, scoring: str = "sigmoid", selection_bias=None):
    """Module-7 router: softmax or sigmoid clean scores, optional selection-only bias.

    Returns ``(clean (T,E), selected (T,k), gates (T,k), counts (E))``.
    """
    s = _f64(s)
    if s.ndim == 1:
        s = s[None, :]
    T, E = s.shape
    if not (1 <= k <= E):
        raise ValueError("k must lie in [1, E]")
    if not np.all(np.isfinite(s)):
        raise ValueError("logits must be finite")
    b = None if selection_bias is None else _f64(selection_bias)
    clean = np.empty((T, E), np.float64)
    sel = np.empty((T, k), np.int64)
    gates = np.empty((T, k), np.float64)
    counts = np.empty(E, np.int64)
    _load().oracle_route_variant(_p(s, _D), T, E, k, SCORING[scoring], _p(b, _D), _p(clean, _D), _p(sel, _I64),
                                 _p(gates, _D), _p(counts, _I64))
    return clean, sel, gates, counts


def renormalize_kept(gates, kept):
    """Kept gates of each token divided by their sum; dropped (and fully dropped) rows are 0."""
    g = _f64(gates)
    T, k = g.shape
    kp = _u8(kept).reshape(T, k)
    out = np.empty((T, k), np.float64)
    _load().oracle_renormalize_kept(_p(g, _D), _p(kp, _U8), T, k, _p(out, _D))
    return out


def dispatch(selected, E: int, C: int):
    """Greedy position-priority slots.

    Returns a dict with ``slot (T,k)``, ``kept (T,k) bool``, ``used (E)``,
    ``overflow (E)``, ``drops (T)``, ``token_of_slot (E,C)`` (all int64 except
    kept) and ``bad_index`` (True when an index outside [0,E) was seen).
    """
    sel = _i64(selected)
    if sel.ndim == 1:
        sel = sel[:, None]
    T, k = sel.shape
    slot = np.empty((T, k), np.int64)
    kept = np.empty((T, k), np.uint8)
    used = np.empty(E, np.int64)
    overflow = np.empty(E, np.int64)
    drops = np.empty(T, np.int64)
    tos = np.empty((E, max(C, 0)), np.int64)
    rc = _load().oracle_dispatch(_p(sel, _I64), T, k, E, C, _p(slot, _I64), _p(kept, _U8),
                                 _p(used, _I64), _p(overflow, _I64), _p(drops, _I64),
                                 _p(tos, _I64))
    return dict(slot=slot, kept=kept.astype(bool), used=used, overflow=overflow, drops=drops,
                token_of_slot=tos, bad_index=(rc != 0))


def _weights(kind: str, w1, b1, w2, b2, w3):
    conv = [None if a is None else _f64(a) for a in (w1, b1, w2, b2, w3)]
    return conv


def layer_rows(kind: str, x, selected, kept, gates, weights: dict, base_kind: str = "zero",
               base=None, tokens=None) -> np.ndarray:
    """``y_t = base_t + sum_{j kept} gate_{t,j} Expert_{e_{t,j}}(x_t)`` for the listed tokens.

    ``weights`` holds ``w1, b1, w2, b2, w3`` in the pages' layout:
    linear ``w1 (E,D,N)``; gelu_mlp ``w1 (E,D,F), b1 (E,F), w2 (E,F,N), b2 (E,N)``;
    swiglu ``w1 = gate (E,D,F), w3 = up (E,D,F), w2 = down (E,F,N)``.
    """
    x = _f64(x)
    T, D = x.shape
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    w1, b1, w2, b2, w3 = _weights(kind, weights.get("w1"), weights.get("b1"), weights.get("w2"),
                                  weights.get("b2"), weights.get("w3"))
    if kind == "linear":
        F, N = 0, w1.shape[2]
    else:
        F, N = w1.shape[2], w2.shape[2]
    toks = np.arange(T, dtype=np.int64) if tokens is None else _i64(tokens)
    bs = None if base is None else _f64(base)
    y = np.empty((toks.shape[0], N), np.float64)
    _load().oracle_layer_rows(KIND[kind], _p(x, _D), T, D, _p(sel, _I64), _p(kp, _U8), _p(g, _D), k,
                              _p(w1, _D), _p(b1, _D), _p(w2, _D), _p(b2, _D), _p(w3, _D), F, N,
                              BASE[base_kind], _p(bs, _D), _p(toks, _I64), toks.shape[0], _p(y, _D))
    return y


def expert_rows(kind: str, x, tokens, experts, weights: dict) -> np.ndarray:
    """Expert outputs (ungated) ``Expert_{experts[i]}(x[tokens[i]])``."""
    x = _f64(x)
    T, D = x.shape
    toks, exps = _i64(tokens), _i64(experts)
    w1, b1, w2, b2, w3 = _weights(kind, weights.get("w1"), weights.get("b1"), weights.get("w2"),
                                  weights.get("b2"), weights.get("w3"))
    if kind == "linear":
        F, N = 0, w1.shape[2]
    else:
        F, N = w1.shape[2], w2.shape[2]
    out = np.empty((toks.shape[0], N), np.float64)
    _load().oracle_expert_rows(KIND[kind], _p(x, _D), D, _p(toks, _I64), _p(exps, _I64),
                               toks.shape[0], _p(w1, _D), _p(b1, _D), _p(w2, _D), _p(b2, _D),
                               _p(w3, _D), F, N, _p(out, _D))
    return out


def aux(counts, prob_sum, T: int, k: int, normalize_by_k: bool = True):
    """``(f, P, aux)`` with ``f = count/T``, ``P = prob_sum/T`` and the Switch aux loss."""
    c, ps = _i64(counts), _f64(prob_sum)
    E = c.shape[0]
    f = np.empty(E, np.float64)
    P = np.empty(E, np.float64)
    a = np.empty(1, np.float64)
    _load().oracle_aux(_p(c, _I64), _p(ps, _D), T, E, k, int(bool(normalize_by_k)), _p(f, _D),
                       _p(P, _D), _p(a, _D))
    return f, P, float(a[0])


def z_loss(s) -> float:
    """Router z-loss ``mean_t logsumexp(s_t)^2`` (module-7 ``router_z_loss``)."""
    s = _f64(s)
    return float(_load().oracle_z_loss(_p(s, _D), s.shape[0], s.shape[1]))


def backward_linear(dy, x, s, selected, kept, gates, W, use_residual: bool = True,
                    aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None):
    """Backward of the linear-expert layer with the kept mask constant.

    ``W`` is ``(E, D, N)``.  Returns ``(dx, dW, dlogits, dgate)``.
    """
    dy, x, s, W = _f64(dy), _f64(x), _f64(s), _f64(W)
    T, D = x.shape
    E = s.shape[1]
    N = W.shape[2]
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    cnt = _i64(counts if counts is not None else np.bincount(sel.ravel(), minlength=E))
    dx = np.empty((T, D), np.float64)
    dW = np.empty((E, D, N), np.float64)
    dl = np.empty((T, E), np.float64)
    dg = np.empty((T, k), np.float64)
    _load().oracle_backward_linear(_p(dy, _D), _p(x, _D), _p(s, _D), _p(sel, _I64), _p(kp, _U8),
                                   _p(g, _D), _p(W, _D), T, k, E, D, N, int(bool(use_residual)),
                                   float(aux_coef), int(bool(normalize_by_k)), _p(cnt, _I64),
                                   _p(dx, _D), _p(dW, _D), _p(dl, _D), _p(dg, _D))
    return dx, dW, dl, dg


def backward_swiglu(dy, x, s, selected, kept, gates, Wg, Wu, Wd, use_residual: bool = False,
                    aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None):
    """Backward of the SwiGLU-expert layer with the kept mask constant.

    ``Wg, Wu`` are ``(E, D, F)``, ``Wd`` is ``(E, F, N)`` (pages' x@W layout).
    Returns ``(dx, dWg, dWu, dWd, dlogits, dgate)``.
    """
    dy, x, s = _f64(dy), _f64(x), _f64(s)
    Wg, Wu, Wd = _f64(Wg), _f64(Wu), _f64(Wd)
    T, D = x.shape
    E = s.shape[1]
    F, N = Wg.shape[2], Wd.shape[2]
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    cnt = _i64(counts if counts is not None else np.bincount(sel.ravel(), minlength=E))
    dx = np.empty((T, D), np.float64)
    dWg = np.empty((E, D, F), np.float64)
    dWu = np.empty((E, D, F), np.float64)
    dWd = np.empty((E, F, N), np.float64)
    dl = np.empty((T, E), np.float64)
    dg = np.empty((T, k), np.float64)
    _load().oracle_backward_swiglu(_p(dy, _D), _p(x, _D), _p(s, _D), _p(sel, _I64), _p(kp, _U8), _p(g, _D),
                                   _p(Wg, _D), _p(Wu, _D), _p(Wd, _D), T, k, E, D, F, N,
                                   int(bool(use_residual)), float(aux_coef), int(bool(normalize_by_k)),
                                   _p(cnt, _I64), _p(dx, _D), _p(dWg, _D), _p(dWu, _D), _p(dWd, _D),
                                   _p(dl, _D), _p(dg, _D))
    return dx, dWg, dWu, dWd, dl, dg


def backward_gelu(dy, x, s, selected, kept, gates, W1, b1, W2, b2, use_residual: bool = False,
                  aux_coef: float = 0.0, normalize_by_k: bool = True, counts=None):
    """Backward of the GELU-MLP-expert layer with the kept mask constant.

    ``W1`` is ``(E, D, F)``, ``b1`` ``(E, F)``, ``W2`` ``(E, F, N)``, ``b2`` ``(E, N)``
    (pages' x@W layout).  Returns ``(dx, dW1, db1, dW2, db2, dlogits, dgate)``.
    """
    dy, x, s = _f64(dy), _f64(x), _f64(s)
    W1, b1, W2, b2 = _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    T, D = x.shape
    E = s.shape[1]
    F, N = W1.shape[2], W2.shape[2]
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    cnt = _i64(counts if counts is not None else np.bincount(sel.ravel(), minlength=E))
    dx = np.empty((T, D), np.float64)
    dW1 = np.empty((E, D, F), np.float64)
    db1 = np.empty((E, F), np.float64)
    dW2 = np.empty((E, F, N), np.float64)
    db2 = np.empty((E, N), np.float64)
    dl = np.empty((T, E), np.float64)
    dg = np.empty((T, k), np.float64)
    _load().oracle_backward_gelu(_p(dy, _D), _p(x, _D), _p(s, _D), _p(sel, _I64), _p(kp, _U8), _p(g, _D),
                                 _p(W1, _D), _p(b1, _D), _p(W2, _D), _p(b2, _D), T, k, E, D, F, N,
                                 int(bool(use_residual)), float(aux_coef), int(bool(normalize_by_k)),
                                 _p(cnt, _I64), _p(dx, _D), _p(dW1, _D), _p(db1, _D), _p(dW2, _D), _p(db2, _D),
                                 _p(dl, _D), _p(dg, _D))
    return dx, dW1, db1, dW2, db2, dl, dg


def combine_precomputed(u, selected, kept, gates, base=None) -> np.ndarray:
    """Router-page form ``y_t = base_t + sum_{j kept} alpha_{t,j} u[t, e_{t,j}]``; u is (T,E,N)."""
    u = _f64(u)
    T, E, N = u.shape
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    bs = None if base is None else _f64(base)
    y = np.empty((T, N), np.float64)
    _load().oracle_combine_precomputed(_p(u, _D), T, E, N, _p(sel, _I64), _p(kp, _U8), _p(g, _D), k,
                                       0 if bs is None else 2, _p(bs, _D), _p(y, _D))
    return y


def combine_slots(ybuf, selected, slot, kept, gates, base=None) -> np.ndarray:
    """Expert-major form: ``y_t = base_t + sum_{j kept} gate_{t,j} ybuf[e_{t,j}, slot_{t,j}]``."""
    yb = _f64(ybuf)
    E, C, N = yb.shape
    sel = _i64(selected)
    T = sel.shape[0]
    sel = sel.reshape(T, -1)
    k = sel.shape[1]
    sl = _i64(slot).reshape(T, k)
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    bs = None if base is None else _f64(base)
    y = np.empty((T, N), np.float64)
    _load().oracle_combine_slots(_p(yb, _D), T, E, C, N, _p(sel, _I64), _p(sl, _I64), _p(kp, _U8),
                                 _p(g, _D), k, 0 if bs is None else 2, _p(bs, _D), _p(y, _D))
    return y


def dense_linear(x, selected, slot, kept, gates, W, C: int, use_residual: bool = True):
    """Dense all-experts reference with explicit ``(T,E,C)`` dispatch/combine tensors.

    Returns ``(y, dispatch_mask (T,E,C) bool, combine_weights (T,E,C))``.
    """
    x, W = _f64(x), _f64(W)
    T, D = x.shape
    E, _, N = W.shape
    sel = _i64(selected).reshape(T, -1)
    k = sel.shape[1]
    sl = _i64(slot).reshape(T, k)
    kp = _u8(kept).reshape(T, k)
    g = _f64(gates).reshape(T, k)
    mask = np.empty((T, E, C), np.uint8)
    comb = np.empty((T, E, C), np.float64)
    y = np.empty((T, N), np.float64)
    _load().oracle_dense_linear(_p(x, _D), _p(sel, _I64), _p(sl, _I64), _p(kp, _U8), _p(g, _D),
                                _p(W, _D), T, k, E, C, D, N, int(bool(use_residual)), _p(mask, _U8),
                                _p(comb, _D), _p(y, _D))
    return y, mask.astype(bool), comb


def forward(kind: str, x, s, k: int, C: int, weights: dict, base_kind: str = "zero", base=None,
            tokens=None, normalize_by_k: bool = True):
    """Whole layer on given logits: route, dispatch, expert outputs, combine, aux.

    Returns a dict with every intermediate the CUDA path also produces.
    """
    s = _f64(s)
    T, E = s.shape
    probs, sel, gates, counts, psum = route(s, k)
    disp = dispatch(sel, E, C)
    y = layer_rows(kind, x, sel, disp["kept"], gates, weights, base_kind, base, tokens)
    f, P, a = aux(counts, psum, T, k, normalize_by_k)
    out = dict(probs=probs, selected=sel, gates=gates, counts=counts, prob_sum=psum, y=y, f=f, P=P,
               aux=a)
    out.update(disp)
    return out
