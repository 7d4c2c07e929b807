"""ctypes wrapper around the plain f64 CPU oracle (oracle/coli_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does.  It
shares no code with the CUDA library.  Inputs are the stored values (fp32 or
bf16 activations, fp32 router weights and bias, packed int4 bytes, fp32
scales); activations are widened to f64 exactly before the call.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_dbl = ctypes.c_double
_ptr = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.coli_oracle_weight.restype = _dbl
        L.coli_oracle_weight.argtypes = [_ptr, _ptr, _i64, _i64, _i64]
        L.coli_oracle_dequant.restype = ctypes.c_int
        L.coli_oracle_dequant.argtypes = [_ptr, _ptr, _i64, _i64, _ptr]
        L.coli_oracle_matvec.restype = ctypes.c_int
        L.coli_oracle_matvec.argtypes = [_ptr, _ptr, _i64, _i64, _ptr, _ptr]
        L.coli_oracle_route.restype = ctypes.c_int
        L.coli_oracle_route.argtypes = [_ptr, _i64, _i64, _ptr, _ptr, _i64, _i64, _dbl,
                                        _ptr, _ptr, _ptr, _ptr, _ptr]
        L.coli_oracle_union.restype = ctypes.c_int
        L.coli_oracle_union.argtypes = [_ptr, _i64, _i64, _i64] + [_ptr] * 6
        L.coli_oracle_expert_ffn.restype = ctypes.c_int
        L.coli_oracle_expert_ffn.argtypes = [_ptr, _i64, _i64] + [_ptr] * 8
        L.coli_oracle_moe_layer.restype = ctypes.c_int
        L.coli_oracle_moe_layer.argtypes = [_ptr, _i64, _i64, _i64, _i64, _i64, _dbl,
                                            _ptr, _ptr] + [_ptr] * 6 + [_ptr, _ptr, _ptr]
        L.coli_oracle_route_top_p.restype = ctypes.c_int
        L.coli_oracle_route_top_p.argtypes = [_ptr, _i64, _i64, _ptr, _ptr, _i64, _i64, _dbl, _dbl, _ptr, _ptr]
        L.coli_oracle_moe_layer_top_p.restype = ctypes.c_int
        L.coli_oracle_moe_layer_top_p.argtypes = [_ptr, _i64, _i64, _i64, _i64, _i64, _dbl, _dbl,
                                                  _ptr, _ptr] + [_ptr] * 6 + [_ptr, _ptr, _ptr]
        L.coli_oracle_quant_i8.restype = ctypes.c_int
        L.coli_oracle_quant_i8.argtypes = [_ptr, _i64, _ptr, _ptr]
        L.coli_oracle_moe_layer_i8.restype = ctypes.c_int
        L.coli_oracle_moe_layer_i8.argtypes = [_ptr, _i64, _i64, _i64, _i64, _i64, _dbl,
                                               _ptr, _ptr] + [_ptr] * 6 + [_ptr, _ptr, _ptr]
        L.coli_oracle_threads.restype = ctypes.c_int
        L.coli_oracle_threads.argtypes = []
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def widen(x):
    """Exact f64 copy of stored activations (fp32 array, or bf16 given as uint16 bits)."""
    x = np.asarray(x)
    if x.dtype == np.uint16:  # bf16 bit patterns
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def threads():
    return lib().coli_oracle_threads()


def dequant(q, s, N, K):
    q = _c(q, np.uint8); s = _c(s, np.float32)
    W = np.empty((N, K), np.float64)
    _check(lib().coli_oracle_dequant(_p(q), _p(s), N, K, _p(W)), "dequant")
    return W


def weight(q, s, K, n, kk):
    q = _c(q, np.uint8); s = _c(s, np.float32)
    return lib().coli_oracle_weight(_p(q), _p(s), K, n, kk)


def matvec(q, s, N, K, x):
    q = _c(q, np.uint8); s = _c(s, np.float32); x = _c(x, np.float64)
    y = np.empty(N, np.float64)
    _check(lib().coli_oracle_matvec(_p(q), _p(s), N, K, _p(x), _p(y)), "matvec")
    return y


def route(x, w_router, sel_bias, k, routed_scale, want_scores=False):
    """Return (idx int32 [T,k], w f64 [T,k]) and, if asked, (logits, sig, biased) [T,E]."""
    x = _c(widen(x), np.float64)
    T, H = x.shape
    w_router = _c(w_router, np.float32); sel_bias = _c(sel_bias, np.float32)
    E = w_router.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    l = s = c = None
    if want_scores:
        l = np.empty((T, E)); s = np.empty((T, E)); c = np.empty((T, E))
    _check(lib().coli_oracle_route(_p(x), T, H, _p(w_router), _p(sel_bias), E, k,
                                   float(routed_scale), _p(idx), _p(w), _p(l), _p(s), _p(c)),
           "route")
    if want_scores:
        return idx, w, (l, s, c)
    return idx, w


def route_top_p(x, w_router, sel_bias, k, routed_scale, top_p):
    """Top-k routing cut by adaptive expert top-p: (idx int32 [T,k], w f64 [T,k]);
    dropped slots have index -1 and weight 0."""
    x = _c(widen(x), np.float64)
    T, H = x.shape
    w_router = _c(w_router, np.float32); sel_bias = _c(sel_bias, np.float32)
    E = w_router.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _check(lib().coli_oracle_route_top_p(_p(x), T, H, _p(w_router), _p(sel_bias), E, k, float(routed_scale),
                                         float(top_p), _p(idx), _p(w)), "route_top_p")
    return idx, w


def union(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    P = T * k
    count = np.empty(E, np.int32)
    offset = np.empty(E + 1, np.int32)
    active = np.empty(E, np.int32)
    n_active = np.empty(1, np.int32)
    perm = np.empty(P, np.int32)
    inv_perm = np.empty(P, np.int32)
    _check(lib().coli_oracle_union(_p(idx), T, k, E, _p(count), _p(offset), _p(active),
                                   _p(n_active), _p(perm), _p(inv_perm)), "union")
    return dict(count=count, offset=offset, active=active, n_active=int(n_active[0]),
                perm=perm, inv_perm=inv_perm)


def expert_ffn(x, H, F, expert, want_h=False):
    """expert: dict with gate_q, gate_s, up_q, up_s, down_q, down_s arrays of one expert."""
    x = _c(widen(x), np.float64)
    arrs = [_c(expert[n], np.uint8 if n.endswith("_q") else np.float32)
            for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")]
    y = np.empty(H, np.float64)
    h = np.empty(F, np.float64) if want_h else None
    _check(lib().coli_oracle_expert_ffn(_p(x), H, F, *[_p(a) for a in arrs], _p(y), _p(h)),
           "expert_ffn")
    return (y, h) if want_h else y


def _expert_tables(experts, E):
    names = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")
    keep, tables = [], []
    for n in names:
        arr = (ctypes.c_void_p * (E + 1))()
        for e in range(E + 1):
            if e in experts:
                a = _c(experts[e][n], np.uint8 if n.endswith("_q") else np.float32)
                keep.append(a)
                arr[e] = a.ctypes.data
            else:
                arr[e] = None
        tables.append(arr)
    return keep, tables


def moe_layer_top_p(x, H, F, E, k, routed_scale, top_p, w_router, sel_bias, experts):
    """The layer with top-p routing.  Returns (idx, w, out [T,H] f64); dropped
    slots have index -1 and weight 0."""
    x = _c(widen(x), np.float64)
    T = x.shape[0]
    w_router = _c(w_router, np.float32); sel_bias = _c(sel_bias, np.float32)
    keep, tables = _expert_tables(experts, E)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    out = np.empty((T, H), np.float64)
    _check(lib().coli_oracle_moe_layer_top_p(_p(x), T, H, F, E, k, float(routed_scale), float(top_p),
                                             _p(w_router), _p(sel_bias),
                                             *[ctypes.cast(t, ctypes.c_void_p) for t in tables],
                                             _p(idx), _p(w), _p(out)), "moe_layer_top_p")
    del keep
    return idx, w, out


def moe_layer(x, H, F, E, k, routed_scale, w_router, sel_bias, experts):
    """experts: mapping expert index (0..E, E = shared) -> dict of the six arrays.
    Experts no token selects may be missing.  Returns (idx, w, out [T,H] f64)."""
    x = _c(widen(x), np.float64)
    T = x.shape[0]
    w_router = _c(w_router, np.float32); sel_bias = _c(sel_bias, np.float32)
    names = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")
    keep = []
    tables = []
    for n in names:
        arr = (ctypes.c_void_p * (E + 1))()
        for e in range(E + 1):
            if e in experts:
                a = _c(experts[e][n], np.uint8 if n.endswith("_q") else np.float32)
                keep.append(a)
                arr[e] = a.ctypes.data
            else:
                arr[e] = None
        tables.append(arr)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    out = np.empty((T, H), np.float64)
    _check(lib().coli_oracle_moe_layer(_p(x), T, H, F, E, k, float(routed_scale),
                                       _p(w_router), _p(sel_bias),
                                       *[ctypes.cast(t, ctypes.c_void_p) for t in tables],
                                       _p(idx), _p(w), _p(out)), "moe_layer")
    return idx, w, out


def quant_i8(x):
    """Integer-activation codes of fp32 values x [..., n] (n a multiple of 32):
    (codes int8 [..., n], scales fp32 [..., n / 32])."""
    x = _c(x, np.float32)
    n = x.shape[-1]
    codes = np.empty(x.shape, np.int8)
    scales = np.empty(x.shape[:-1] + (n // 32,), np.float32)
    _check(lib().coli_oracle_quant_i8(_p(x), x.size, _p(codes), _p(scales)), "quant_i8")
    return codes, scales


def moe_layer_i8(x, H, F, E, k, routed_scale, w_router, sel_bias, experts):
    """The layer with int8 activations into every expert product.  Returns
    (idx, w, out [T,H] f64)."""
    x = _c(widen(x), np.float64)
    T = x.shape[0]
    w_router = _c(w_router, np.float32); sel_bias = _c(sel_bias, np.float32)
    keep, tables = _expert_tables(experts, E)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    out = np.empty((T, H), np.float64)
    _check(lib().coli_oracle_moe_layer_i8(_p(x), T, H, F, E, k, float(routed_scale),
                                          _p(w_router), _p(sel_bias),
                                          *[ctypes.cast(t, ctypes.c_void_p) for t in tables],
                                          _p(idx), _p(w), _p(out)), "moe_layer_i8")
    del keep
    return idx, w, out
