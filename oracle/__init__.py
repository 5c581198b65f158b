"""CPU oracle of the quantized MoE expert forward.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the package smoke
check and by the bench's CPU-baseline leg, never by the product path. The
arithmetic lives in ``oracle.c`` (plain C, double precision, naive loops);
this module only builds it, loads it and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
                               "-Wno-unused-parameter", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Mat(C.Structure):
    _fields_ = [("q", C.c_void_p), ("s", C.c_void_p), ("b", C.c_void_p)]


class _Expert(C.Structure):
    _fields_ = [("gate", _Mat), ("up", _Mat), ("down", _Mat)]


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.oracle_bf16_to_double.restype = C.c_double
        _lib.oracle_bf16_to_double.argtypes = [C.c_uint16]
        _lib.oracle_double_to_bf16.restype = C.c_uint16
        _lib.oracle_double_to_bf16.argtypes = [C.c_double]
        _lib.oracle_silu.restype = C.c_double
        _lib.oracle_silu.argtypes = [C.c_double]
        _lib.oracle_sigmoid.restype = C.c_double
        _lib.oracle_sigmoid.argtypes = [C.c_double]
        _lib.oracle_e2m1.restype = C.c_double
        _lib.oracle_e2m1.argtypes = [C.c_uint]
        _lib.oracle_e8m0.restype = C.c_double
        _lib.oracle_e8m0.argtypes = [C.c_uint]
        _lib.oracle_mx_weight.restype = C.c_double
        _lib.oracle_mx_weight.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int]
        _lib.oracle_weight.restype = C.c_double
        _lib.oracle_weight.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p] + [C.c_int] * 5
        _lib.oracle_combine_norm.argtypes = [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                             C.c_double, C.c_void_p, C.c_void_p, C.c_double,
                                             C.c_void_p, C.c_void_p, C.c_void_p]
        _lib.oracle_layer.argtypes = ([C.c_int] * 7 + [C.c_double] + [C.c_void_p] * 14)
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> int:
    return lib().oracle_set_threads(int(n))


def bf16_to_f64(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return np.array([lib().oracle_bf16_to_double(int(v)) for v in b.ravel()]).reshape(b.shape)


def f64_to_bf16(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    return np.array([lib().oracle_double_to_bf16(float(t)) for t in v.ravel()], dtype=np.uint16).reshape(v.shape)


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def sigmoid(z: float) -> float:
    return lib().oracle_sigmoid(float(z))


def dequant(q, s, b, K: int, G: int, bits: int) -> np.ndarray:
    q = _c(q, np.uint32); s = _c(s, np.uint16); b = _c(b, np.uint16)
    R = s.shape[0]
    w = np.empty((R, K), dtype=np.float64)
    rc = lib().oracle_dequant(R, K, G, bits, _p(q), _p(s), _p(b), _p(w))
    if rc:
        raise ValueError("oracle_dequant: invalid arguments")
    return w


def qgemv(q, s, b, x, K: int, G: int, bits: int) -> np.ndarray:
    q = _c(q, np.uint32); s = _c(s, np.uint16); b = _c(b, np.uint16); x = _c(x, np.float64)
    R = s.shape[0]
    y = np.empty(R, dtype=np.float64)
    rc = lib().oracle_qgemv(R, K, G, bits, _p(q), _p(s), _p(b), _p(x), _p(y))
    if rc:
        raise ValueError("oracle_qgemv: invalid arguments")
    return y


def e2m1(code: int) -> float:
    """Value of a 4-bit FP4 E2M1 code (MXFP4 element)."""
    return lib().oracle_e2m1(int(code))


def e8m0(byte: int) -> float:
    """Value of an E8M0 scale byte (MXFP4 block scale); NaN for 0xFF."""
    return lib().oracle_e8m0(int(byte))


def mx_dequant(q, e, K: int) -> np.ndarray:
    """MXFP4 matrix (codes uint32 [R][K/8], scales uint8 [R][K/32]) as double [R][K]."""
    q = _c(q, np.uint32); e = _c(e, np.uint8)
    R = e.shape[0]
    w = np.empty((R, K), dtype=np.float64)
    if lib().oracle_mx_dequant(R, K, _p(q), _p(e), _p(w)):
        raise ValueError("oracle_mx_dequant: invalid arguments")
    return w


def mx_gemv(q, e, x, K: int) -> np.ndarray:
    """y = W x for an MXFP4 matrix W, index-order double sums."""
    q = _c(q, np.uint32); e = _c(e, np.uint8); x = _c(x, np.float64)
    R = e.shape[0]
    y = np.empty(R, dtype=np.float64)
    if lib().oracle_mx_gemv(R, K, _p(q), _p(e), _p(x), _p(y)):
        raise ValueError("oracle_mx_gemv: invalid arguments")
    return y


def mx_gemm(q, e, x, K: int) -> np.ndarray:
    """Y[t] = W x[t] for every row of x (bf16 bits [T][K] or doubles): the dequantised
    matrix (double) times the activations by one library matrix product."""
    x = np.asarray(x)
    xd = bf16_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)
    return xd @ mx_dequant(q, e, K).T


def swiglu(g, u) -> np.ndarray:
    g = _c(g, np.float64); u = _c(u, np.float64)
    a = np.empty_like(g)
    lib().oracle_swiglu(len(g), _p(g), _p(u), _p(a))
    return a


def expert(ex, x, H: int, I: int, G: int, bits: int, want_a: bool = False):
    """ex = ((gq, gs, gb), (uq, us, ub), (dq, ds, db)); x float64 [H] -> y float64 [H]."""
    (gq, gs, gb), (uq, us, ub), (dq, ds, db) = [tuple(_c(a, t) for a, t in zip(m, (np.uint32, np.uint16, np.uint16))) for m in ex]
    x = _c(x, np.float64)
    y = np.empty(H, dtype=np.float64)
    a = np.empty(I, dtype=np.float64) if want_a else None
    rc = lib().oracle_expert(H, I, G, bits, _p(gq), _p(gs), _p(gb), _p(uq), _p(us), _p(ub),
                             _p(dq), _p(ds), _p(db), _p(x), _p(y), _p(a))
    if rc:
        raise ValueError("oracle_expert: invalid arguments")
    return (y, a) if want_a else y


def route(x, Wr, k: int, bias=None, gs=None, want_logits: bool = False):
    """x bf16 [T][H], Wr bf16 [E][H] -> idx int32 [T][k], w float64 [T][k], shared gate [T] (or None)."""
    x = _c(np.atleast_2d(x), np.uint16); Wr = _c(Wr, np.uint16)
    bias = _c(bias, np.float32); gs = _c(gs, np.uint16)
    T, H = x.shape
    E = Wr.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    sg = np.empty(T, dtype=np.float64) if gs is not None else None
    logits = np.empty((T, E), dtype=np.float64) if want_logits else None
    rc = lib().oracle_route(T, H, E, k, _p(x), _p(Wr), _p(bias), _p(gs), _p(logits), _p(idx), _p(w), _p(sg))
    if rc:
        raise ValueError("oracle_route: invalid arguments")
    return (idx, w, sg, logits) if want_logits else (idx, w, sg)


def combine_norm(y_routed, w, y_shared, sg: float, h_in, gamma, eps: float):
    """One token: y_routed float64 [k][H] -> (h_out, x_out float64 [H], x_out bf16 [H])."""
    y_routed = _c(np.atleast_2d(y_routed), np.float64); w = _c(w, np.float64)
    y_shared = _c(y_shared, np.float64); h_in = _c(h_in, np.float64); gamma = _c(gamma, np.uint16)
    k, H = y_routed.shape
    h_out = np.empty(H); x_out = np.empty(H); xb = np.empty(H, dtype=np.uint16)
    rc = lib().oracle_combine_norm(H, k, _p(y_routed), _p(w), _p(y_shared), float(sg), _p(h_in),
                                   _p(gamma), float(eps), _p(h_out), _p(x_out), _p(xb))
    if rc:
        raise ValueError("oracle_combine_norm: invalid arguments")
    return h_out, x_out, xb


def mx_layer(x, h_in, Wr, gamma, experts, shared, *, k: int, eps: float, router_bias=None, gs=None):
    """One layer with MXFP4 experts, composed of the oracle's steps: route; per token, for each
    chosen expert (rank order) and then the shared one, g = G x and u = U x (mx_gemv), a =
    swiglu(g, u), y = D a; then combine + residual + RMSNorm.
    experts: list of E ((qg, eg), (qu, eu), (qd, ed)); shared: one such tuple or None.
    Returns dict(h_out, x_out, x_out_bf16, idx, w, shared_gate)."""
    x = _c(np.atleast_2d(x), np.uint16); h_in = np.atleast_2d(np.asarray(h_in, dtype=np.float64))
    T, H = x.shape
    idx, w, sg = route(x, Wr, k, bias=router_bias, gs=gs if shared is not None else None)

    def run(ex, xt):
        (qg, eg), (qu, eu), (qd, ed) = ex
        g = mx_gemv(qg, eg, xt, H)
        u = mx_gemv(qu, eu, xt, H)
        return mx_gemv(qd, ed, swiglu(g, u), g.shape[0])

    out = {"h_out": np.empty((T, H)), "x_out": np.empty((T, H)), "x_out_bf16": np.empty((T, H), dtype=np.uint16),
           "idx": idx, "w": w, "shared_gate": sg}
    for t in range(T):
        xt = bf16_to_f64(x[t])
        yr = np.stack([run(experts[e], xt) for e in idx[t]])
        ys = run(shared, xt) if shared is not None else None
        out["h_out"][t], out["x_out"][t], out["x_out_bf16"][t] = combine_norm(
            yr, w[t], ys, sg[t] if shared is not None else 0.0, h_in[t], gamma, eps)
    return out


def group_by_expert(idx, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32); offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    rc = lib().oracle_group_by_expert(T, k, E, _p(idx), _p(counts), _p(offsets), _p(perm))
    if rc:
        raise ValueError("oracle_group_by_expert: invalid arguments")
    return counts, offsets, perm


def layer(x, h_in, Wr, gamma, experts, shared, *, I: int, k: int, G: int, bits: int, eps: float,
          router_bias=None, gs=None):
    """Whole layer with every expert in host memory.

    experts: list of E expert tuples (see ``expert``); shared: one tuple or None.
    Returns dict(h_out, x_out, x_out_bf16, idx, w, shared_gate)."""
    x = _c(np.atleast_2d(x), np.uint16); h_in = _c(np.atleast_2d(h_in), np.float64)
    Wr = _c(Wr, np.uint16); gamma = _c(gamma, np.uint16)
    router_bias = _c(router_bias, np.float32); gs = _c(gs, np.uint16)
    T, H = x.shape
    E = Wr.shape[0]
    keep = []

    def mk(ex):
        mats = []
        for (q, s, b) in ex:
            q = _c(q, np.uint32); s = _c(s, np.uint16); b = _c(b, np.uint16)
            keep.extend((q, s, b))
            mats.append(_Mat(q.ctypes.data, s.ctypes.data, b.ctypes.data))
        return _Expert(*mats)

    arr = (_Expert * E)(*[mk(e) for e in experts])
    sh = mk(shared) if shared is not None else None
    h_out = np.empty((T, H)); x_out = np.empty((T, H)); xb = np.empty((T, H), dtype=np.uint16)
    idx = np.empty((T, k), dtype=np.int32); w = np.empty((T, k)); sgo = np.empty(T)
    rc = lib().oracle_layer(T, H, I, E, k, G, bits, float(eps), _p(Wr), _p(router_bias), _p(gs),
                            _p(gamma), C.cast(arr, C.c_void_p), C.cast(C.pointer(sh), C.c_void_p) if sh is not None else None,
                            _p(x), _p(h_in), _p(h_out), _p(x_out), _p(xb), _p(idx), _p(w), _p(sgo))
    if rc:
        raise ValueError("oracle_layer: invalid arguments")
    return dict(h_out=h_out, x_out=x_out, x_out_bf16=xb, idx=idx, w=w, shared_gate=sgo)
