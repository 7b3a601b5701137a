"""ctypes binding of the plain-C fp64 oracle (``liboracle.so``).

TEST INFRASTRUCTURE: imported only by the tests, by ``__graft_entry__.smoke()``
and by the benchmark's CPU-baseline leg. The product path never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")

F32, BF16 = 0, 1


class Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("n_shared", ctypes.c_int), ("expert_top_p", ctypes.c_double)]


def build(verbose: bool = False) -> None:
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
           "-o", SO, os.path.join(HERE, "oracle.c"), "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} missing: run __graft_entry__.build()")
        L = ctypes.CDLL(SO)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_f16.argtypes = [ctypes.c_uint16]
        L.oracle_f16.restype = f64
        L.oracle_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_bf16.restype = f64
        L.oracle_code.argtypes = [vp, i32]
        L.oracle_code.restype = i32
        L.oracle_dequant.argtypes = [vp, vp, i32, i32, vp]
        L.oracle_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
        L.oracle_topk.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_topk.restype = i32
        L.oracle_weights_full_softmax.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_expert_topp.argtypes = [i32, i32, f64, vp, vp]
        L.oracle_expert_topp.restype = i32
        L.oracle_union.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
        L.oracle_union.restype = i32
        L.oracle_expert_ffn.argtypes = [vp, vp, i32, i32, vp, vp, vp]
        L.oracle_moe_forward.argtypes = [ctypes.POINTER(Cfg), vp, vp, vp, vp, vp, i32, i32, vp, vp, vp]
        L.oracle_moe_forward.restype = i32
        L.oracle_moe_forward_dense.argtypes = [ctypes.POINTER(Cfg), vp, vp, vp, vp, vp, i32, i32, vp]
        L.oracle_moe_forward_dense.restype = i32
        L.oracle_rmsnorm.argtypes = [vp, i32, i32, f64, vp]
        L.oracle_stack_step.argtypes = [ctypes.POINTER(Cfg), vp, vp, vp, vp, vp, i32, f64, vp]
        L.oracle_stack_step.restype = i32
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "arrays must be C-contiguous"
    return a.ctypes.data


def f16(bits: int) -> float:
    return lib().oracle_f16(bits)


def bf16(bits: int) -> float:
    return lib().oracle_bf16(bits)


def code(row: np.ndarray, c: int) -> int:
    row = np.ascontiguousarray(row, np.uint8)
    return lib().oracle_code(_p(row), c)


def dequant(q: np.ndarray, s: np.ndarray, rows: int, cols: int) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint16)
    w = np.empty((rows, cols), np.float64)
    lib().oracle_dequant(_p(q), _p(s), rows, cols, _p(w))
    return w


def _xdtype(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return F32
    if x.dtype == np.uint16:
        return BF16
    raise TypeError("x must be float32 or uint16 (bf16 bits)")


def router_logits(wr, bias, x):
    wr = np.ascontiguousarray(wr, np.float32)
    E, H = wr.shape
    x = np.ascontiguousarray(x)
    T = x.shape[0]
    out = np.empty((T, E), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    lib().oracle_router_logits(_p(wr), _p(b), _p(x), _xdtype(x), T, H, E, _p(out))
    return out


def topk(logits, K, top_p=None):
    """ids [T][K], weights [T][K]; with top_p in (0, 1) the adaptive expert
    top-p reduction follows (dropped slots: id -1, weight 0)."""
    logits = np.ascontiguousarray(logits, np.float64)
    T, E = logits.shape
    ids = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float64)
    if lib().oracle_topk(_p(logits), T, E, K, _p(ids), _p(w)):
        raise ValueError("oracle_topk: bad arguments or NaN logit")
    if top_p is not None and 0.0 < top_p < 1.0:
        lib().oracle_expert_topp(T, K, top_p, _p(ids), _p(w))
    return ids, w


def expert_topp(ids, w, p):
    """In-place adaptive expert top-p on a top-K result; returns slots kept."""
    assert ids.dtype == np.int32 and w.dtype == np.float64 and ids.flags["C_CONTIGUOUS"] and w.flags["C_CONTIGUOUS"]
    T, K = ids.shape
    return lib().oracle_expert_topp(T, K, p, _p(ids), _p(w))


def weights_full_softmax(logits, ids):
    logits = np.ascontiguousarray(logits, np.float64)
    ids = np.ascontiguousarray(ids, np.int32)
    T, E = logits.shape
    K = ids.shape[1]
    w = np.empty((T, K), np.float64)
    lib().oracle_weights_full_softmax(_p(logits), T, E, K, _p(ids), _p(w))
    return w


def union(ids, E):
    """Returns dict(cnt, off, unique, pos, tok)."""
    ids = np.ascontiguousarray(ids, np.int32)
    T, K = ids.shape
    cnt = np.empty(E, np.int32)
    off = np.empty(E + 1, np.int32)
    uniq = np.empty(E, np.int32)
    nu = np.zeros(1, np.int32)
    pos = np.empty(max(T * K, 1), np.int32)
    tok = np.empty(max(T * K, 1), np.int32)
    if lib().oracle_union(_p(ids), T, K, E, _p(cnt), _p(off), _p(uniq), _p(nu), _p(pos), _p(tok)):
        raise ValueError("oracle_union: id out of range")
    n = int(nu[0])
    return dict(cnt=cnt, off=off, unique=uniq[:n].copy(), pos=pos[:T * K].reshape(T, K), tok=tok[:T * K])


def expert_ffn(q, s, H, I, x, want_h=False):
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint16)
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(H, np.float64)
    h = np.empty(I, np.float64) if want_h else None
    lib().oracle_expert_ffn(_p(q), _p(s), H, I, _p(x), _p(out), _p(h))
    return (out, h) if want_h else out


def _ptr_arrays(experts):
    """experts: list (routed 0..E-1 then shared) of (q, s) or None."""
    n = len(experts)
    qa = (ctypes.c_void_p * n)()
    sa = (ctypes.c_void_p * n)()
    keep = []
    for i, e in enumerate(experts):
        if e is None:
            qa[i] = None
            sa[i] = None
        else:
            q = np.ascontiguousarray(e[0], np.uint8)
            s = np.ascontiguousarray(e[1], np.uint16)
            keep += [q, s]
            qa[i] = q.ctypes.data
            sa[i] = s.ctypes.data
    return qa, sa, keep


def moe_forward(cfg: Cfg, wr, bias, experts, x, dense=False):
    """y [T][H] fp64, ids [T][K], w [T][K] (ids/w None for dense)."""
    wr = np.ascontiguousarray(wr, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    x = np.ascontiguousarray(x)
    T = x.shape[0]
    y = np.empty((T, cfg.hidden), np.float64)
    qa, sa, keep = _ptr_arrays(experts)
    if dense:
        rc = lib().oracle_moe_forward_dense(ctypes.byref(cfg), _p(wr), _p(b), ctypes.cast(qa, ctypes.c_void_p),
                                            ctypes.cast(sa, ctypes.c_void_p), _p(x), _xdtype(x), T, _p(y))
        if rc:
            raise ValueError(f"oracle_moe_forward_dense rc={rc}")
        return y
    ids = np.empty((T, cfg.top_k), np.int32)
    w = np.empty((T, cfg.top_k), np.float64)
    rc = lib().oracle_moe_forward(ctypes.byref(cfg), _p(wr), _p(b), ctypes.cast(qa, ctypes.c_void_p),
                                  ctypes.cast(sa, ctypes.c_void_p), _p(x), _xdtype(x), T, _p(y), _p(ids), _p(w))
    if rc:
        raise ValueError(f"oracle_moe_forward rc={rc}")
    return y, ids, w


def rmsnorm(x, eps=1e-6):
    x = np.ascontiguousarray(x, np.float64)
    T, H = x.shape
    out = np.empty_like(x)
    lib().oracle_rmsnorm(_p(x), T, H, eps, _p(out))
    return out


def stack_step(cfg: Cfg, wr, bias, experts, x, eps=1e-6):
    """In-place residual step on an fp32 [T][H] array; returns ids."""
    assert x.dtype == np.float32 and x.flags["C_CONTIGUOUS"]
    wr = np.ascontiguousarray(wr, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    T = x.shape[0]
    ids = np.empty((T, cfg.top_k), np.int32)
    qa, sa, keep = _ptr_arrays(experts)
    rc = lib().oracle_stack_step(ctypes.byref(cfg), _p(wr), _p(b), ctypes.cast(qa, ctypes.c_void_p),
                                 ctypes.cast(sa, ctypes.c_void_p), _p(x), T, eps, _p(ids))
    if rc:
        raise ValueError(f"oracle_stack_step rc={rc}")
    return ids
