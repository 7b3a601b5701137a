"""Seeded synthetic inputs for the int4 expert-FFN MoE layer.

Inputs only: router weights, routed/shared experts encoded in the int4 gs64
container, activations and a Zipf-skewed router bias. Nothing of the layer's
arithmetic lives here. The host generator (``libsynth_host.so``, gcc) and its
device twin (``libsynth_dev.so``, nvcc) compile the same definitions
(``synth_core.h``) and produce identical bytes.

Workload recipe (the shapes of the pages' layer: 256 routed experts, top-8,
~19 MB per int4 expert, groups of 64):
  * weights ~ 0.02 * N(0,1) (Irwin-Hall approximation), encoded per group of
    64 along the input dimension with an fp16 absmax/7 scale;
  * router weights 0.02 * N(0,1) in fp32, bias 0 or Zipf-skewed;
  * activations N(0,1) in fp32, or rounded to bf16.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libsynth_host.so")
DEV_SO = os.path.join(HERE, "libsynth_dev.so")

WSCALE = 0.02
ZIPF_S = 1.1
# Bias strength for Zipf(s=1.1) popularity, calibrated with
# tests/golden/calibrate_zipf.py (least-squares slope of log selection count
# against log popularity rank over 8192 tokens of the full-size layer = -1.10).
ZIPF_KAPPA = 0.0  # replaced by the calibrated value below, if present
_KAPPA_FILE = os.path.join(HERE, "zipf_kappa.txt")
if os.path.exists(_KAPPA_FILE):
    with open(_KAPPA_FILE) as _f:
        ZIPF_KAPPA = float(_f.read().split()[0])

GATE, UP, DOWN = 0, 1, 2


def build(verbose: bool = False) -> None:
    """Compile the host generator (gcc) and its device twin (nvcc, sm_100a)."""
    cmds = [
        ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
         "-o", HOST_SO, os.path.join(HERE, "synth_host.c"), "-lm"],
        ["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "-o", DEV_SO, os.path.join(HERE, "synth_dev.cu")],
    ]
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.check_call(c)


_host = None
_dev = None


def host_lib() -> ctypes.CDLL:
    global _host
    if _host is None:
        if not os.path.exists(HOST_SO):
            raise RuntimeError(f"{HOST_SO} missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(HOST_SO)
        u64, i32, f32, f64, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        lib.synth_expert.argtypes = [u64, i32, i32, i32, i32, f32, vp, vp]
        lib.synth_matrix_f32.argtypes = [u64, i32, i32, i32, i32, i32, f32, vp]
        lib.synth_encode.argtypes = [vp, i32, i32, vp, vp]
        lib.synth_router.argtypes = [u64, i32, i32, i32, f32, vp]
        lib.synth_x_f32.argtypes = [u64, i32, i32, i32, vp]
        lib.synth_x_bf16.argtypes = [u64, i32, i32, i32, vp]
        lib.synth_zipf_bias.argtypes = [u64, i32, i32, f64, f64, vp, vp]
        _host = lib
    return _host


def dev_lib() -> ctypes.CDLL:
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_SO):
            raise RuntimeError(f"{DEV_SO} missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(DEV_SO)
        u64, i32, f32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        lib.synth_expert_dev.argtypes = [u64, i32, i32, i32, i32, i32, f32, vp, vp, vp]
        lib.synth_router_dev.argtypes = [u64, i32, i32, i32, f32, vp, vp]
        lib.synth_x_dev.argtypes = [u64, i32, i32, i32, i32, vp, vp]
        _dev = lib
    return _dev


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def expert_sizes(H: int, I: int) -> tuple[int, int]:
    """(nibble bytes, fp16 scales) of one canonical expert."""
    return 3 * H * I // 2, 3 * H * I // 64


def expert(seed: int, layer: int, e: int, H: int, I: int, wscale: float = WSCALE):
    """Canonical (q bytes, fp16 scale bits) of expert ``e`` (routed 0..E-1, shared E..)."""
    nq, ns = expert_sizes(H, I)
    q = np.empty(nq, np.uint8)
    s = np.empty(ns, np.uint16)
    rc = host_lib().synth_expert(seed, layer, e, H, I, wscale, _ptr(q), _ptr(s))
    if rc:
        raise ValueError("synth_expert: bad sizes")
    return q, s


def matrix_f32(seed: int, layer: int, e: int, matrix: int, rows: int, cols: int, wscale: float = WSCALE):
    """The unencoded fp32 weights behind one expert matrix."""
    w = np.empty((rows, cols), np.float32)
    host_lib().synth_matrix_f32(seed, layer, e, matrix, rows, cols, wscale, _ptr(w))
    return w


def encode(w: np.ndarray):
    """Encode an fp32 matrix [rows][cols] into (q bytes [rows][cols/2], scales [rows][cols/64])."""
    w = np.ascontiguousarray(w, np.float32)
    rows, cols = w.shape
    q = np.empty((rows, cols // 2), np.uint8)
    s = np.empty((rows, cols // 64), np.uint16)
    if host_lib().synth_encode(_ptr(w), rows, cols, _ptr(q), _ptr(s)):
        raise ValueError("synth_encode: bad sizes")
    return q, s


def router(seed: int, layer: int, E: int, H: int, wscale: float = WSCALE):
    wr = np.empty((E, H), np.float32)
    host_lib().synth_router(seed, layer, E, H, wscale, _ptr(wr))
    return wr


def x_f32(seed: int, step: int, T: int, H: int):
    x = np.empty((T, H), np.float32)
    host_lib().synth_x_f32(seed, step, T, H, _ptr(x) if T else None)
    return x


def x_bf16(seed: int, step: int, T: int, H: int):
    """bf16 activations as raw uint16 bit patterns."""
    x = np.empty((T, H), np.uint16)
    host_lib().synth_x_bf16(seed, step, T, H, _ptr(x) if T else None)
    return x


def zipf_bias(seed: int, layer: int, E: int, kappa: float | None = None, s_exp: float = ZIPF_S):
    """(bias [E] fp32, popularity rank [E] int32) of a Zipf(s_exp) skew."""
    b = np.empty(E, np.float32)
    r = np.empty(E, np.int32)
    host_lib().synth_zipf_bias(seed, layer, E, ZIPF_KAPPA if kappa is None else kappa, s_exp, _ptr(b), _ptr(r))
    return b, r


# ----------------------------------------------------------------- device twin
def expert_dev(seed: int, layer: int, e0: int, n: int, H: int, I: int, q_ptr: int, s_ptr: int, stream=None,
               wscale: float = WSCALE) -> None:
    """Write experts e0..e0+n-1 (canonical) into device buffers."""
    rc = dev_lib().synth_expert_dev(seed, layer, e0, n, H, I, wscale, q_ptr, s_ptr, stream)
    if rc:
        raise RuntimeError(f"synth_expert_dev failed: cudaError {rc}")


def router_dev(seed: int, layer: int, E: int, H: int, ptr: int, stream=None, wscale: float = WSCALE) -> None:
    rc = dev_lib().synth_router_dev(seed, layer, E, H, wscale, ptr, stream)
    if rc:
        raise RuntimeError(f"synth_router_dev failed: cudaError {rc}")


def x_dev(seed: int, step: int, T: int, H: int, dtype: int, ptr: int, stream=None) -> None:
    """dtype 0: fp32, 1: bf16 bits."""
    rc = dev_lib().synth_x_dev(seed, step, T, H, dtype, ptr, stream)
    if rc:
        raise RuntimeError(f"synth_x_dev failed: cudaError {rc}")
