"""Python face of the CPU checker (``bonsai_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg are the only callers.  Nothing in the
CUDA library or its binding imports this package, and this package imports
nothing from them.

All arithmetic happens in the C file in float64; this module only converts
arrays (FP16 -> float64 is exact) and calls it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bonsai_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

FMT_PTQ1_0 = 1
FMT_PQ2_0 = 2
FMT_Q1_0 = 3
FMT_PQ2_0_G64 = 4  # PQ2_0 codes, one FP16 scale per 64 weights
GROUP = 128
INVALID_TRIT = -128

_lib = None


def scale_group(fmt: int) -> int:
    """Weights per FP16 scale: 64 for PQ2_0 g64, 128 for the others."""
    return 64 if fmt == FMT_PQ2_0_G64 else GROUP


def build(force: bool = False) -> str:
    """Compile the checker with gcc (OpenMP on) unless an up-to-date build exists."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                           "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        ll, p, i = ctypes.c_longlong, ctypes.c_void_p, ctypes.c_int
        L.oracle_packed_bytes.restype = ll
        L.oracle_packed_bytes.argtypes = [i, ll, ll]
        for name in ("oracle_pack_ptq1", "oracle_pack_pq2", "oracle_pack_q1", "oracle_unpack_ptq1",
                     "oracle_unpack_pq2", "oracle_unpack_q1"):
            getattr(L, name).restype = ll
            getattr(L, name).argtypes = [p, p, ll, ll]
        for name in ("oracle_check_ptq1", "oracle_check_pq2", "oracle_check_q1"):
            getattr(L, name).restype = ll
            getattr(L, name).argtypes = [p, ll, ll]
        L.oracle_unpack.restype = ll
        L.oracle_unpack.argtypes = [i, p, p, ll, ll]
        L.oracle_sylvester128.restype = None
        L.oracle_sylvester128.argtypes = [p]
        L.oracle_hadamard128.restype = None
        L.oracle_hadamard128.argtypes = [p, p, ll, ll]
        L.oracle_fwht_recursive.restype = None
        L.oracle_fwht_recursive.argtypes = [p, ll]
        L.oracle_ternary_linear.restype = ll
        L.oracle_ternary_linear.argtypes = [p, p, p, p, ll, ll, ll, i, i, i]
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [p, p, ll, ll]
        L.oracle_max_threads.restype = i
        L.oracle_max_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def packed_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().oracle_packed_bytes(fmt, N, K))


def pack(fmt: int, trits: np.ndarray) -> np.ndarray:
    """N x K int8 trits -> packed uint8 plane (PTQ1_0: N x (K/128*26); PQ2_0: N x K/4;
    Q1_0: N x K/8, weights +-1)."""
    t = np.ascontiguousarray(trits, dtype=np.int8)
    N, K = t.shape
    nbytes = packed_bytes(fmt, N, K)
    if nbytes < 0:
        raise ValueError("bad format or shape")
    out = np.zeros(nbytes, dtype=np.uint8)
    fn = {FMT_PTQ1_0: lib().oracle_pack_ptq1, FMT_PQ2_0: lib().oracle_pack_pq2,
          FMT_Q1_0: lib().oracle_pack_q1, FMT_PQ2_0_G64: lib().oracle_pack_pq2}[fmt]
    fn(_ptr(t), _ptr(out), N, K)
    return out.reshape(N, -1) if N else out.reshape(0, 0)


def unpack(fmt: int, packed: np.ndarray, N: int, K: int):
    """Packed plane -> (N x K int8 trits, count of invalid codes met)."""
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if p.size != packed_bytes(fmt, N, K):
        raise ValueError("packed size does not match N, K")
    t = np.zeros((N, K), dtype=np.int8)
    bad = lib().oracle_unpack(fmt, _ptr(p), _ptr(t), N, K)
    if bad < 0:
        raise ValueError("bad format")
    return t, int(bad)


def check(fmt: int, packed: np.ndarray, N: int, K: int) -> int:
    """Number of non-canonical codes in a packed plane (0 for a valid one)."""
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    fn = {FMT_PTQ1_0: lib().oracle_check_ptq1, FMT_PQ2_0: lib().oracle_check_pq2,
          FMT_Q1_0: lib().oracle_check_q1, FMT_PQ2_0_G64: lib().oracle_check_pq2}[fmt]
    return int(fn(_ptr(p), N, K))


def sylvester128() -> np.ndarray:
    H = np.zeros((GROUP, GROUP), dtype=np.float64)
    lib().oracle_sylvester128(_ptr(H))
    return H


def hadamard128(x: np.ndarray) -> np.ndarray:
    """Float64 x' = blockdiag(Hn) x of an M x K (K % 128 == 0) array."""
    xd = np.ascontiguousarray(x, dtype=np.float64)
    M, K = xd.shape
    out = np.zeros_like(xd)
    lib().oracle_hadamard128(_ptr(xd), _ptr(out), M, K)
    return out


def fwht_recursive(v: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester transform of one power-of-two-length vector."""
    out = np.array(v, dtype=np.float64, copy=True)
    lib().oracle_fwht_recursive(_ptr(out), out.size)
    return out


def ternary_linear(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, N: int, K: int,
                   fmt: int, apply_hadamard: bool = True, nthreads: int = 0) -> np.ndarray:
    """Float64 y = x' . Wdeq^T for FP16 (or float64) x (M x K) and scales (N x K/128;
    N x K/64 for PQ2_0 g64)."""
    xd = np.ascontiguousarray(np.asarray(x).reshape(-1, K), dtype=np.float64)
    sd = np.ascontiguousarray(np.asarray(scales).reshape(N, K // scale_group(fmt)), dtype=np.float64)
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if p.size != packed_bytes(fmt, N, K):
        raise ValueError("packed size does not match N, K")
    M = xd.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    bad = lib().oracle_ternary_linear(_ptr(xd), _ptr(p), _ptr(sd), _ptr(y), M, N, K, fmt,
                                      1 if apply_hadamard else 0, nthreads)
    if bad < 0:
        raise ValueError("bad argument")
    return y


def swiglu(y: np.ndarray) -> np.ndarray:
    """h = silu(y[:, :F]) * y[:, F:] for an M x 2F float array (float64 result)."""
    yd = np.ascontiguousarray(y, dtype=np.float64)
    M, F2 = yd.shape
    if F2 % 2:
        raise ValueError("the fused gate/up output has an even number of columns")
    h = np.zeros((M, F2 // 2), dtype=np.float64)
    lib().oracle_swiglu(_ptr(yd), _ptr(h), M, F2 // 2)
    return h


def swiglu_linear(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, F: int, K: int, fmt: int,
                  nthreads: int = 0) -> np.ndarray:
    """The fused gate/up layer (2F weight rows: gate, then up) followed by SwiGLU: M x F."""
    return swiglu(ternary_linear(x, packed, scales, 2 * F, K, fmt, nthreads=nthreads))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def compare(y, y_ref, rel_l2: float = 1e-3, max_abs_rms: float = 1e-2):
    """The parity bar: relative L2 <= rel_l2 and max |y - y_ref| <= max_abs_rms * rms(y_ref).

    Returns (ok, rel_l2_error, max_abs_error / rms(y_ref))."""
    y = np.asarray(y, dtype=np.float64).reshape(-1)
    r = np.asarray(y_ref, dtype=np.float64).reshape(-1)
    if r.size == 0:
        return True, 0.0, 0.0
    nrm = float(np.sqrt(np.sum(r * r)))
    rms = nrm / np.sqrt(r.size)
    diff = y - r
    rel = float(np.sqrt(np.sum(diff * diff)) / nrm) if nrm > 0 else float(np.max(np.abs(diff)))
    mx = float(np.max(np.abs(diff)) / rms) if rms > 0 else float(np.max(np.abs(diff)))
    ok = bool(np.all(np.isfinite(y))) and rel <= rel_l2 and mx <= max_abs_rms
    return ok, rel, mx
