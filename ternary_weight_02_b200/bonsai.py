"""Python binding of libbonsai (include/bonsai.h): argument marshalling only.

Every function has the name of the C entry point it calls and forwards raw
device pointers, sizes and the CUDA stream; all computation happens in the CUDA
kernels.  Tensors are torch CUDA tensors (torch is used for device memory and
streams only); plain integers are accepted as device pointers too.

Importing this module fails loudly if libbonsai.so has not been built: there is
no CPU fallback.  Build with ``python -m ternary_weight_02_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbonsai.so")

BONSAI_FMT_PTQ1_0 = 1
BONSAI_FMT_PQ2_0 = 2
BONSAI_FMT_Q1_0 = 3
BONSAI_FMT_PQ2_0_G64 = 4  # PQ2_0 codes, one FP16 scale per 64 weights

BONSAI_OK = 0
BONSAI_ERR_NULL = -1
BONSAI_ERR_SHAPE = -2
BONSAI_ERR_FMT = -3
BONSAI_ERR_ALIGN = -4
BONSAI_ERR_CUDA = -5
BONSAI_ERR_ARCH = -6
BONSAI_ERR_NOMEM = -7
BONSAI_ERR_ALGO = -8
BONSAI_ERR_TOO_LARGE = -9

BONSAI_DEVICE_GEMV_COPY_TIMEOUT = 1
BONSAI_DEVICE_GEMV_PIECE_TIMEOUT = 2
BONSAI_DEVICE_GEMM_TIMEOUT = 4
BONSAI_DEVICE_SKINNY_TIMEOUT = 8

BONSAI_ALGO_AUTO = 0
BONSAI_ALGO_SIMPLE = 1
BONSAI_ALGO_GEMV = 2
BONSAI_ALGO_SKINNY = 3
BONSAI_ALGO_GEMM = 4
BONSAI_ALGO_IMMA = 5

FORMATS = {"ptq1": BONSAI_FMT_PTQ1_0, "pq2": BONSAI_FMT_PQ2_0, "q1": BONSAI_FMT_Q1_0,
           "pq2g64": BONSAI_FMT_PQ2_0_G64}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libbonsai.so is missing at {LIB_PATH}; build it with "
        "`python -m ternary_weight_02_b200.build` (there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)
_i64, _int, _p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p

_SIGS = {
    "bonsai_version": (_int, []),
    "bonsai_status_string": (ctypes.c_char_p, [_int]),
    "bonsai_check_device": (_int, []),
    "bonsai_packed_bytes": (_i64, [_int, _i64, _i64]),
    "bonsai_pack_ptq1": (_int, [_p, _p, _i64, _i64, _p]),
    "bonsai_pack_pq2": (_int, [_p, _p, _i64, _i64, _p]),
    "bonsai_pack_q1": (_int, [_p, _p, _i64, _i64, _p]),
    "bonsai_unpack": (_int, [_int, _p, _p, _i64, _i64, _p]),
    "bonsai_hadamard128": (_int, [_p, _p, _i64, _i64, _p]),
    "bonsai_ternary_linear": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _int, _p]),
    "bonsai_ternary_linear_algo": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _int, _int, _int, _p]),
    "bonsai_ternary_linear_noalloc": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _int, _p]),
    "bonsai_launch_count": (_int, [_i64, _i64, _i64, _int, _int, _int]),
    "bonsai_swiglu": (_int, [_p, _p, _i64, _i64, _p]),
    "bonsai_ternary_linear_swiglu": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _int, _p]),
    "bonsai_reserve": (_int, [_i64, _i64, _i64]),
    "bonsai_device_status": (_int, [_p, ctypes.POINTER(ctypes.c_uint32), _int]),
    "bonsai_debug_force_timeouts": (_int, [_int]),
    "bonsai_shutdown": (None, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class BonsaiError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {bonsai_status_string(status)} (status {status})")


def raw():
    """The ctypes handle of libbonsai.so."""
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> int:
    if rc != BONSAI_OK:
        raise BonsaiError(rc, where)
    return rc


def bonsai_version() -> int:
    return _lib.bonsai_version()


def bonsai_status_string(status: int) -> str:
    return _lib.bonsai_status_string(status).decode()


def bonsai_check_device() -> int:
    return _lib.bonsai_check_device()


def bonsai_packed_bytes(fmt: int, N: int, K: int) -> int:
    v = _lib.bonsai_packed_bytes(fmt, N, K)
    if v < 0:
        raise BonsaiError(int(v), "bonsai_packed_bytes")
    return int(v)


def bonsai_pack_ptq1(trits, packed, N: int, K: int, stream=None) -> None:
    _check(_lib.bonsai_pack_ptq1(_ptr(trits), _ptr(packed), N, K, _stream(stream)), "bonsai_pack_ptq1")


def bonsai_pack_pq2(trits, packed, N: int, K: int, stream=None) -> None:
    _check(_lib.bonsai_pack_pq2(_ptr(trits), _ptr(packed), N, K, _stream(stream)), "bonsai_pack_pq2")


def bonsai_pack_q1(trits, packed, N: int, K: int, stream=None) -> None:
    _check(_lib.bonsai_pack_q1(_ptr(trits), _ptr(packed), N, K, _stream(stream)), "bonsai_pack_q1")


def bonsai_unpack(fmt: int, packed, trits, N: int, K: int, stream=None) -> None:
    _check(_lib.bonsai_unpack(fmt, _ptr(packed), _ptr(trits), N, K, _stream(stream)), "bonsai_unpack")


def bonsai_hadamard128(x, x_out, M: int, K: int, stream=None) -> None:
    _check(_lib.bonsai_hadamard128(_ptr(x), _ptr(x_out), M, K, _stream(stream)), "bonsai_hadamard128")


def bonsai_ternary_linear(x, packed, scales, y, M: int, N: int, K: int, fmt: int,
                          stream=None) -> None:
    _check(_lib.bonsai_ternary_linear(_ptr(x), _ptr(packed), _ptr(scales), _ptr(y), M, N, K, fmt,
                                      _stream(stream)), "bonsai_ternary_linear")


def bonsai_ternary_linear_algo(x, packed, scales, y, M: int, N: int, K: int, fmt: int, algo: int,
                               split_k: int = 0, stream=None) -> None:
    _check(_lib.bonsai_ternary_linear_algo(_ptr(x), _ptr(packed), _ptr(scales), _ptr(y), M, N, K,
                                           fmt, algo, split_k, _stream(stream)),
           "bonsai_ternary_linear_algo")


def bonsai_ternary_linear_noalloc(x, packed, scales, y, M: int, N: int, K: int, fmt: int,
                                  stream=None) -> None:
    """Batch-1 layer on the library's fixed device scratch: allocates nothing."""
    _check(_lib.bonsai_ternary_linear_noalloc(_ptr(x), _ptr(packed), _ptr(scales), _ptr(y), M, N, K,
                                              fmt, _stream(stream)), "bonsai_ternary_linear_noalloc")


def bonsai_launch_count(M: int, N: int, K: int, fmt: int, algo: int = BONSAI_ALGO_AUTO,
                        split_k: int = 0) -> int:
    n = _lib.bonsai_launch_count(M, N, K, fmt, algo, split_k)
    if n < 0:
        raise BonsaiError(n, "bonsai_launch_count")
    return n


def bonsai_reserve(M: int, N: int, K: int) -> None:
    _check(_lib.bonsai_reserve(M, N, K), "bonsai_reserve")


def bonsai_device_status(stream=None, clear: bool = False) -> int:
    """The calling device's status bits (BONSAI_DEVICE_*), after synchronising `stream`."""
    bits = ctypes.c_uint32(0)
    _check(_lib.bonsai_device_status(_stream(stream), ctypes.byref(bits), 1 if clear else 0),
           "bonsai_device_status")
    return int(bits.value)


def bonsai_debug_force_timeouts(enable: bool) -> None:
    """Test hook: cross-CTA waits give up (NaN outputs, status bits) while enabled."""
    _check(_lib.bonsai_debug_force_timeouts(1 if enable else 0), "bonsai_debug_force_timeouts")


def bonsai_shutdown() -> None:
    _lib.bonsai_shutdown()


# ---------------------------------------------------------------- conveniences

def bonsai_swiglu(y, h, M: int, F: int, stream=None) -> None:
    _check(_lib.bonsai_swiglu(_ptr(y), _ptr(h), M, F, _stream(stream)), "bonsai_swiglu")


def bonsai_ternary_linear_swiglu(x, packed, scales, h, M: int, F: int, K: int, fmt: int, stream=None) -> None:
    _check(_lib.bonsai_ternary_linear_swiglu(_ptr(x), _ptr(packed), _ptr(scales), _ptr(h), M, F, K, fmt,
                                             _stream(stream)), "bonsai_ternary_linear_swiglu")


def pack(fmt: int, trits, stream=None):
    """Packs an N x K int8 CUDA tensor of trits; returns the uint8 plane (N x bytes/row)."""
    import torch
    N, K = trits.shape
    out = torch.empty(bonsai_packed_bytes(fmt, N, K), dtype=torch.uint8, device=trits.device)
    fn = {BONSAI_FMT_PTQ1_0: bonsai_pack_ptq1, BONSAI_FMT_PQ2_0: bonsai_pack_pq2,
          BONSAI_FMT_Q1_0: bonsai_pack_q1, BONSAI_FMT_PQ2_0_G64: bonsai_pack_pq2}[fmt]
    fn(trits, out, N, K, stream)
    return out.view(N, -1) if N else out


def ternary_linear(x, packed, scales, N: int, fmt: int, algo: int = BONSAI_ALGO_AUTO,
                   split_k: int = 0, stream=None):
    """y = x' . Wdeq^T for an M x K FP16 CUDA tensor x; returns a new M x N FP16 tensor."""
    import torch
    M, K = x.shape
    y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, fmt, algo, split_k, stream)
    return y
