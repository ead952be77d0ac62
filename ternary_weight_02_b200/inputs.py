"""Seeded synthetic inputs for the ternary linear layer.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no packing, no Hadamard transform, no dot product).
Both the CUDA path and the CPU checker are fed from it.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based generator.  The
i-th output of a SplitMix64 stream whose state starts at ``s`` is
``mix64(s + (i + 1) * GAMMA)`` (all arithmetic mod 2**64), so any element
can be produced on its own, in any order and on any number of workers.
A tensor's stream state is itself the ``stream_id``-th output of the
stream seeded with ``seed``.

Distributions (the workload of the Bonsai 2 ternary linear layers: ternary
trits with one FP16 scale per 128 weights and FP16 activations):

* trits: u < 0.38 -> 0, u < 0.69 -> -1, else +1  (P(0)=.38, P(+-1)=.31);
* signs (the 1-bit Q1_0 weights): u < 0.5 -> -1, else +1;
* scales: 0.01 + 0.04 u in float64, rounded to FP16 (round to nearest even);
* x: standard normal by the Box-Muller transform in float64, rounded to FP16.

Element order is row-major: element (r, c) of an R x C tensor has counter
index r * C + c (for x, the Box-Muller pair p = index // 2 uses uniforms
2p and 2p+1).
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_TRITS = 1
STREAM_SCALES = 2
STREAM_X = 3
STREAM_SIGNS = 4

P_ZERO = 0.38
P_MINUS = 0.31
SCALE_LO = 0.01
SCALE_HI = 0.05

_CHUNK = 1 << 22  # elements generated per vectorised pass


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (in place on a uint64 array)."""
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, stream_id: int) -> np.uint64:
    """State of the sub-stream ``stream_id`` of the generator seeded with ``seed``."""
    with np.errstate(over="ignore"):
        s = np.array([seed], dtype=np.uint64)
        s += np.uint64(stream_id + 1) * GAMMA
        return _mix64(s)[0]


def raw_u64(key: np.uint64, index: np.ndarray) -> np.ndarray:
    """Outputs ``index`` (uint64 array) of the SplitMix64 stream with state ``key``."""
    with np.errstate(over="ignore"):
        z = (index.astype(np.uint64) + np.uint64(1)) * GAMMA
        z += key
        return _mix64(z)


def uniform(key: np.uint64, index: np.ndarray) -> np.ndarray:
    """Uniform doubles in [0, 1) from the top 53 bits of each output."""
    return (raw_u64(key, index) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _indices(rows: np.ndarray, cols: int) -> np.ndarray:
    return (rows.astype(np.uint64)[:, None] * np.uint64(cols)
            + np.arange(cols, dtype=np.uint64)[None, :])


def trits_rows(seed: int, K: int, rows, stream_id: int = STREAM_TRITS) -> np.ndarray:
    """Trits (int8 in {-1,0,1}) of the given rows of an N x K weight matrix."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    key = stream_key(seed, stream_id)
    out = np.empty((rows.size, K), dtype=np.int8)
    step = max(1, _CHUNK // max(K, 1))
    for r0 in range(0, rows.size, step):
        u = uniform(key, _indices(rows[r0:r0 + step], K))
        t = np.where(u < P_ZERO, 0, np.where(u < P_ZERO + P_MINUS, -1, 1))
        out[r0:r0 + step] = t.astype(np.int8)
    return out


def trits(seed: int, N: int, K: int, stream_id: int = STREAM_TRITS) -> np.ndarray:
    """N x K int8 trits, row-major."""
    return trits_rows(seed, K, np.arange(N), stream_id)


def signs_rows(seed: int, K: int, rows, stream_id: int = STREAM_SIGNS) -> np.ndarray:
    """1-bit weights (int8 in {-1, +1}) of the given rows of an N x K weight matrix."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    key = stream_key(seed, stream_id)
    out = np.empty((rows.size, K), dtype=np.int8)
    step = max(1, _CHUNK // max(K, 1))
    for r0 in range(0, rows.size, step):
        u = uniform(key, _indices(rows[r0:r0 + step], K))
        out[r0:r0 + step] = np.where(u < 0.5, -1, 1).astype(np.int8)
    return out


def signs(seed: int, N: int, K: int, stream_id: int = STREAM_SIGNS) -> np.ndarray:
    """N x K int8 weights in {-1, +1}, row-major."""
    return signs_rows(seed, K, np.arange(N), stream_id)


def scales_rows(seed: int, G: int, rows, stream_id: int = STREAM_SCALES) -> np.ndarray:
    """FP16 group scales of the given rows of an N x G scale plane."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    key = stream_key(seed, stream_id)
    u = uniform(key, _indices(rows, G))
    return (SCALE_LO + (SCALE_HI - SCALE_LO) * u).astype(np.float16)


def scales(seed: int, N: int, K: int, stream_id: int = STREAM_SCALES, group: int = 128) -> np.ndarray:
    """N x (K/group) FP16 scales, row-major (one scale per `group` weights of a row)."""
    return scales_rows(seed, K // group, np.arange(N), stream_id)


def normal_rows(seed: int, K: int, rows, stream_id: int = STREAM_X) -> np.ndarray:
    """FP16 N(0,1) activations of the given rows of an M x K matrix (K even)."""
    if K % 2:
        raise ValueError("K must be even for paired Box-Muller draws")
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    key = stream_key(seed, stream_id)
    out = np.empty((rows.size, K), dtype=np.float16)
    step = max(1, _CHUNK // max(K, 1))
    for r0 in range(0, rows.size, step):
        idx = _indices(rows[r0:r0 + step], K)
        u1 = uniform(key, idx[:, 0::2])
        u2 = uniform(key, idx[:, 1::2])
        rad = np.sqrt(-2.0 * np.log1p(-u1))  # 1 - u1 lies in (0, 1]
        ang = 2.0 * np.pi * u2
        z = np.empty(idx.shape, dtype=np.float64)
        z[:, 0::2] = rad * np.cos(ang)
        z[:, 1::2] = rad * np.sin(ang)
        out[r0:r0 + step] = z.astype(np.float16)
    return out


def activations(seed: int, M: int, K: int, stream_id: int = STREAM_X) -> np.ndarray:
    """M x K FP16 activations ~ N(0, 1), row-major."""
    return normal_rows(seed, K, np.arange(M), stream_id)
