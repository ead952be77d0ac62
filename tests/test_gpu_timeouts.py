"""The bounded waits' failure path, without any GPU fault: the library's test hook makes
the integer GEMV's waits for the later pieces of its split row tiles look for a call
number that nobody writes, so they give up after a few polls.  The call must then write
NaN for exactly the row tiles split between CTAs, set the device status bit, and leave
nothing behind that a following call could mistake for its own data."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import Problem, to_numpy_f16

pytestmark = pytest.mark.gpu

PQ2 = oracle.FMT_PQ2_0


@pytest.fixture(scope="module")
def bz():
    import torch
    from ternary_weight_02_b200 import bonsai
    assert bonsai.bonsai_check_device() == bonsai.BONSAI_OK
    torch.cuda.init()
    return bonsai


def imma_split_tiles(N, K, sms):
    """Row tiles (32 rows) of the integer GEMV whose 512-weight items fall to two or more
    CTAs, from its work split: items (row tile, K chunk), CTA b taking items
    [I b / C, I (b + 1) / C), C = max(ceil(I / 96), min(ceil(I / 16), SMs))."""
    KC, RT = (K + 511) // 512, (N + 31) // 32
    I = RT * KC
    C = max(-(-I // 96), min(-(-I // 16), sms))
    bounds = {I * b // C for b in range(1, C)}
    return sorted({c // KC for c in bounds if c % KC != 0})


def _run(bz, x, packed, scales, N, K, M=1):
    import torch
    y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, PQ2, bz.BONSAI_ALGO_IMMA)
    torch.cuda.synchronize()
    got = to_numpy_f16(y)
    return got[0] if M == 1 else got


@pytest.mark.parametrize("M,N,K", [(1, 7168, 5120), (1, 5120, 17408), (2, 7168, 5120), (3, 7168, 5120)])
def test_forced_piece_timeouts_nan_status_and_recovery(bz, M, N, K):
    """M = 2: both tokens' pieces go through the same waits; every split tile is NaN in
    both rows of y."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p = Problem(M, N, K, PQ2, seed=N + K)
    x, packed, scales = p.device()
    ref = p.oracle_y()
    ref = ref[0] if M == 1 else ref
    split = imma_split_tiles(N, K, sms)
    assert len(split) > 0
    bz.bonsai_device_status(clear=True)
    bz.bonsai_debug_force_timeouts(True)
    try:
        got = _run(bz, x, packed, scales, N, K, M)
    finally:
        bz.bonsai_debug_force_timeouts(False)
    status = bz.bonsai_device_status(clear=True)
    assert status & bz.BONSAI_DEVICE_GEMV_PIECE_TIMEOUT
    assert not status & bz.BONSAI_DEVICE_GEMV_COPY_TIMEOUT
    bad = np.zeros(got.shape, dtype=bool)
    for t in split:
        bad[..., 32 * t:min(32 * t + 32, N)] = True
    assert np.all(np.isnan(got[bad]))
    assert np.all(np.isfinite(got[~bad]))
    ok, rel, mx = oracle.compare(got[~bad], ref[~bad])
    assert ok, (rel, mx)
    # the pieces that arrived after their reader gave up carry that call's number: the
    # next call (hook off) takes none of them
    for _ in range(2):
        again = _run(bz, x, packed, scales, N, K, M)
        ok, rel, mx = oracle.compare(again, ref)
        assert ok, (rel, mx)
    assert bz.bonsai_device_status() == 0


def test_status_is_clear_after_normal_calls(bz):
    p = Problem(1, 3000, 5120, PQ2, seed=3)
    x, packed, scales = p.device()
    bz.bonsai_device_status(clear=True)
    got = _run(bz, x, packed, scales, 3000, 5120)
    assert oracle.compare(got, p.oracle_y()[0])[0]
    assert bz.bonsai_device_status() == 0


def gemm_split_tiles(M, N, K, sms, pair=False):
    """Output tiles of the prefill GEMM that are split between CTAs, from its work split:
    tiles of 128 acc rows x 256 columns (row tile fastest), acc = 2 when M > 128; C = min(SMs,
    ceil(units / 4)) CTAs; W = T / C - 1 whole-tile waves when T >= 2C; the remaining tiles'
    64-wide K stages split evenly, CTA b taking units [Ur b / C, Ur (b + 1) / C).  CTA pairs
    (pair=True): tiles of 256 acc rows, acc = 2 when M > 256, and C = min(SMs / 2,
    ceil(units / 4)) pairs in place of CTAs.  Returns (tm, tn, rows of a tile)."""
    if pair:
        acc = 2 if M > 256 else 1
        rows = 256 * acc
    else:
        acc = 2 if M > 128 else 1
        rows = 128 * acc
    mt, nt, nk = -(-M // rows), -(-N // 256), K // 64
    C = max(1, min(sms // 2 if pair else sms, -(-(mt * nt * nk) // 4)))
    T = mt * nt
    W = T // C - 1 if T // C >= 2 else 0
    Ur = (T - W * C) * nk
    split = set()
    for b in range(1, C):
        u = Ur * b // C
        if u % nk != 0:
            split.add(W * C + u // nk)
    return [(s % mt, s // mt, rows) for s in sorted(split)]


@pytest.mark.parametrize("M,N,K", [(300, 1000, 640), (600, 2000, 1152)])
@pytest.mark.parametrize("tile", [0, 3])
def test_forced_gemm_flag_timeouts_nan_status_and_recovery(bz, M, N, K, tile):
    """tile 0: the automatic tiles; tile 3: CTA pairs, where both CTAs of an owner pair
    wait for their halves of the later pieces."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    p = Problem(M, N, K, PQ2, seed=M + N)
    x, packed, scales = p.device()
    ref = p.oracle_y()
    split = gemm_split_tiles(M, N, K, sms, pair=tile == 3)
    assert len(split) > 0

    def run():
        y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
        bz.bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, PQ2, bz.BONSAI_ALGO_GEMM, tile)
        torch.cuda.synchronize()
        return to_numpy_f16(y)

    bz.bonsai_device_status(clear=True)
    bz.bonsai_debug_force_timeouts(True)
    try:
        got = run()
    finally:
        bz.bonsai_debug_force_timeouts(False)
    status = bz.bonsai_device_status(clear=True)
    assert status & bz.BONSAI_DEVICE_GEMM_TIMEOUT
    bad = np.zeros((M, N), dtype=bool)
    for tm, tn, rows in split:
        bad[rows * tm:rows * (tm + 1), 256 * tn:256 * (tn + 1)] = True
    assert np.all(np.isnan(got[bad]))
    assert np.all(np.isfinite(got[~bad]))
    ok, rel, mx = oracle.compare(got[~bad], ref[~bad])
    assert ok, (rel, mx)
    for _ in range(2):
        again = run()
        ok, rel, mx = oracle.compare(again, ref)
        assert ok, (rel, mx)
    assert bz.bonsai_device_status() == 0
