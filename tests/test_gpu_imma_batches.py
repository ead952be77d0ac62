"""The integer tensor-core GEMV on small batches (M = 2 and 3 for PQ2_0, M = 2 for PQ2_0
g64), against the float64 checker at the parity bar, and against itself at M = 1.

Each token has its own block fixed-point x~ (its own exponent per 128-block), and the
products of a group with x~ are exact integers in either layout; only the FP32 sums over
groups are taken in another order at M > 1 than at M = 1.  So every row of y at M > 1 is
within one FP16 rounding of what the kernel gives for that token alone.
"""
import numpy as np
import pytest

import oracle
from tests.gpu_util import Problem, to_numpy_f16

pytestmark = pytest.mark.gpu

PQ2, G64 = oracle.FMT_PQ2_0, oracle.FMT_PQ2_0_G64


@pytest.fixture(scope="module")
def bz():
    import torch
    from ternary_weight_02_b200 import bonsai
    assert bonsai.bonsai_check_device() == bonsai.BONSAI_OK
    torch.cuda.init()
    return bonsai


def _run(bz, x, packed, scales, M, N, K, fmt, algo):
    import torch
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, fmt, algo, 0)
    torch.cuda.synchronize()
    return to_numpy_f16(y)


# (N, K): ragged N (a partial last row tile), K not a multiple of 512 (per-lane scale
# loads instead of copies), one item per row tile, several CTAs per tile, and the largest K
SHAPES = [(1, 128), (33, 640), (1000, 1024), (777, 2432), (3000, 5120), (700, 12288)]
SHAPES3 = [(1, 128), (33, 640), (1000, 1024), (777, 2432), (3000, 5120), (700, 6144)]
CASES = ([(2, PQ2, N, K) for N, K in SHAPES] + [(2, G64, N, K) for N, K in SHAPES] +
         [(3, PQ2, N, K) for N, K in SHAPES3])


@pytest.mark.parametrize("M,fmt,N,K", CASES)
def test_small_batches_against_the_checker(bz, M, fmt, N, K):
    p = Problem(M, N, K, fmt, seed=N + K + M)
    x, packed, scales = p.device()
    got = _run(bz, x, packed, scales, M, N, K, fmt, bz.BONSAI_ALGO_IMMA)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


def _fp32_order_bound(p, m):
    """Bound on how far two FP32 summation orders of row n's per-group terms can lie apart:
    each term s[n,g] * sum_k t x~ 2^-e is at most s[n,g] * sum_k |x'_k| (plus the x~
    rounding, well inside the factor 2 below), and a sum of n terms in any order is within
    n 2^-24 of the sum of their magnitudes of the exact sum; two orders, so twice that."""
    gs = oracle.scale_group(p.fmt)
    xr = np.abs(oracle.hadamard128(p.x[m:m + 1].astype(np.float64))[0]).reshape(-1, gs).sum(axis=1)
    s = p.scales.astype(np.float64).reshape(p.N, -1)
    n_terms = 2 * s.shape[1] + 16
    return 2 * n_terms * 2.0 ** -24 * (s * xr[None, :]).sum(axis=1) * 2


@pytest.mark.parametrize("M,fmt", [(2, PQ2), (2, G64), (3, PQ2)])
@pytest.mark.parametrize("N,K", [(1000, 1024), (7168, 5120)])
def test_each_token_within_rounding_of_itself_alone(bz, M, fmt, N, K):
    """Each row of a batch against the same token alone: the integer group sums are the
    same, so the rows differ by no more than two FP32 summation orders of the group terms
    (bound above) and one FP16 rounding each."""
    p = Problem(M, N, K, fmt, seed=7 + N)
    x, packed, scales = p.device()
    batch = _run(bz, x, packed, scales, M, N, K, fmt, bz.BONSAI_ALGO_IMMA)
    for m in range(M):
        alone = _run(bz, x[m:m + 1].contiguous(), packed, scales, 1, N, K, fmt, bz.BONSAI_ALGO_IMMA)[0]
        ulp = np.spacing(np.abs(alone).astype(np.float16)).astype(np.float64)
        bound = _fp32_order_bound(p, m) + 2 * ulp
        err = np.abs(batch[m] - alone)
        assert np.all(err <= bound), (m, float(np.max(err / bound)))
        assert np.mean(batch[m] == alone) > 0.9  # most rows round to the same FP16 value


def test_two_tokens_of_very_different_range(bz):
    """One token 2^12 times the other: each token's blocks get their own exponent, so the
    small token keeps its precision."""
    import torch
    p = Problem(2, 2000, 2048, PQ2, seed=5)
    p.x = (p.x.astype(np.float64) * np.array([[2.0 ** 6], [2.0 ** -6]])).astype(np.float16)
    x, packed, scales = p.device()
    got = _run(bz, x, packed, scales, 2, p.N, p.K, PQ2, bz.BONSAI_ALGO_IMMA)
    ref = p.oracle_y()
    for m in range(2):
        ok, rel, mx = oracle.compare(got[m:m + 1], ref[m:m + 1])
        assert ok, (m, rel, mx)
    del torch


@pytest.mark.parametrize("M,fmt", [(2, PQ2), (2, G64), (3, PQ2)])
@pytest.mark.parametrize("name,K,N", [("qkv", 5120, 7168), ("o", 5120, 5120), ("gate_up", 5120, 34816)])
def test_small_batches_full_shapes_through_auto(bz, M, fmt, name, K, N):
    """The default entry point at M = 2, 3 on the 27B-class projections that fit
    (K = 5120): one launch, every output against the checker."""
    assert bz.bonsai_launch_count(M, N, K, fmt) == 1
    p = Problem(M, N, K, fmt, seed=60 + N + M)
    x, packed, scales = p.device()
    got = _run(bz, x, packed, scales, M, N, K, fmt, bz.BONSAI_ALGO_AUTO)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (name, rel, mx)


def test_two_tokens_repeatable(bz):
    """Split row tiles hand over both tokens' pieces through (value, epoch) pairs: the same
    call twice, and after a differently split shape, gives the same bits."""
    p = Problem(2, 7168, 5120, PQ2, seed=9)
    q = Problem(2, 1000, 3072, PQ2, seed=10)
    x, packed, scales = p.device()
    xq, pq, sq = q.device()
    a = _run(bz, x, packed, scales, 2, p.N, p.K, PQ2, bz.BONSAI_ALGO_IMMA)
    _run(bz, xq, pq, sq, 2, q.N, q.K, PQ2, bz.BONSAI_ALGO_IMMA)
    b = _run(bz, x, packed, scales, 2, p.N, p.K, PQ2, bz.BONSAI_ALGO_IMMA)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("M,fmt,K", [(2, PQ2, 17408), (3, PQ2, 7168), (3, G64, 1024), (4, PQ2, 1024)])
def test_past_the_small_batch_limits(bz, M, fmt, K):
    """Past the limits (M = 2 with K above 12288, e.g. the down projection; M = 3 with K
    above 6144; g64 with M = 3; M = 4) an explicit request is refused and the automatic
    choice takes the skinny kernel, against the checker."""
    import torch
    N = 640
    p = Problem(M, N, K, fmt, seed=4 + M)
    x, packed, scales = p.device()
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with pytest.raises(bz.BonsaiError):
        bz.bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, fmt, bz.BONSAI_ALGO_IMMA)
    assert bz.bonsai_launch_count(M, N, K, fmt) == bz.bonsai_launch_count(M, N, K, fmt, bz.BONSAI_ALGO_SKINNY)
    got = _run(bz, x, packed, scales, M, N, K, fmt, bz.BONSAI_ALGO_AUTO)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
