"""The no-allocation batch-1 entry point, for callers that cannot call cudaMalloc
(code running during CUDA-graph capture, allocators that own every byte of the
device, hosts that forbid allocation after start-up).  It runs the batch-1 layer on
a fixed scratch array inside the library's device image; its output must match the
regular entry point's and the float64 checker's within the parity bar, call after
call."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import Problem, to_numpy_f16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", [oracle.FMT_PTQ1_0, oracle.FMT_PQ2_0])
def test_noalloc_matches_regular_entry_point_two_calls(fmt):
    import torch
    from ternary_weight_02_b200 import bonsai as bz
    L = bz.raw()
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row on different shapes: the second reuses the scratch the first left
    for N, K, seed in ((3000, 5120, 11), (5120, 17408, 12)):
        p = Problem(1, N, K, fmt, seed=seed)
        x, packed, scales = p.device()
        y_reg = torch.empty((1, N), dtype=torch.float16, device="cuda")
        y_na = torch.full((1, N), float("nan"), dtype=torch.float16, device="cuda")
        assert L.bonsai_ternary_linear(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), y_reg.data_ptr(),
                                       1, N, K, fmt, stream) == bz.BONSAI_OK
        assert L.bonsai_ternary_linear_noalloc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(),
                                               y_na.data_ptr(), 1, N, K, fmt, stream) == bz.BONSAI_OK
        torch.cuda.synchronize()
        got, want = to_numpy_f16(y_na), to_numpy_f16(y_reg)
        ok, rel, mx = oracle.compare(got, want)
        assert ok, (N, K, rel, mx)
        ok, rel, mx = oracle.compare(got, p.oracle_y())
        assert ok, ("checker", N, K, rel, mx)


def test_noalloc_rejects_beyond_its_scratch():
    import torch
    from ternary_weight_02_b200 import bonsai as bz
    L = bz.raw()
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    # (K / 512) * N above 2^20 partials
    assert L.bonsai_ternary_linear_noalloc(p, p, p, p, 1, 40000, 17408, 2, stream) == bz.BONSAI_ERR_TOO_LARGE
    # batches are not served by this entry point
    assert L.bonsai_ternary_linear_noalloc(p, p, p, p, 2, 64, 512, 2, stream) == bz.BONSAI_ERR_TOO_LARGE
    assert L.bonsai_ternary_linear_noalloc(p, p, p, p, 1, 64, 384, 2, stream) == bz.BONSAI_ERR_TOO_LARGE
    assert "scratch" in bz.bonsai_status_string(bz.BONSAI_ERR_TOO_LARGE)
    # only PTQ1_0 and PQ2_0; a NULL pointer is reported before the size limit
    assert L.bonsai_ternary_linear_noalloc(p, p, p, p, 1, 64, 512, 3, stream) == bz.BONSAI_ERR_FMT
    assert L.bonsai_ternary_linear_noalloc(p, p, p, p, 1, 64, 512, 4, stream) == bz.BONSAI_ERR_FMT
    assert L.bonsai_ternary_linear_noalloc(p, None, p, p, 1, 40000, 17408, 2, stream) == bz.BONSAI_ERR_NULL
