"""GPU parity through the C ABI against the CPU checker.

Integer work (packing, unpacking) must be bit-exact; the linear layer must meet
rel-L2 <= 1e-3 and max|y - y_ref| <= 1e-2 * rms(y_ref) against the float64
checker on the same seeded inputs."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import Problem, to_numpy_f16

pytestmark = pytest.mark.gpu

PTQ1, PQ2, Q1, G64 = oracle.FMT_PTQ1_0, oracle.FMT_PQ2_0, oracle.FMT_Q1_0, oracle.FMT_PQ2_0_G64


@pytest.fixture(scope="module")
def bz():
    import torch
    from ternary_weight_02_b200 import bonsai
    assert bonsai.bonsai_check_device() == bonsai.BONSAI_OK
    torch.cuda.init()
    return bonsai


# ------------------------------------------------------------ codec

@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("N,K", [(1, 128), (3, 384), (37, 1024), (64, 5120), (5, 17408)])
def test_pack_bit_exact(bz, fmt, N, K):
    import torch
    p = Problem(0, N, K, fmt, seed=N + K)
    packed = bz.pack(fmt, torch.from_numpy(p.trits).cuda())
    torch.cuda.synchronize()
    want = p.oracle_packed()
    got = packed.cpu().numpy().reshape(want.shape)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, G64])
def test_unpack_bit_exact_and_invalid_codes(bz, fmt):
    import torch
    N, K = 9, 640
    p = Problem(0, N, K, fmt, seed=3)
    packed = p.oracle_packed().copy()
    # plant invalid codes in the host-side plane before upload
    flat = packed.reshape(-1)
    if fmt == PTQ1:
        flat[[5, 77, 300]] = [243, 255, 250]
    else:
        flat[[5, 77, 300]] = [0xFF, 0x03, 0xC0]
    want, bad = oracle.unpack(fmt, packed, N, K)
    assert bad > 0
    t = torch.empty((N, K), dtype=torch.int8, device="cuda")
    bz.bonsai_unpack(fmt, torch.from_numpy(packed).cuda(), t, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(t.cpu().numpy(), want)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2])
def test_pack_marks_invalid_trits(bz, fmt):
    import torch
    t = np.zeros((2, 256), dtype=np.int8)
    t[1, 77] = 3
    t[0, 200] = -2
    got = bz.pack(fmt, torch.from_numpy(t).cuda()).cpu().numpy()
    assert np.array_equal(got.reshape(-1), oracle.pack(fmt, t).reshape(-1))
    assert oracle.check(fmt, got, 2, 256) == 2


def test_q1_unpack_every_byte_and_pack_non_binary(bz):
    import torch
    N, K = 2, 2048  # 512 bytes: every byte value twice
    packed = np.tile(np.arange(256, dtype=np.uint8), 2).reshape(N, K // 8)
    want, bad = oracle.unpack(Q1, packed, N, K)
    assert bad == 0
    t = torch.empty((N, K), dtype=torch.int8, device="cuda")
    bz.bonsai_unpack(Q1, torch.from_numpy(packed).cuda(), t, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(t.cpu().numpy(), want)
    # weights other than +-1 are stored as -1, as the checker's packer does
    w = np.ones((2, 256), dtype=np.int8)
    w[0, 5] = 0
    w[1, 200] = 3
    got = bz.pack(Q1, torch.from_numpy(w).cuda()).cpu().numpy()
    assert np.array_equal(got.reshape(-1), oracle.pack(Q1, w).reshape(-1))


# ------------------------------------------------------------ Hadamard

@pytest.mark.parametrize("M,K", [(1, 128), (3, 1024), (17, 5120), (2, 17408)])
def test_hadamard128(bz, M, K):
    import torch
    p = Problem(M, 1, K, PQ2, seed=M)
    x, _, _ = p.device()
    out = torch.empty_like(x)
    bz.bonsai_hadamard128(x, out, M, K)
    torch.cuda.synchronize()
    got = to_numpy_f16(out)
    ref = oracle.hadamard128(p.x.astype(np.float64))
    ok, rel, mx = oracle.compare(got, ref)
    assert ok, (rel, mx)
    # FP32 butterflies then one rounding: within one FP16 ulp of the exact value
    ref16 = ref.astype(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - ref16) <= ulp)
    assert np.mean(got == ref16) > 0.99
    # in place gives the same bits
    bz.bonsai_hadamard128(x, x, M, K)
    torch.cuda.synchronize()
    assert torch.equal(x, out)


# ------------------------------------------------------------ linear

def _run(bz, p, algo, split_k=0):
    import torch
    x, packed, scales = p.device()
    y = torch.full((p.M, p.N), float("nan"), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear_algo(x, packed, scales, y, p.M, p.N, p.K, p.fmt, algo, split_k)
    torch.cuda.synchronize()
    return to_numpy_f16(y)


SIMPLE_CASES = [(1, 1, 128), (1, 33, 384), (3, 100, 1024), (17, 65, 640), (1, 1024, 1024)]


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("M,N,K", SIMPLE_CASES)
def test_linear_simple(bz, fmt, M, N, K):
    p = Problem(M, N, K, fmt, seed=M * 7 + N)
    got = _run(bz, p, bz.BONSAI_ALGO_SIMPLE)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
def test_linear_auto_config1(bz, fmt):
    """Single ternary linear, M=1, K=1024 -> N=1024, seed 0, through the default entry point."""
    import torch
    p = Problem(1, 1024, 1024, fmt, seed=0)
    x, packed, scales = p.device()
    y = torch.empty((1, 1024), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear(x, packed, scales, y, 1, 1024, 1024, fmt)
    torch.cuda.synchronize()
    got = to_numpy_f16(y)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
    # negative: the same output is far from the product without the rotation
    bad_ok, bad_rel, _ = oracle.compare(got, p.oracle_y(apply_hadamard=False))
    assert not bad_ok and bad_rel > 0.5


def test_argument_errors_on_device(bz):
    import torch
    x = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    y = torch.zeros((1, 16), dtype=torch.float16, device="cuda")
    s = torch.zeros((16, 2), dtype=torch.float16, device="cuda")
    w = torch.zeros((16, 64), dtype=torch.uint8, device="cuda")
    L = bz.raw()
    stream = torch.cuda.current_stream().cuda_stream
    assert L.bonsai_ternary_linear(x.data_ptr() + 2, w.data_ptr(), s.data_ptr(), y.data_ptr(), 1,
                                   16, 256, 2, stream) == bz.BONSAI_ERR_ALIGN
    assert L.bonsai_ternary_linear_algo(x.data_ptr(), w.data_ptr(), s.data_ptr(), y.data_ptr(), 2,
                                        16, 256, 2, bz.BONSAI_ALGO_GEMV, 0, stream) in (
        bz.BONSAI_ERR_ALGO,)


# ------------------------------------------------------------ batch-1 GEMV (lookup tables)

GEMV_CASES = [(1, 512), (33, 512), (100, 1024), (1024, 1024), (1000, 2048), (37, 17408)]


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, G64])
@pytest.mark.parametrize("N,K", GEMV_CASES)
def test_gemv_small(bz, fmt, N, K):
    p = Problem(1, N, K, fmt, seed=N + 3 * K)
    got = _run(bz, p, bz.BONSAI_ALGO_GEMV)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


# Q1_0 (1-bit): a byte covers 8 activations, so the lookup-table GEMV's K slice is 1024
Q1_GEMV_CASES = [(1, 1024), (33, 1024), (100, 3072), (1000, 2048), (37, 17408)]


@pytest.mark.parametrize("N,K", Q1_GEMV_CASES)
def test_gemv_small_q1(bz, N, K):
    p = Problem(1, N, K, Q1, seed=N + 5 * K)
    got = _run(bz, p, bz.BONSAI_ALGO_GEMV)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


def test_q1_k_not_multiple_of_1024(bz):
    """The lookup-table GEMV refuses Q1_0 at K % 1024 != 0; the default entry point then
    takes the plain kernel, still against the checker."""
    p = Problem(1, 50, 640, Q1, seed=4)
    with pytest.raises(bz.BonsaiError):
        _run(bz, p, bz.BONSAI_ALGO_GEMV)
    ok, rel, mx = oracle.compare(_run(bz, p, bz.BONSAI_ALGO_AUTO), p.oracle_y())
    assert ok, (rel, mx)


# 27B-class decode projections (K -> N): qkv, o, fused gate/up, down
DECODE_SHAPES = [(5120, 7168), (5120, 5120), (5120, 34816), (17408, 5120)]


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("K,N", DECODE_SHAPES)
def test_gemv_decode_shapes_full(bz, fmt, K, N):
    """Every output of the full-size M=1 projections against the float64 checker."""
    p = Problem(1, N, K, fmt, seed=0)
    got = _run(bz, p, bz.BONSAI_ALGO_GEMV)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
    if fmt in (PTQ1, Q1):  # through the default entry point too (M == 1 dispatches here)
        import torch
        x, packed, scales = p.device()
        y = torch.empty((1, N), dtype=torch.float16, device="cuda")
        bz.bonsai_ternary_linear(x, packed, scales, y, 1, N, K, fmt)
        torch.cuda.synchronize()
        assert np.array_equal(to_numpy_f16(y), got)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
def test_gemv_repeatable_and_counters_reset(bz, fmt):
    """Split-K arrival counters return to zero: back-to-back calls on different shapes
    give bit-identical results (the slice-ordered reduction is deterministic)."""
    import torch
    pa = Problem(1, 3000, 5120, fmt, seed=1)
    pb = Problem(1, 77, 17408, fmt, seed=2)
    da, db = pa.device(), pb.device()
    outs = []
    for _ in range(3):
        for p, (x, packed, scales) in ((pa, da), (pb, db)):
            y = torch.empty((1, p.N), dtype=torch.float16, device="cuda")
            bz.bonsai_ternary_linear_algo(x, packed, scales, y, 1, p.N, p.K, p.fmt,
                                          bz.BONSAI_ALGO_GEMV, 0)
            outs.append(y)
    torch.cuda.synchronize()
    for i in range(2, 6):
        assert torch.equal(outs[i], outs[i % 2])
    assert oracle.compare(to_numpy_f16(outs[0]), pa.oracle_y())[0]
    assert oracle.compare(to_numpy_f16(outs[1]), pb.oracle_y())[0]


def test_gemv_rejects_batches(bz):
    import torch
    x = torch.zeros((2, 512), dtype=torch.float16, device="cuda")
    y = torch.zeros((2, 8), dtype=torch.float16, device="cuda")
    s = torch.zeros((8, 4), dtype=torch.float16, device="cuda")
    w = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(bz.BonsaiError):
        bz.bonsai_ternary_linear_algo(x, w, s, y, 2, 8, 512, PQ2, bz.BONSAI_ALGO_GEMV)


# ------------------------------------------------------------ batch-1 GEMV (integer tensor cores)

# ragged N (not a multiple of the 32-row item) and ragged K (not a multiple of the
# 512-weight item), one item, many items, the largest K the kernel takes
IMMA_CASES = [(1, 128), (33, 384), (31, 640), (100, 1024), (1024, 1024), (1000, 2048), (5000, 1152),
              (37, 17408), (70, 24576),
              # enough items that every consumer warp walks its ring several times, with
              # ragged N / K, and K not a multiple of 1024 (scales loaded without TMA)
              (6000, 6144), (4099, 8192), (9000, 2560), (4000, 9728),
              # more items per warp than ring buffers: the producer waits for released buffers
              (20000, 8192), (12000, 10752)]


@pytest.mark.parametrize("fmt", [PQ2, G64])
@pytest.mark.parametrize("N,K", IMMA_CASES)
def test_imma_small(bz, fmt, N, K):
    p = Problem(1, N, K, fmt, seed=N + 5 * K)
    got = _run(bz, p, bz.BONSAI_ALGO_IMMA)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


@pytest.mark.parametrize("fmt", [PQ2, G64])
@pytest.mark.parametrize("K,N", DECODE_SHAPES)
def test_imma_decode_shapes_full(bz, fmt, K, N):
    """Every output of the full-size M=1 PQ2_0 (and g64) projections against the float64
    checker, and the default entry point (which dispatches M == 1 here) bit-equal to it."""
    import torch
    p = Problem(1, N, K, fmt, seed=0)
    got = _run(bz, p, bz.BONSAI_ALGO_IMMA)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
    x, packed, scales = p.device()
    y = torch.empty((1, N), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear(x, packed, scales, y, 1, N, K, fmt)
    torch.cuda.synchronize()
    assert np.array_equal(to_numpy_f16(y), got)
    assert bz.bonsai_launch_count(1, N, K, fmt) == 1


def test_imma_repeatable_and_counters_reset(bz):
    """Row tiles split between CTAs are summed through (value, epoch) pairs that their
    reader clears, so back-to-back calls on shapes with different splits (among them the
    34816 x 5120 and 20000 x 8192 ones, many row tiles per CTA) give bit-identical
    results."""
    import torch
    probs = [Problem(1, 3000, 5120, PQ2, seed=1), Problem(1, 77, 17408, PQ2, seed=2),
             Problem(1, 34816, 5120, PQ2, seed=4), Problem(1, 5120, 17408, PQ2, seed=3),
             Problem(1, 20000, 8192, PQ2, seed=5), Problem(1, 34816, 5120, G64, seed=6),
             Problem(1, 5000, 1152, G64, seed=7)]
    devs = [p.device() for p in probs]
    outs = []
    for _ in range(3):
        for p, (x, packed, scales) in zip(probs, devs):
            y = torch.empty((1, p.N), dtype=torch.float16, device="cuda")
            bz.bonsai_ternary_linear_algo(x, packed, scales, y, 1, p.N, p.K, p.fmt, bz.BONSAI_ALGO_IMMA, 0)
            outs.append(y)
    torch.cuda.synchronize()
    n = len(probs)
    for i in range(n, 3 * n):
        assert torch.equal(outs[i], outs[i % n])
    for i, p in enumerate(probs):
        assert oracle.compare(to_numpy_f16(outs[i]), p.oracle_y())[0]


@pytest.mark.parametrize("fmt", [PQ2, G64])
def test_imma_input_with_large_and_small_groups(bz, fmt):
    """Groups of x whose magnitudes differ by 2^20 get their own power-of-two scales."""
    p = Problem(1, 256, 2048, fmt, seed=9)
    xs = p.x.astype(np.float32)
    for g in range(16):
        xs[:, 128 * g:128 * (g + 1)] *= 2.0 ** (5 if g % 2 else -15)
    p.x = xs.astype(np.float16)
    got = _run(bz, p, bz.BONSAI_ALGO_IMMA)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


def test_imma_rejects_what_it_cannot_run(bz):
    import torch
    x = torch.zeros((4, 512), dtype=torch.float16, device="cuda")
    y = torch.zeros((4, 8), dtype=torch.float16, device="cuda")
    s = torch.zeros((8, 4), dtype=torch.float16, device="cuda")
    w = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(bz.BonsaiError):  # a batch of four
        bz.bonsai_ternary_linear_algo(x, w, s, y, 4, 8, 512, PQ2, bz.BONSAI_ALGO_IMMA)
    with pytest.raises(bz.BonsaiError):  # PTQ1_0
        bz.bonsai_ternary_linear_algo(x[:1], w, s, y[:1], 1, 8, 512, PTQ1, bz.BONSAI_ALGO_IMMA)


# ------------------------------------------------------------ prefill GEMM (tcgen05 / TMEM)

# The last one or two waves of tiles are split over the CTAs by 64-wide K stages (at
# least 4 per CTA): these shapes put a tile on 1 to ~5 CTAs, so split tiles are handed
# over through chains of one to four later pieces, and some CTAs hold several tiles.
# (2000, 9500, 256) has more than two waves of tiles on 148 SMs: whole-tile waves first,
# then the split remainder.
GEMM_SMALL = [(1, 64, 128), (17, 256, 128), (130, 300, 384), (256, 512, 1024), (300, 1000, 640),
              (600, 2000, 1152), (1000, 3000, 2048), (2000, 9500, 256)]


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("M,N,K", GEMM_SMALL)
@pytest.mark.parametrize("tile", [1, 2, 3])
def test_gemm_small(bz, fmt, M, N, K, tile):
    """tile 1: one 128-row TMEM accumulator per CTA; tile 2: two (256 rows); tile 3: CTA
    pairs sharing each MMA (cta_group::2), 256 or 512 rows per tile."""
    p = Problem(M, N, K, fmt, seed=M + N + K)
    got = _run(bz, p, bz.BONSAI_ALGO_GEMM, tile)
    assert np.all(np.isfinite(got))
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("tile", [0, 3])
def test_gemm_split_tiles_repeatable(bz, fmt, tile):
    """Split tiles hand their partial sums over through flags that carry the call's
    epoch: the same call twice, and after a differently split shape, gives the same bits."""
    p = Problem(2048, 8192, 384, fmt, seed=11)
    q = Problem(300, 1000, 640, fmt, seed=12)
    a = _run(bz, p, bz.BONSAI_ALGO_GEMM, tile)
    _run(bz, q, bz.BONSAI_ALGO_GEMM, tile)
    b = _run(bz, p, bz.BONSAI_ALGO_GEMM, tile)
    assert np.array_equal(a, b)
    ok, rel, mx = oracle.compare(a, p.oracle_y())
    assert ok, (rel, mx)


def _sampled_reference(fmt, M, N, K, seed, ms, ns):
    """Checker values of y at the (m, n) pairs of ms x ns, from regenerated input rows."""
    from ternary_weight_02_b200 import inputs
    um, un = np.unique(ms), np.unique(ns)
    x = inputs.normal_rows(seed, K, um)
    t = inputs.signs_rows(seed, K, un) if fmt == Q1 else inputs.trits_rows(seed, K, un)
    s = inputs.scales_rows(seed, K // oracle.scale_group(fmt), un)
    y = oracle.ternary_linear(x, oracle.pack(fmt, t), s, len(un), K, fmt)
    return y, um, un


# prefill: M tokens x 27B-class projections (K -> N)
PREFILL = [(2048, 5120, 34816), (512, 17408, 5120), (8192, 5120, 7168)]


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1, G64])
@pytest.mark.parametrize("M,K,N", PREFILL)
def test_gemm_prefill_full_size_sampled(bz, fmt, M, K, N):
    """Full-size GEMM on the device; 64 x 64 sampled outputs against the checker."""
    import torch
    from ternary_weight_02_b200 import inputs
    seed = 5
    dev = torch.device("cuda")
    w = inputs.signs(seed, N, K) if fmt == Q1 else inputs.trits(seed, N, K)
    t = torch.from_numpy(w).to(dev)
    del w
    packed = bz.pack(fmt, t)
    del t
    s = torch.from_numpy(inputs.scales(seed, N, K, group=oracle.scale_group(fmt)).view(np.int16))
    s = s.to(dev).view(torch.float16)
    x = torch.from_numpy(inputs.activations(seed, M, K).view(np.int16)).to(dev).view(torch.float16)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device=dev)
    bz.bonsai_ternary_linear(x, packed, s, y, M, N, K, fmt)
    torch.cuda.synchronize()
    assert bz.bonsai_launch_count(M, N, K, fmt) == 1  # the rotation runs inside the GEMM
    rng = np.random.default_rng(M + N)
    ms = np.concatenate([[0, M - 1], rng.integers(0, M, 62)])
    ns = np.concatenate([[0, N - 1], rng.integers(0, N, 62)])
    ref, um, un = _sampled_reference(fmt, M, N, K, seed, ms, ns)
    got = y[torch.from_numpy(um).to(dev)][:, torch.from_numpy(un).to(dev)].float().cpu().numpy()
    ok, rel, mx = oracle.compare(got, ref)
    assert ok, (rel, mx)
    assert bool(torch.isfinite(y).all())


# ------------------------------------------------------------ skinny batches (mma.sync, PQ2_0)

SKINNY_SMALL = [(2, 64, 128), (3, 129, 384), (8, 300, 1024), (9, 100, 640), (16, 257, 2048)]


@pytest.mark.parametrize("fmt", [PQ2, G64, Q1, PTQ1])
@pytest.mark.parametrize("M,N,K", SKINNY_SMALL)
@pytest.mark.parametrize("split_k", [0, 1, 3])
def test_skinny_small(bz, fmt, M, N, K, split_k):
    p = Problem(M, N, K, fmt, seed=M * 31 + N)
    got = _run(bz, p, bz.BONSAI_ALGO_SKINNY, split_k)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


@pytest.mark.parametrize("fmt", [PQ2, G64, Q1, PTQ1])
@pytest.mark.parametrize("M", [2, 4, 8, 16])
@pytest.mark.parametrize("K,N", [(5120, 7168), (5120, 5120), (17408, 5120), (5120, 34816)])
def test_skinny_decode_shapes_full(bz, fmt, M, K, N):
    """Skinny decode batches on 27B-class projections, every output against the checker
    (the default entry point takes the skinny kernel for every packing); one launch when
    the kernel's grid is resident at once, as it is at these shapes."""
    p = Problem(M, N, K, fmt, seed=M)
    got = _run(bz, p, bz.BONSAI_ALGO_AUTO)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
    assert bz.bonsai_launch_count(M, N, K, fmt) == 1


@pytest.mark.parametrize("fmt", [PQ2, G64, Q1, PTQ1])
@pytest.mark.parametrize("M", [2, 3])
@pytest.mark.parametrize("K,N", [(5120, 7168), (17408, 5120)])
def test_skinny_explicit_small_batches_full(bz, fmt, M, K, N):
    """The skinny kernel asked for explicitly at M = 2, 3 on full shapes (the default entry
    point gives most of these to the integer GEMV; down and the explicit choice still run
    the skinny kernel, with its TMA ring for every packing but PTQ1_0)."""
    p = Problem(M, N, K, fmt, seed=70 + M)
    got = _run(bz, p, bz.BONSAI_ALGO_SKINNY)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)


@pytest.mark.parametrize("fmt", [PQ2, G64, Q1, PTQ1])
def test_skinny_split_is_deterministic(bz, fmt):
    import torch
    p = Problem(8, 5120, 17408, fmt, seed=3)
    x, packed, scales = p.device()
    outs = []
    for sk in (0, 0, 5, 5):
        y = torch.empty((8, 5120), dtype=torch.float16, device="cuda")
        bz.bonsai_ternary_linear_algo(x, packed, scales, y, 8, 5120, 17408, fmt, bz.BONSAI_ALGO_SKINNY, sk)
        outs.append(y)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[2], outs[3])
    assert oracle.compare(to_numpy_f16(outs[2]), to_numpy_f16(outs[0]))[0]


@pytest.mark.parametrize("M", [2, 5, 16])
@pytest.mark.parametrize("N,K", [(300, 1024), (3, 128), (77, 640)])
def test_small_batches_ptq1(bz, M, N, K):
    """PTQ1_0 batches take the skinny kernel (base-3 bytes transcoded to 2-bit codes); the
    small N puts the plane's last group, whose lanes read its final bytes, in most warps."""
    p = Problem(M, N, K, PTQ1, seed=M + N)
    got = _run(bz, p, bz.BONSAI_ALGO_AUTO)
    ok, rel, mx = oracle.compare(got, p.oracle_y())
    assert ok, (rel, mx)
    assert np.array_equal(got, _run(bz, p, bz.BONSAI_ALGO_SKINNY))


# ------------------------------------------------------------ SwiGLU after the fused gate/up projection

def swiglu_ok(h, y_ref):
    """The SwiGLU output's bar, derived from the linear layer's: with |dy| <= 1e-2 rms(y)
    on every gate and up value (the linear bar) and |silu'| <= 1.1, each h = silu(g) u may
    move by (1.1 |u| + |silu(g)|) 1e-2 rms(y), plus one FP16 rounding of h; and rel-L2 of h
    <= 1e-3 as for the linear output.  Returns (ok, rel-L2, worst ratio of error to bound)."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    F = y_ref.shape[1] // 2
    g, u = y_ref[:, :F], y_ref[:, F:]
    h_ref = oracle.swiglu(y_ref)
    rms_y = np.sqrt(np.mean(y_ref ** 2))
    bound = (1.1 * np.abs(u) + np.abs(g / (1.0 + np.exp(-g)))) * 1e-2 * rms_y + 2.0 ** -11 * np.abs(h_ref)
    err = np.abs(np.asarray(h, dtype=np.float64) - h_ref)
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(h_ref), 1e-300))
    worst = float(np.max(err / np.maximum(bound, 1e-300)))
    return rel <= 1e-3 and worst <= 1.0, rel, worst


def _run_swiglu(bz, p, F):
    import torch
    x, packed, scales = p.device()
    h = torch.full((p.M, F), float("nan"), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear_swiglu(x, packed, scales, h, p.M, F, p.K, p.fmt)
    torch.cuda.synchronize()
    return to_numpy_f16(h)


# (M, F, K, fmt): fused in the integer GEMV (M = 1 PQ2_0 and g64, M = 2 both, M = 3 PQ2_0;
# F = 24 leaves a part-used last tile; the M = 1 and 2 cases at F = 17408 are the full
# 27B-class gate/up) or the GEMM (tiles split between CTAs; F = 200 and 1270 part-used);
# the other packings at M = 1 and the skinny batches take the linear kernel and then the
# SwiGLU kernel
SWIGLU_CASES = [(1, 16, 512, PQ2), (1, 1024, 2048, PQ2), (1, 4000, 1152, PQ2), (1, 24, 512, PQ2),
                (1, 1024, 1024, PTQ1), (1, 1024, 2048, Q1), (4, 512, 1024, PQ2), (300, 640, 640, PQ2),
                (300, 640, 640, Q1), (300, 384, 1152, PTQ1), (600, 1280, 384, PQ2), (300, 200, 640, PQ2), (300, 1270, 256, Q1),
                (1, 1024, 2048, G64), (1, 24, 512, G64), (1, 4000, 1152, G64), (300, 200, 640, G64),
                (600, 1280, 384, G64), (4, 512, 1024, G64), (4, 512, 1024, Q1), (1, 17408, 5120, PQ2), (1, 17408, 5120, G64),
                (2, 1024, 2048, PQ2), (2, 24, 512, PQ2), (2, 4000, 1152, G64), (2, 17408, 5120, PQ2),
                (3, 1024, 2048, PQ2), (3, 24, 640, PQ2)]


@pytest.mark.parametrize("M,F,K,fmt", SWIGLU_CASES)
def test_linear_swiglu(bz, M, F, K, fmt):
    p = Problem(M, 2 * F, K, fmt, seed=M + F + K)
    got = _run_swiglu(bz, p, F)
    assert np.all(np.isfinite(got))
    ok, rel, worst = swiglu_ok(got, p.oracle_y())
    assert ok, (rel, worst)


def test_swiglu_elementwise(bz):
    import torch
    rng = np.random.default_rng(3)
    M, F = 3, 1000
    y = (rng.normal(0, 2, (M, 2 * F))).astype(np.float16)
    h = torch.empty((M, F), dtype=torch.float16, device="cuda")
    bz.bonsai_swiglu(torch.from_numpy(y.view(np.int16)).cuda().view(torch.float16), h, M, F)
    torch.cuda.synchronize()
    # exact inputs: FP32 arithmetic and one FP16 rounding of h
    ref = oracle.swiglu(y.astype(np.float64))
    got = to_numpy_f16(h)
    assert np.all(np.abs(got - ref) <= 2.0 ** -10 * np.abs(ref) + 1e-6)


def test_swiglu_fused_repeatable_and_near_unfused(bz):
    """The fused epilogue (FP32 sums into silu) gives the same bits on every call, split
    row tiles included, and stays within FP16 rounding of linear-then-SwiGLU."""
    import torch
    F, K = 17408, 5120
    p = Problem(1, 2 * F, K, PQ2, seed=21)
    a = _run_swiglu(bz, p, F)
    b = _run_swiglu(bz, p, F)
    assert np.array_equal(a, b)
    x, packed, scales = p.device()
    y = torch.empty((1, 2 * F), dtype=torch.float16, device="cuda")
    bz.bonsai_ternary_linear(x, packed, scales, y, 1, 2 * F, K, PQ2)
    h = torch.empty((1, F), dtype=torch.float16, device="cuda")
    bz.bonsai_swiglu(y, h, 1, F)
    torch.cuda.synchronize()
    ok, rel, worst = swiglu_ok(to_numpy_f16(h), p.oracle_y())
    assert ok, (rel, worst)
    assert swiglu_ok(a, p.oracle_y())[0]


def test_swiglu_gemm_full_size_sampled(bz):
    """Prefill M=2048 through the fused gate/up 5120 -> 2 x 17408 with SwiGLU in the GEMM's
    epilogue; 48 x 48 sampled outputs against the checker."""
    import torch
    from ternary_weight_02_b200 import inputs
    M, F, K, seed = 2048, 17408, 5120, 8
    dev = torch.device("cuda")
    t = torch.from_numpy(inputs.trits(seed, 2 * F, K)).to(dev)
    packed = bz.pack(PQ2, t)
    del t
    s = torch.from_numpy(inputs.scales(seed, 2 * F, K).view(np.int16)).to(dev).view(torch.float16)
    x = torch.from_numpy(inputs.activations(seed, M, K).view(np.int16)).to(dev).view(torch.float16)
    h = torch.full((M, F), float("nan"), dtype=torch.float16, device=dev)
    bz.bonsai_ternary_linear_swiglu(x, packed, s, h, M, F, K, PQ2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    ms = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 46)]))
    fs = np.unique(np.concatenate([[0, F - 1], rng.integers(0, F, 46)]))
    rows = np.concatenate([fs, F + fs])  # the gate rows, then the matching up rows
    xr = inputs.normal_rows(seed, K, ms)
    w = inputs.trits_rows(seed, K, rows)
    sc = inputs.scales_rows(seed, K // 128, rows)
    y_ref = oracle.ternary_linear(xr, oracle.pack(PQ2, w), sc, len(rows), K, PQ2)
    got = h[torch.from_numpy(ms).to(dev)][:, torch.from_numpy(fs).to(dev)].float().cpu().numpy()
    ok, rel, worst = swiglu_ok(got, y_ref)
    assert ok, (rel, worst)
    assert bool(torch.isfinite(h).all())
