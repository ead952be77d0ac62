"""The C-ABI library without a GPU: it loads, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bonsai.h")


@pytest.fixture(scope="module")
def bz():
    from ternary_weight_02_b200 import build
    build.build()
    from ternary_weight_02_b200 import bonsai
    return bonsai


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(bonsai_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("bonsai_pack_ptq1", "bonsai_pack_pq2", "bonsai_hadamard128",
                     "bonsai_ternary_linear", "bonsai_unpack", "bonsai_packed_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(bz):
    lib = bz.raw()
    for name in declared_functions():
        assert hasattr(lib, name), name
    with open("/proc/self/maps") as f:
        assert any(bz.LIB_PATH in line for line in f)


def test_packed_bytes_host_arithmetic(bz):
    assert bz.bonsai_packed_bytes(bz.BONSAI_FMT_PTQ1_0, 5120, 17408) == 5120 * 136 * 26
    assert bz.bonsai_packed_bytes(bz.BONSAI_FMT_PQ2_0, 34816, 5120) == 34816 * 1280
    assert bz.bonsai_packed_bytes(bz.BONSAI_FMT_Q1_0, 34816, 5120) == 34816 * 640
    assert bz.bonsai_packed_bytes(bz.BONSAI_FMT_PQ2_0_G64, 34816, 5120) == 34816 * 1280  # PQ2_0's plane
    assert bz.raw().bonsai_packed_bytes(bz.BONSAI_FMT_PQ2_0, 4, 100) == bz.BONSAI_ERR_SHAPE
    assert bz.raw().bonsai_packed_bytes(7, 4, 128) == bz.BONSAI_ERR_FMT
    assert bz.raw().bonsai_packed_bytes(1, -1, 128) == bz.BONSAI_ERR_SHAPE


def test_host_validation_needs_no_gpu(bz):
    L = bz.raw()
    good = 1 << 20  # an aligned non-null value; validation rejects before it is used
    # NULL pointers
    assert L.bonsai_ternary_linear(None, good, good, good, 1, 8, 128, 2, None) == bz.BONSAI_ERR_NULL
    assert L.bonsai_pack_pq2(good, None, 4, 128, None) == bz.BONSAI_ERR_NULL
    assert L.bonsai_hadamard128(None, good, 1, 128, None) == bz.BONSAI_ERR_NULL
    # shapes
    assert L.bonsai_ternary_linear(good, good, good, good, 1, 8, 100, 2, None) == bz.BONSAI_ERR_SHAPE
    assert L.bonsai_ternary_linear(good, good, good, good, -1, 8, 128, 2, None) == bz.BONSAI_ERR_SHAPE
    assert L.bonsai_ternary_linear(good, good, good, good, 1, 8, 0, 2, None) == bz.BONSAI_ERR_SHAPE
    assert L.bonsai_hadamard128(good, good, 2, 64, None) == bz.BONSAI_ERR_SHAPE
    # format
    assert L.bonsai_ternary_linear(good, good, good, good, 1, 8, 128, 0, None) == bz.BONSAI_ERR_FMT
    assert L.bonsai_unpack(5, good, good, 1, 128, None) == bz.BONSAI_ERR_FMT
    # alignment
    assert L.bonsai_ternary_linear(good + 2, good, good, good, 1, 8, 128, 2, None) == bz.BONSAI_ERR_ALIGN
    assert L.bonsai_pack_ptq1(good, good + 8, 4, 128, None) == bz.BONSAI_ERR_ALIGN
    # algorithm choice that cannot take the shape
    assert (L.bonsai_ternary_linear_algo(good, good, good, good, 1, 8, 128, 2, 99, 0, None)
            == bz.BONSAI_ERR_ALGO)
    # the status query needs somewhere to write
    assert L.bonsai_device_status(None, None, 0) == bz.BONSAI_ERR_NULL
    # empty problems are accepted and launch nothing
    assert L.bonsai_ternary_linear(None, None, None, None, 0, 8, 128, 2, None) == bz.BONSAI_OK
    assert L.bonsai_pack_pq2(None, None, 0, 128, None) == bz.BONSAI_OK


def test_integer_gemv_batch_limits_on_the_host(bz):
    """The integer tensor-core GEMV takes PQ2_0 and g64 at M = 1 (K <= 24576), M = 2
    (K <= 12288) and, for PQ2_0, M = 3 (K <= 6144); an explicit request past those
    limits is refused on the host, before any device is touched.  Within them the call
    gets as far as the device (none here, or the GPU's answer)."""
    import torch
    L = bz.raw()
    good = 1 << 20
    IMMA, PQ2, G64, PTQ1 = bz.BONSAI_ALGO_IMMA, bz.BONSAI_FMT_PQ2_0, bz.BONSAI_FMT_PQ2_0_G64, bz.BONSAI_FMT_PTQ1_0

    def call(M, K, fmt):
        return L.bonsai_ternary_linear_algo(good, good, good, good, M, 64, K, fmt, IMMA, 0, None)
    for M, K, fmt in [(4, 1024, PQ2), (2, 12288 + 128, PQ2), (3, 6144 + 128, PQ2), (3, 1024, G64),
                      (1, 24576 + 128, PQ2), (1, 1024, PTQ1), (2, 1024, PTQ1)]:
        assert call(M, K, fmt) == bz.BONSAI_ERR_ALGO, (M, K, fmt)
    if not torch.cuda.is_available():
        for M, K, fmt in [(1, 24576, PQ2), (2, 12288, PQ2), (2, 12288, G64), (3, 6144, PQ2)]:
            assert call(M, K, fmt) == bz.BONSAI_ERR_CUDA, (M, K, fmt)


def test_binding_constants_match_the_header(bz):
    """Every enumerator and BONSAI_DEVICE_* bit the header defines has the same value in
    the Python binding, and the binding defines no other BONSAI_ constant."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    header = {n: int(v) for n, v in re.findall(r"\b(BONSAI_[A-Z0-9_]+)\s*=\s*(-?\d+)", text)}
    header.update({n: int(v) for n, v in re.findall(r"#define\s+(BONSAI_DEVICE_[A-Z0-9_]+)\s+(\d+)u", text)})
    assert len(header) >= 24  # 4 formats, 10 status codes, 6 kernel choices, 4 device bits
    binding = {n: getattr(bz, n) for n in dir(bz) if n.startswith("BONSAI_") and isinstance(getattr(bz, n), int)}
    assert binding == header


def test_status_strings(bz):
    for code in range(-9, 1):
        s = bz.bonsai_status_string(code)
        assert s and s != "unknown status"
    assert bz.bonsai_status_string(-99) == "unknown status"
    assert bz.bonsai_version() >= (0 << 16) | (1 << 8)


def test_no_device_reports_cuda_error(bz):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    good = 1 << 20
    assert bz.bonsai_check_device() == bz.BONSAI_ERR_CUDA
    assert bz.raw().bonsai_ternary_linear(good, good, good, good, 1, 8, 128, 2, None) == bz.BONSAI_ERR_CUDA


def test_every_entry_point_is_documented():
    """Each function the header declares is preceded by its own comment block (the
    operation, argument layouts, ownership and error behaviour live there)."""
    text = open(HEADER).read()
    for name in declared_functions():
        m = re.search(r"(/\*(?:(?!\*/).)*\*/)\s*(?:[A-Za-z_][A-Za-z0-9_ ]*[ *])" + name + r"\s*\(", text, flags=re.S)
        assert m is not None, f"{name} has no comment block right before its declaration"
        assert len(m.group(1)) > 40, name
