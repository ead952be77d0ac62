"""Pins of the CPU checker against what the pages and the mathematics fix.

Each test checks the checker against something other than itself: values worked
out by hand from the pages (tests/golden), library routines that compute the same
quantity another way (numpy base-3 strings, Kronecker products, matmul), closed
forms and invariants.  Plausible slips -- a wrong digit order, a dropped group
scale, a transposed operand, a wrong Hadamard sign, an off-by-one block -- each
fail at least one test here.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
from ternary_weight_02_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PTQ1, PQ2, Q1 = oracle.FMT_PTQ1_0, oracle.FMT_PQ2_0, oracle.FMT_Q1_0
G64 = oracle.FMT_PQ2_0_G64


def _weights(fmt, seed, N, K):
    """Seeded weights a format can hold: trits, or signs for the 1-bit Q1_0."""
    return inputs.signs(seed, N, K) if fmt == Q1 else inputs.trits(seed, N, K)


def _golden_codec():
    rows = []
    with open(os.path.join(GOLDEN, "codec_examples.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if line:
                rows.append((line[0], [int(v) for v in line[1:-1]], int(line[-1])))
    return rows


def _golden_sizes():
    out = {}
    with open(os.path.join(GOLDEN, "pages_sizes.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if line:
                out[line[0]] = float(line[1])
    return out


# ---------------------------------------------------------------- codecs

def _ptq1_group(prefix_pos, trits):
    """A one-row, one-group trit vector with `trits` placed at weight 5*prefix_pos."""
    t = np.zeros((1, 128), dtype=np.int8)
    t[0, 5 * prefix_pos:5 * prefix_pos + len(trits)] = trits
    return t


def test_codec_hand_worked_bytes():
    for fmt, trits, byte in _golden_codec():
        if fmt == "ptq1":
            # 5-trit examples go to byte 0, 3-trit examples to the last byte (25)
            pos = 0 if len(trits) == 5 else 25
            t = _ptq1_group(pos, trits)
            packed = oracle.pack(PTQ1, t)
            assert packed.shape == (1, 26)
            assert int(packed[0, pos]) == byte, (trits, int(packed[0, pos]))
        else:
            t = np.zeros((1, 128), dtype=np.int8)
            t[0, 8:12] = trits  # byte 2 of the row
            packed = oracle.pack(PQ2, t)
            assert packed.shape == (1, 32)
            assert int(packed[0, 2]) == byte, (trits, int(packed[0, 2]))


def test_ptq1_all_243_codes_match_base3_library():
    # np.base_repr gives the base-3 digits most significant first; the format
    # stores the first weight as the least significant digit, with digit = trit + 1.
    for v in range(243):
        digits = [int(c) for c in np.base_repr(v, base=3).rjust(5, "0")][::-1]
        t = _ptq1_group(0, [d - 1 for d in digits])
        packed = oracle.pack(PTQ1, t)
        assert int(packed[0, 0]) == v
        back, bad = oracle.unpack(PTQ1, packed, 1, 128)
        assert bad == 0
        assert list(back[0, :5]) == [d - 1 for d in digits]


def test_ptq1_all_trit_tuples_round_trip():
    tuples = np.array(list(itertools.product([-1, 0, 1], repeat=5)), dtype=np.int8)
    assert tuples.shape == (243, 5)
    # 243 tuples laid out as 243 rows x byte 0 of one group each
    t = np.zeros((243, 128), dtype=np.int8)
    t[:, :5] = tuples
    packed = oracle.pack(PTQ1, t)
    assert sorted(packed[:, 0].tolist()) == list(range(243))  # a bijection onto 0..242
    back, bad = oracle.unpack(PTQ1, packed, 243, 128)
    assert bad == 0 and np.array_equal(back, t)


def test_ptq1_last_byte_27_codes():
    tuples = np.array(list(itertools.product([-1, 0, 1], repeat=3)), dtype=np.int8)
    t = np.zeros((27, 128), dtype=np.int8)
    t[:, 125:] = tuples
    packed = oracle.pack(PTQ1, t)
    assert sorted(packed[:, 25].tolist()) == list(range(27))  # padding digits are zero
    back, bad = oracle.unpack(PTQ1, packed, 27, 128)
    assert bad == 0 and np.array_equal(back, t)
    assert oracle.check(PTQ1, packed, 27, 128) == 0


def test_ptq1_invalid_bytes_rejected():
    packed = np.full((1, 26), 121, dtype=np.uint8)  # all-zero trits, canonical
    packed[0, 25] = 13  # (0, 0, 0) in the last byte
    assert oracle.check(PTQ1, packed, 1, 128) == 0
    for v in range(243, 256):
        p = packed.copy()
        p[0, 3] = v
        t, bad = oracle.unpack(PTQ1, p, 1, 128)
        assert bad == 1
        assert np.all(t[0, 15:20] == oracle.INVALID_TRIT)
        assert oracle.check(PTQ1, p, 1, 128) == 1
    p = packed.copy()
    p[0, 25] = 27  # padding digit 3 set: decodes, but is not canonical
    t, bad = oracle.unpack(PTQ1, p, 1, 128)
    assert bad == 0 and list(t[0, 125:]) == [-1, -1, -1]
    assert oracle.check(PTQ1, p, 1, 128) == 1


def test_pq2_all_81_codes_round_trip_and_invalid_175():
    valid = []
    for v in range(256):
        codes = [(v >> (2 * i)) & 3 for i in range(4)]
        t, bad = oracle.unpack(PQ2, np.full((1, 32), v, dtype=np.uint8), 1, 128)
        if 3 in codes:
            assert bad == 32 * codes.count(3)
            assert oracle.check(PQ2, np.array([[v] * 32], dtype=np.uint8), 1, 128) == 32 * codes.count(3)
        else:
            valid.append(v)
            assert bad == 0
            assert list(t[0, :4]) == [c - 1 for c in codes]
            assert np.array_equal(oracle.pack(PQ2, t), np.full((1, 32), v, dtype=np.uint8))
    assert len(valid) == 81


def test_pack_marks_invalid_trits():
    t = np.zeros((1, 128), dtype=np.int8)
    t[0, 7] = 2
    p1 = oracle.pack(PTQ1, t)
    assert int(p1[0, 1]) == 0xFF and oracle.check(PTQ1, p1, 1, 128) == 1
    p2 = oracle.pack(PQ2, t)
    assert (int(p2[0, 1]) >> 6) & 3 == 3 and oracle.check(PQ2, p2, 1, 128) == 1


def test_random_round_trip_both_formats():
    t = inputs.trits(7, 5, 1024)
    for fmt in (PTQ1, PQ2):
        packed = oracle.pack(fmt, t)
        back, bad = oracle.unpack(fmt, packed, 5, 1024)
        assert bad == 0 and np.array_equal(back, t)
        assert oracle.check(fmt, packed, 5, 1024) == 0


def test_row_layout_is_row_major_groups():
    # Row n, group g of PTQ1_0 starts at byte (n*G + g)*26; of PQ2_0 at n*K/4 + 32g.
    N, K = 3, 384
    t = np.zeros((N, K), dtype=np.int8)
    t[2, 256] = 1  # row 2, group 2, first weight
    p1 = oracle.pack(PTQ1, t).reshape(-1)
    nz = np.nonzero(p1 != oracle.pack(PTQ1, np.zeros_like(t)).reshape(-1))[0]
    assert nz.tolist() == [(2 * 3 + 2) * 26]
    p2 = oracle.pack(PQ2, t).reshape(-1)
    nz = np.nonzero(p2 != oracle.pack(PQ2, np.zeros_like(t)).reshape(-1))[0]
    assert nz.tolist() == [2 * K // 4 + 64]


# ---------------------------------------------------------------- sizes

def test_bits_per_weight_match_pages():
    pages = _golden_sizes()
    K = 5120
    scale_bits = 16 / 128
    bpw1 = oracle.packed_bytes(PTQ1, 1, K) * 8 / K + scale_bits
    bpw2 = oracle.packed_bytes(PQ2, 1, K) * 8 / K + scale_bits
    assert bpw1 == 1.75 and round(bpw1, 2) == pages["ptq1_bits_per_weight"]
    assert bpw2 == 2.125 and round(bpw2 + 1e-9, 2) == pages["pq2_bits_per_weight"]
    # unpadded base-3 storage: 8/5 bits per trit (the pages' bound) + the scale
    assert abs(8 / 5 - pages["trit_bound_bits"]) < 1e-12
    unpadded = 8 / 5 + scale_bits
    assert pages["true_bits_per_weight"] <= unpadded + 0.01 and unpadded <= bpw1
    # the file-size ratio of the two packings matches the padded layout
    ratio_pages = pages["pq2_file_gb"] / pages["ptq1_file_gb"]
    assert abs(ratio_pages - bpw2 / bpw1) < 0.005
    assert abs(ratio_pages - bpw2 / unpadded) > 0.015
    # both files imply the same ~27e9 weights
    n1 = pages["ptq1_file_gb"] * 8e9 / bpw1
    n2 = pages["pq2_file_gb"] * 8e9 / bpw2
    assert 26.5e9 < n1 < 27.5e9 and 26.5e9 < n2 < 27.5e9 and abs(n1 - n2) / n1 < 0.01


def test_packed_bytes_bad_shapes():
    assert oracle.packed_bytes(PTQ1, 4, 100) == -1
    assert oracle.packed_bytes(5, 4, 128) == -1
    assert oracle.packed_bytes(PQ2, 0, 128) == 0
    assert oracle.packed_bytes(Q1, 4, 256) == 128 and oracle.packed_bytes(Q1, 1, 64) == -1


def test_q1_bits_per_weight_match_pages():
    # one bit per weight plus one FP16 scale per 128: 1.125, the 1-bit family's figure
    pages = _golden_sizes()
    K = 5120
    bpw = oracle.packed_bytes(Q1, 1, K) * 8 / K + 16 / 128
    assert bpw == 1.125 == pages["q1_bits_per_weight"]
    # the 3.9 GB file then holds ~27.7e9 weights at that rate: the 27B model (the file
    # also carries the unquantised parts, so the count is an upper bound)
    n = pages["q1_file_gb"] * 8e9 / bpw
    assert 26.5e9 < n < 28.5e9


def test_q1_all_256_bytes_round_trip():
    # bit i of byte b is weight 8b + i: 1 -> +1, 0 -> -1 (least significant first)
    for v in range(256):
        t, bad = oracle.unpack(Q1, np.full((1, 16), v, dtype=np.uint8), 1, 128)
        assert bad == 0
        want = np.array([1 if (v >> i) & 1 else -1 for i in range(8)] * 16, dtype=np.int8)
        assert np.array_equal(t[0], want)
        assert np.array_equal(oracle.pack(Q1, t), np.full((1, 16), v, dtype=np.uint8))
        assert oracle.check(Q1, np.full((1, 16), v, dtype=np.uint8), 1, 128) == 0


def test_q1_pack_counts_non_binary_and_stores_minus_one():
    t = np.ones((2, 128), dtype=np.int8)
    t[0, 3] = 0
    t[1, 127] = 2
    p = oracle.pack(Q1, t)
    assert p[0, 0] == 0xF7 and p[1, 15] == 0x7F
    u, bad = oracle.unpack(Q1, p, 2, 128)
    assert u[0, 3] == -1 and u[1, 127] == -1 and bad == 0
    assert int(oracle.lib().oracle_pack_q1(oracle._ptr(t), oracle._ptr(np.zeros(32, np.uint8)), 2, 128)) == 2


# ---------------------------------------------------------------- Hadamard

def test_sylvester_matches_kronecker_definition():
    H2 = np.array([[1.0, 1.0], [1.0, -1.0]])
    H = np.array([[1.0]])
    for _ in range(7):
        H = np.kron(H2, H)  # H_2n = [[H_n, H_n], [H_n, -H_n]]
    assert np.array_equal(oracle.sylvester128() * np.sqrt(128.0), H)


def test_sylvester_orthonormal_symmetric():
    Hn = oracle.sylvester128()
    Hi = np.rint(Hn * np.sqrt(128.0)).astype(np.int64)
    assert np.array_equal(Hi @ Hi.T, 128 * np.eye(128, dtype=np.int64))
    assert np.array_equal(Hn, Hn.T)
    assert np.allclose(Hn @ Hn, np.eye(128), atol=1e-14)
    assert np.all(Hi[0] == 1) and np.all(Hi[:, 0] == 1)


def test_hadamard_norm_involution_and_recursive_route():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 512))
    xr = oracle.hadamard128(x)
    assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.allclose(oracle.hadamard128(xr), x, atol=1e-12)
    for m in range(3):
        for b in range(4):
            blk = x[m, 128 * b:128 * (b + 1)]
            want = oracle.fwht_recursive(blk) / np.sqrt(128.0)
            assert np.allclose(xr[m, 128 * b:128 * (b + 1)], want, atol=1e-13)
    # library matmul on the block-reshaped matrix
    H = oracle.sylvester128()
    assert np.allclose(xr, (x.reshape(3, 4, 128) @ H.T).reshape(3, 512), atol=1e-13)


def test_hadamard_blocks_do_not_mix():
    x = np.zeros((1, 384))
    x[0, 128 + 5] = 1.0  # a delta inside block 1
    xr = oracle.hadamard128(x)
    assert np.all(xr[0, :128] == 0) and np.all(xr[0, 256:] == 0)
    H = oracle.sylvester128()
    assert np.allclose(xr[0, 128:256], H[:, 5], atol=0)
    # closed forms: delta at 0 -> flat 1/sqrt(128); flat ones -> sqrt(128) e_0
    x = np.zeros((1, 128)); x[0, 0] = 1.0
    assert np.allclose(oracle.hadamard128(x), 1 / np.sqrt(128), atol=1e-15)
    x = np.ones((1, 128))
    e0 = np.zeros((1, 128)); e0[0, 0] = np.sqrt(128)
    assert np.allclose(oracle.hadamard128(x), e0, atol=1e-13)


def test_rotation_identity_dense():
    # Folding the rotation into the weights and rotating the input gives back W0 x
    # ("10100.com" page, section 它怎么做到的: rotation keeps the information; the
    # input must get the matching transform).
    rng = np.random.default_rng(2)
    K, N = 384, 5
    W0 = rng.standard_normal((N, K))
    x = rng.standard_normal((2, K))
    B = np.kron(np.eye(K // 128), oracle.sylvester128())  # blockdiag(Hn)
    xr = oracle.hadamard128(x)
    assert np.allclose(xr, x @ B.T, atol=1e-12)
    assert np.allclose(xr @ (W0 @ B.T).T, x @ W0.T, atol=1e-11)


# ---------------------------------------------------------------- linear

def _dense(trits, scales):
    """Dequantised weight Wdeq[n][k] = s[n][k // 128] * t[n][k] (float64)."""
    return trits.astype(np.float64) * np.repeat(scales.astype(np.float64), 128, axis=1)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2, Q1])
@pytest.mark.parametrize("N,K,M", [(1, 128, 1), (3, 256, 2), (8, 128, 3), (5, 384, 1)])
def test_linear_brute_force_dense(fmt, N, K, M):
    t = _weights(fmt, 11, N, K)
    s = inputs.scales(11, N, K)
    x = inputs.activations(11, M, K)
    y = oracle.ternary_linear(x, oracle.pack(fmt, t), s, N, K, fmt)
    H = oracle.sylvester128()
    xr = (x.astype(np.float64).reshape(M, K // 128, 128) @ H.T).reshape(M, K)
    want = xr @ _dense(t, s).T
    assert y.shape == (M, N)
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt", [PTQ1, PQ2])
def test_linear_hand_cases(fmt):
    K = 256
    s = np.array([[0.5, 0.25]], dtype=np.float16)
    x = inputs.activations(3, 1, K)
    xr = oracle.hadamard128(x.astype(np.float64))
    # all +1: y = sum_g s_g * sum(x' in group g)
    t = np.ones((1, K), dtype=np.int8)
    y = oracle.ternary_linear(x, oracle.pack(fmt, t), s, 1, K, fmt)
    assert np.isclose(y[0, 0], 0.5 * xr[0, :128].sum() + 0.25 * xr[0, 128:].sum(), rtol=1e-13)
    # all zero: y = 0
    t = np.zeros((1, K), dtype=np.int8)
    assert oracle.ternary_linear(x, oracle.pack(fmt, t), s, 1, K, fmt)[0, 0] == 0.0
    # one -1 at k = 200 (group 1): y = -0.25 * x'[200]
    t[0, 200] = -1
    y = oracle.ternary_linear(x, oracle.pack(fmt, t), s, 1, K, fmt)
    assert np.isclose(y[0, 0], -0.25 * xr[0, 200], rtol=1e-14)
    # x = delta at the start of block 1, all trits +1: x' = 1/sqrt(128) over block 1,
    # so y = 0.25 * 128 / sqrt(128) = 0.25 * sqrt(128)
    xd = np.zeros((1, K), dtype=np.float16); xd[0, 128] = 1
    t = np.ones((1, K), dtype=np.int8)
    y = oracle.ternary_linear(xd, oracle.pack(fmt, t), s, 1, K, fmt)
    assert np.isclose(y[0, 0], 0.25 * np.sqrt(128.0), rtol=1e-14)


# ---------------------------------------------------------------- PQ2_0 with 64-weight scale groups

def test_g64_plane_and_bits():
    # the codes are PQ2_0's byte for byte; only the scale plane doubles
    t = inputs.trits(2, 3, 256)
    assert np.array_equal(oracle.pack(G64, t), oracle.pack(PQ2, t))
    assert oracle.packed_bytes(G64, 3, 256) == oracle.packed_bytes(PQ2, 3, 256) == 192
    assert oracle.packed_bytes(G64, 1, 5120) * 8 / 5120 + 16 / 64 == 2.25
    assert oracle.scale_group(G64) == 64 and oracle.scale_group(PQ2) == 128


def test_g64_hand_case_halves():
    # all trits +1, K = 128, scales (a, b): y = a * sum x'[:64] + b * sum x'[64:]
    x = inputs.activations(4, 1, 128)
    xr = oracle.hadamard128(x.astype(np.float64))
    s = np.array([[0.5, -0.125]], dtype=np.float16)
    y = oracle.ternary_linear(x, oracle.pack(G64, np.ones((1, 128), np.int8)), s, 1, 128, G64)
    assert np.isclose(y[0, 0], 0.5 * xr[0, :64].sum() - 0.125 * xr[0, 64:].sum(), rtol=1e-13)


def test_g64_equals_pq2_with_paired_scales():
    N, K, M = 9, 640, 2
    t = inputs.trits(5, N, K)
    S = inputs.scales(5, N, K)
    s64 = np.repeat(S, 2, axis=1)  # both halves of a 128-group carry its scale
    x = inputs.activations(5, M, K)
    y2 = oracle.ternary_linear(x, oracle.pack(PQ2, t), S, N, K, PQ2)
    y64 = oracle.ternary_linear(x, oracle.pack(G64, t), s64, N, K, G64)
    assert np.allclose(y64, y2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("N,K,M", [(1, 128, 1), (4, 384, 2)])
def test_g64_brute_force_dense(N, K, M):
    t = inputs.trits(13, N, K)
    s = inputs.scales_rows(13, K // 64, np.arange(N))
    x = inputs.activations(13, M, K)
    y = oracle.ternary_linear(x, oracle.pack(G64, t), s, N, K, G64)
    H = oracle.sylvester128()
    xr = (x.astype(np.float64).reshape(M, K // 128, 128) @ H.T).reshape(M, K)
    W = t.astype(np.float64) * np.repeat(s.astype(np.float64), 64, axis=1)
    assert np.allclose(y, xr @ W.T, rtol=1e-12, atol=1e-12)


def test_linear_q1_hand_cases():
    K = 256
    s = np.array([[0.5, 0.25]], dtype=np.float16)
    x = inputs.activations(3, 1, K)
    xr = oracle.hadamard128(x.astype(np.float64))
    full = 0.5 * xr[0, :128].sum() + 0.25 * xr[0, 128:].sum()
    t = np.ones((1, K), dtype=np.int8)
    assert np.isclose(oracle.ternary_linear(x, oracle.pack(Q1, t), s, 1, K, Q1)[0, 0], full, rtol=1e-13)
    # all -1: the negation
    assert np.isclose(oracle.ternary_linear(x, oracle.pack(Q1, -t), s, 1, K, Q1)[0, 0], -full, rtol=1e-13)
    # one weight flipped to -1 at k = 200 (group 1): y = full - 2 * 0.25 * x'[200]
    t[0, 200] = -1
    y = oracle.ternary_linear(x, oracle.pack(Q1, t), s, 1, K, Q1)
    assert np.isclose(y[0, 0], full - 0.5 * xr[0, 200], rtol=1e-12)


def test_linear_q1_agrees_with_ternary_formats_on_signs():
    # weights +-1 are valid in all three packings: the three decodes give one result
    N, K, M = 17, 384, 3
    t = inputs.signs(6, N, K)
    s = inputs.scales(6, N, K)
    x = inputs.activations(6, M, K)
    yq = oracle.ternary_linear(x, oracle.pack(Q1, t), s, N, K, Q1)
    for fmt in (PTQ1, PQ2):
        assert np.array_equal(yq, oracle.ternary_linear(x, oracle.pack(fmt, t), s, N, K, fmt))


def test_signs_generator():
    t = inputs.signs(1, 64, 1024)
    assert set(np.unique(t)) == {-1, 1} and abs(float((t == 1).mean()) - 0.5) < 0.01
    assert np.array_equal(inputs.signs_rows(1, 1024, [5, 63]), t[[5, 63]])


# ---------------------------------------------------------------- SwiGLU

def test_swiglu_closed_forms():
    z = np.array([[0.0, 1.0, -1.0, 40.0, -40.0, 2.0,  # gate
                   3.0, 1.0, 2.0, 0.5, 7.0, -1.0]])   # up
    h = oracle.swiglu(z)[0]
    e1 = np.exp(-1.0)
    assert h[0] == 0.0
    assert h[1] == 1.0 / (1.0 + e1) * 1.0           # silu(1) = sigma(1)
    assert np.isclose(h[2], -1.0 * (1.0 - 1.0 / (1.0 + e1)) * 2.0, rtol=1e-15)
    assert np.isclose(h[3], 40.0 * 0.5, rtol=1e-15)  # sigma(40) = 1 to double precision
    assert np.isclose(h[4], -280.0 * np.exp(-40.0), rtol=1e-14)  # sigma(-40) = e^-40 (1 - e^-40 ...)
    assert np.isclose(h[5], 2.0 / (1.0 + np.exp(-2.0)) * -1.0, rtol=1e-15)


def test_swiglu_odd_identity_and_layout():
    # silu(z) - silu(-z) = z for every z; gate is the first half of the columns
    rng = np.random.default_rng(0)
    g = rng.normal(0, 3, (3, 50))
    ones = np.ones_like(g)
    hp = oracle.swiglu(np.concatenate([g, ones], axis=1))
    hm = oracle.swiglu(np.concatenate([-g, ones], axis=1))
    assert np.allclose(hp - hm, g, rtol=0, atol=1e-13)
    # swapping the halves changes the result (the layout is pinned, not symmetric)
    u = rng.normal(0, 3, (3, 50))
    assert not np.allclose(oracle.swiglu(np.concatenate([g, u], 1)), oracle.swiglu(np.concatenate([u, g], 1)))


@pytest.mark.parametrize("fmt", [PQ2, PTQ1])
def test_swiglu_linear_brute_force(fmt):
    F, K, M = 6, 256, 3
    t = _weights(fmt, 9, 2 * F, K)
    s = inputs.scales(9, 2 * F, K)
    x = inputs.activations(9, M, K)
    h = oracle.swiglu_linear(x, oracle.pack(fmt, t), s, F, K, fmt)
    H = oracle.sylvester128()
    xr = (x.astype(np.float64).reshape(M, K // 128, 128) @ H.T).reshape(M, K)
    y = xr @ _dense(t, s).T
    gate, up = y[:, :F], y[:, F:]
    want = gate * (1.0 / (1.0 + np.exp(-gate))) * up
    assert h.shape == (M, F)
    assert np.allclose(h, want, rtol=1e-12, atol=1e-13)


def test_linear_formats_agree_and_threads_agree():
    N, K, M = 33, 640, 2
    t = inputs.trits(5, N, K)
    s = inputs.scales(5, N, K)
    x = inputs.activations(5, M, K)
    y1 = oracle.ternary_linear(x, oracle.pack(PTQ1, t), s, N, K, PTQ1, nthreads=1)
    y2 = oracle.ternary_linear(x, oracle.pack(PQ2, t), s, N, K, PQ2, nthreads=3)
    assert np.array_equal(y1, y2)


def test_negative_skipping_hadamard_fails_tolerance():
    # Without the input-side transform the output is silent garbage ("allhereai"
    # page, paragraph on running the files; "10100.com" page, 它怎么做到的).
    N, K = 64, 1024
    t = inputs.trits(0, N, K)
    s = inputs.scales(0, N, K)
    x = inputs.activations(0, 1, K)
    p = oracle.pack(PQ2, t)
    y = oracle.ternary_linear(x, p, s, N, K, PQ2)
    y_bad = oracle.ternary_linear(x, p, s, N, K, PQ2, apply_hadamard=False)
    ok, rel, _ = oracle.compare(y_bad, y)
    assert not ok and rel > 0.5
    assert oracle.compare(y, y)[0]


def test_compare_bar():
    y = np.array([1.0, -2.0, 3.0, 0.5])
    assert oracle.compare(y, y)[0]
    assert oracle.compare(y * (1 + 5e-4), y)[0]
    assert not oracle.compare(y * (1 + 2e-3), y)[0]
    z = y.copy(); z[0] += 0.05  # one outlier beyond 1e-2 * rms
    assert not oracle.compare(z, y)[0]
    assert not oracle.compare(np.array([np.nan, 0, 0, 0]), y)[0]
