"""The seeded input generator: published SplitMix64 outputs, independence of
element order, and the stated distributions."""
import numpy as np

from ternary_weight_02_b200 import inputs

_MASK = (1 << 64) - 1


def _splitmix64_sequential(state, count):
    """Plain-integer SplitMix64 as published (state += gamma; mix)."""
    out = []
    for _ in range(count):
        state = (state + 0x9E3779B97F4A7C15) & _MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_seed0_outputs():
    # first outputs of SplitMix64 seeded with 0 (Vigna's reference splitmix64.c)
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    assert _splitmix64_sequential(0, 4) == want
    got = inputs.raw_u64(np.uint64(0), np.arange(4, dtype=np.uint64))
    assert [int(v) for v in got] == want


def test_counter_based_matches_sequential_stream():
    key = inputs.stream_key(123, inputs.STREAM_X)
    assert int(key) == _splitmix64_sequential(123, inputs.STREAM_X + 1)[-1]
    seq = _splitmix64_sequential(int(key), 50)
    got = inputs.raw_u64(key, np.arange(50, dtype=np.uint64))
    assert [int(v) for v in got] == seq


def test_rows_are_order_independent():
    full = inputs.trits(3, 20, 256)
    part = inputs.trits_rows(3, 256, [17, 2, 9])
    assert np.array_equal(part, full[[17, 2, 9]])
    xs = inputs.activations(3, 6, 256)
    assert np.array_equal(inputs.normal_rows(3, 256, [5, 0]), xs[[5, 0]])
    ss = inputs.scales(3, 10, 512)
    assert np.array_equal(inputs.scales_rows(3, 4, [9]), ss[[9]])
    # one scale per 64 weights: a 10 x 8 plane whose rows regenerate alone
    s64 = inputs.scales(3, 10, 512, group=64)
    assert s64.shape == (10, 8) and np.array_equal(inputs.scales_rows(3, 8, [9, 0]), s64[[9, 0]])


def test_distributions():
    t = inputs.trits(0, 256, 4096)
    n = t.size
    p0 = np.count_nonzero(t == 0) / n
    pm = np.count_nonzero(t == -1) / n
    pp = np.count_nonzero(t == 1) / n
    assert abs(p0 - 0.38) < 0.003 and abs(pm - 0.31) < 0.003 and abs(pp - 0.31) < 0.003
    s = inputs.scales(0, 512, 4096).astype(np.float64)
    assert s.min() >= 0.0099 and s.max() <= 0.0501 and abs(s.mean() - 0.03) < 0.001
    x = inputs.activations(0, 64, 4096).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert x.dtype == np.float64 and inputs.activations(0, 1, 128).dtype == np.float16


def test_seeds_and_streams_differ():
    a = inputs.trits(0, 4, 128)
    assert not np.array_equal(a, inputs.trits(1, 4, 128))
    assert not np.array_equal(a, inputs.trits(0, 4, 128, stream_id=9))
