"""The bench's algorithmic byte counts (the numerator of its GB/s figures), recomputed
from the packings' definitions: PTQ1_0 26 bytes per 128-weight group, PQ2_0 one byte per
4 weights, Q1_0 one byte per 8 weights, one FP16 scale per 128 weights (64 for the g64
variant), plus the FP16 x and y of one token."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# (K, N) of the four projections, and the trit + scale bytes of each per packing
EXPECTED = {
    (5120, 34816): {1: 38_993_920, 2: 47_349_760},   # gate/up
    (17408, 5120): {1: 19_496_960, 2: 23_674_880},   # down
    (5120, 7168): {1: 8_028_160, 2: 9_748_480},      # qkv
    (5120, 5120): {1: 5_734_400, 2: 6_963_200},      # o
}


def test_plane_bytes_per_projection():
    for (K, N), want in EXPECTED.items():
        for fmt, b in want.items():
            assert bench.plane_bytes(fmt, N, K) == b
        # Q1_0: an eighth of a byte per weight; g64: PQ2_0's plane with twice the scales
        assert bench.plane_bytes(3, N, K) == N * K // 8 + N * (K // 128) * 2
        assert bench.plane_bytes(4, N, K) == N * K // 4 + N * (K // 64) * 2


def test_step_bytes_are_64_layers_of_weights_x_and_y():
    for fmt in (1, 2):
        weights = 64 * sum(EXPECTED[(K, N)][fmt] for _, K, N in bench.SHAPES)
        xy = 64 * sum(2 * K + 2 * N for _, K, N in bench.SHAPES)
        assert bench.step_bytes(fmt) == weights + xy
    assert 64 * sum(EXPECTED[(K, N)][1] for _, K, N in bench.SHAPES) == 4_624_220_160
    assert 64 * sum(EXPECTED[(K, N)][2] for _, K, N in bench.SHAPES) == 5_615_124_480


def test_whole_job_rate():
    assert abs(bench.whole_job_gbs(bench.step_bytes(2), 1, 2.0) - bench.step_bytes(2) / 2e-3 / 1e9) < 1e-6
    assert abs(bench.whole_job_gbs(10**9, 8, 1.0) - 8000.0) < 1e-9


def test_clock_samples_median_and_reasons():
    idle, cap = 0x1, 0x4
    samples = [(1965, 1965, 0), (1950, 1965, cap), (1965, 1965, cap | idle), (0, 1965, 0), (None, None, 0)]
    c = bench.summarize_clock_samples(samples)
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    thermal = [(1400, 1965, 0x8 | 0x40 | 0x20)]
    assert bench.summarize_clock_samples(thermal)["reasons"] == [
        "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clock_samples([]) is None
