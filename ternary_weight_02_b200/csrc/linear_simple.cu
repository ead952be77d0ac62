// linear_simple.cu -- the plain CUDA ternary linear layer (any M, every packing).
//
// y[m][n] = sum_g s[n][g] * sum_j t[n][128g+j] * x'[m][128g+j], x' the block
// Hadamard rotation of x.  Source: "27B 模型压到 5.95GB，推理能力还保住 98%"
// (allhereai.com), method paragraph and packings paragraph.
//
// Two launches: the rotation writes x' in FP32 to the workspace, then one warp
// per (row n, 4 tokens) walks the row's groups (lane = group), decodes each trit
// with scalar arithmetic and accumulates in FP32.  It makes no attempt at speed;
// it is the straightforward device path every faster kernel is compared with,
// and the fallback for shapes the specialised kernels do not take.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kTokensPerWarp = 4;

template <int kFmt>
__global__ void __launch_bounds__(256) linear_simple_kernel(
    const float *__restrict__ xr, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, int64_t M, int64_t N,
    int64_t K) {
    const int lane = threadIdx.x & 31;
    const int64_t G = K / kGroup;
    const int64_t mchunks = (M + kTokensPerWarp - 1) / kTokensPerWarp;
    const int64_t tasks = N * mchunks;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t task = warp; task < tasks; task += nwarps) {
        const int64_t n = task / mchunks;
        const int64_t m0 = (task - n * mchunks) * kTokensPerWarp;
        float acc[kTokensPerWarp] = {0.f, 0.f, 0.f, 0.f};
        for (int64_t g = lane; g < G; g += 32) {
            float dot[kTokensPerWarp] = {0.f, 0.f, 0.f, 0.f};
            float dot_hi[kTokensPerWarp] = {0.f, 0.f, 0.f, 0.f};  // PQ2_0 g64: weights 64 .. 127
            for (int j = 0; j < kGroup; j++) {
                int t;
                if (kFmt == 1) {
                    int v = packed[(n * G + g) * kPtq1GroupBytes + j / 5];
                    for (int d = 0; d < j % 5; d++) v /= 3;
                    t = v % 3 - 1;
                } else if (kFmt == 3) {
                    const int v = packed[n * (K / 8) + g * kQ1GroupBytes + j / 8];
                    t = ((v >> (j % 8)) & 1) ? 1 : -1;
                } else {
                    const int v = packed[n * (K / 4) + g * kPq2GroupBytes + j / 4];
                    t = ((v >> (2 * (j % 4))) & 3) - 1;
                }
                for (int i = 0; i < kTokensPerWarp; i++)
                    if (m0 + i < M) {
                        const float p = (float)t * xr[(m0 + i) * K + g * kGroup + j];
                        if (kFmt == 4 && j >= 64)
                            dot_hi[i] += p;
                        else
                            dot[i] += p;
                    }
            }
            if (kFmt == 4) {  // two scales per 128 weights
                const float s0 = half_bits_to_float(scales[n * 2 * G + 2 * g]);
                const float s1 = half_bits_to_float(scales[n * 2 * G + 2 * g + 1]);
                for (int i = 0; i < kTokensPerWarp; i++) acc[i] += s0 * dot[i] + s1 * dot_hi[i];
            } else {
                const float sc = half_bits_to_float(scales[n * G + g]);
                for (int i = 0; i < kTokensPerWarp; i++) acc[i] += sc * dot[i];
            }
        }
        for (int i = 0; i < kTokensPerWarp; i++) {
            const float total = warp_sum(acc[i]);
            if (lane == 0 && m0 + i < M) y[(m0 + i) * N + n] = float_to_half_bits(total);
        }
    }
}

}  // namespace

size_t simple_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    (void)N;
    return (size_t)M * (size_t)K * sizeof(float);
}

cudaError_t launch_linear_simple(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                 uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt,
                                 const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    float *xr = reinterpret_cast<float *>(ws.data);
    cudaError_t err = launch_hadamard_f32(x, xr, M, K, s, dev);
    if (err != cudaSuccess) return err;
    const int64_t tasks = N * ((M + kTokensPerWarp - 1) / kTokensPerWarp);
    const int64_t want = (tasks + 7) / 8;
    const int64_t cap = (int64_t)dev.sm_count * 16;
    const int grid = (int)(want < cap ? want : cap);
    if (fmt == 1)
        linear_simple_kernel<1><<<grid, 256, 0, s>>>(xr, packed, scales, y, M, N, K);
    else if (fmt == 3)
        linear_simple_kernel<3><<<grid, 256, 0, s>>>(xr, packed, scales, y, M, N, K);
    else if (fmt == 4)
        linear_simple_kernel<4><<<grid, 256, 0, s>>>(xr, packed, scales, y, M, N, K);
    else
        linear_simple_kernel<2><<<grid, 256, 0, s>>>(xr, packed, scales, y, M, N, K);
    return cudaGetLastError();
}

}  // namespace bonsai
