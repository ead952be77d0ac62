// hadamard.cu -- standalone block-Hadamard(128) rotation of activations.
//
// x'[m, 128b + i] = sum_j Hn[i][j] x[m, 128b + j], Hn = H_128 / sqrt(128), Sylvester
// order.  Source: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com), method
// paragraph (block Hadamard rotation) and paragraph on running the files (the
// activation-side Hadamard runtime); "Bonsai 2，把27B压进6个G" (10100.com), section
// 它怎么做到的 (the input must receive the matching transform).
//
// HBM-bound: 2 bytes read + 2 (or 4) bytes written per element.  One warp per
// 128-block, 8-byte loads (a warp moves 256 contiguous bytes), FP32 butterflies
// in registers and shuffles, grid = a multiple of the SM count.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

// kPerm (FP16 output only): 0 natural order; 8: each 8 consecutive outputs in the order
// [0, 4, 1, 5, 2, 6, 3, 7]; 16: each 16 in the order [0, 8, 1, 9, ..., 7, 15].  The
// prefill GEMM expands its PQ2_0 (8) or Q1_0 (16) weights in the same order within each
// block (a contraction does not depend on the order of its terms), which lets it build
// two FP16 weights with one byte permute.
template <bool kOutF32, int kPerm>
__global__ void __launch_bounds__(256) hadamard128_kernel(const uint16_t *x, void *out,
                                                          int64_t nblocks) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t blk = warp; blk < nblocks; blk += nwarps) {
        float v[4];
        load_half4(x + blk * kGroup + 4 * lane, v);
        fwht128_warp(v, lane);
        if (kOutF32) {
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + blk * kGroup) + lane;
            *o = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            if (kPerm == 16) {
                // lanes 4b .. 4b+3 hold outputs 16b .. 16b+15; lane r of the four stores
                // (e, e + 8, e + 1, e + 9) with e = 4 (r >> 1) + 2 (r & 1): elements e, e + 1
                // of lane r >> 1 and of lane 2 + (r >> 1)
                const int base = lane & ~3, r = lane & 3;
                const int la = base + (r >> 1), lb = base + 2 + (r >> 1);
                float a[4], b[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    a[k] = __shfl_sync(0xffffffffu, v[k], la);
                    b[k] = __shfl_sync(0xffffffffu, v[k], lb);
                }
                const bool odd = r & 1;
                float o[4];
                o[0] = odd ? a[2] : a[0];
                o[1] = odd ? b[2] : b[0];
                o[2] = odd ? a[3] : a[1];
                o[3] = odd ? b[3] : b[1];
                store_half4(static_cast<uint16_t *>(out) + blk * kGroup + 4 * lane, o);
            } else if (kPerm == 8) {
                // lanes 2b, 2b + 1 hold outputs 8b .. 8b + 7; the even lane stores
                // (0, 4, 1, 5), the odd one (2, 6, 3, 7)
                const bool odd = lane & 1;
                const float r0 = __shfl_xor_sync(0xffffffffu, odd ? v[0] : v[2], 1);
                const float r1 = __shfl_xor_sync(0xffffffffu, odd ? v[1] : v[3], 1);
                float o[4];
                if (odd) {
                    o[0] = r0, o[1] = v[2], o[2] = r1, o[3] = v[3];
                } else {
                    o[0] = v[0], o[1] = r0, o[2] = v[1], o[3] = r1;
                }
                store_half4(static_cast<uint16_t *>(out) + blk * kGroup + 4 * lane, o);
            } else {
                store_half4(static_cast<uint16_t *>(out) + blk * kGroup + 4 * lane, v);
            }
        }
    }
}

template <bool kOutF32, int kPerm = 0>
cudaError_t launch(const uint16_t *x, void *out, int64_t M, int64_t K, cudaStream_t s,
                   const DeviceInfo &dev) {
    const int64_t nblocks = M * (K / kGroup);
    if (nblocks == 0) return cudaSuccess;
    const int64_t want = (nblocks + 7) / 8;  // 8 warps per CTA
    const int64_t cap = (int64_t)dev.sm_count * 8;
    const int grid = (int)(want < cap ? want : cap);
    hadamard128_kernel<kOutF32, kPerm><<<grid, 256, 0, s>>>(x, out, nblocks);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard_f16(const uint16_t *x, uint16_t *out, int64_t M, int64_t K,
                                cudaStream_t s, const DeviceInfo &dev) {
    return launch<false>(x, out, M, K, s, dev);
}

cudaError_t launch_hadamard_f16_perm8(const uint16_t *x, uint16_t *out, int64_t M, int64_t K,
                                      cudaStream_t s, const DeviceInfo &dev) {
    return launch<false, 8>(x, out, M, K, s, dev);
}

cudaError_t launch_hadamard_f16_perm16(const uint16_t *x, uint16_t *out, int64_t M, int64_t K,
                                       cudaStream_t s, const DeviceInfo &dev) {
    return launch<false, 16>(x, out, M, K, s, dev);
}

cudaError_t launch_hadamard_f32(const uint16_t *x, float *out, int64_t M, int64_t K,
                                cudaStream_t s, const DeviceInfo &dev) {
    return launch<true>(x, out, M, K, s, dev);
}

}  // namespace bonsai
