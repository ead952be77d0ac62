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

// kPerm (FP16 output only): the output order of rotate_block_f16 (common.cuh).
template <bool kOutF32, int kPerm>
__global__ void __launch_bounds__(256) hadamard128_kernel(const uint16_t *x, void *out,
                                                          int64_t nblocks) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t blk = warp; blk < nblocks; blk += nwarps) {
        if (kOutF32) {
            float v[4];
            load_half4(x + blk * kGroup + 4 * lane, v);
            fwht128_warp(v, lane);
            float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(out) + blk * kGroup) + lane;
            *o = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            rotate_block_f16<kPerm>(x, static_cast<uint16_t *>(out), blk, lane);
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

cudaError_t launch_hadamard_f32(const uint16_t *x, float *out, int64_t M, int64_t K,
                                cudaStream_t s, const DeviceInfo &dev) {
    return launch<true>(x, out, M, K, s, dev);
}

}  // namespace bonsai
