// common.cuh -- device helpers shared by the libbonsai kernels.
//
// The block Hadamard rotation (source: "27B 模型压到 5.95GB，推理能力还保住 98%",
// allhereai.com, the method paragraph and the paragraph on running the files;
// "Bonsai 2，把27B压进6个G", 10100.com, section 它怎么做到的) is applied to each run
// of 128 activations: x'[i] = sum_j Hn[i][j] x[j], Hn[i][j] = (-1)^popcount(i&j)/sqrt(128).
// The fast Walsh-Hadamard transform below computes it with 7 butterfly stages
// (one per index bit), which is the Sylvester matrix in natural order.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace bonsai {

constexpr int kGroup = 128;           // weights per FP16 scale == Hadamard block size
constexpr int kPtq1GroupBytes = 26;   // 25 bytes x 5 trits + 1 byte x 3 trits
constexpr int kPq2GroupBytes = 32;    // 128 trits x 2 bits
constexpr int kQ1GroupBytes = 16;     // 128 signs x 1 bit
constexpr float kHadamardNorm = 0.088388347648318440550f;  // 1/sqrt(128)

// Programmatic dependent launch.  pdl_launch_dependents lets the next kernel on the stream
// start its set-up; pdl_wait returns once the kernel in front has finished and its memory
// is visible.  Both return at once for a kernel launched without the
// programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// Asynchronous global -> shared copies (cp.async).  The _zfill forms copy the n bytes when
// `valid` and write n zero bytes otherwise (the source is then not read).
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async8_zfill(void *dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 8 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t float_to_half_bits(float f) {
    return __half_as_ushort(__float2half_rn(f));
}

// One 128-block held by a warp, lane l holding elements 4l .. 4l+3 in v[0..3].
// On return v holds the same positions of Hn * block (FP32 throughout).
__device__ __forceinline__ void fwht128_warp(float v[4], int lane) {
    // index bits 0 and 1 live inside the lane
    const float a0 = v[0] + v[1], a1 = v[0] - v[1];
    const float a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[2] = a0 - a2;
    v[1] = a1 + a3;
    v[3] = a1 - a3;
    // index bits 2..6 are lane bits 0..4: butterfly (a, b) -> (a + b, a - b)
#pragma unroll
    for (int b = 0; b < 5; b++) {
        const int mask = 1 << b;
        const bool upper = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float p = __shfl_xor_sync(0xffffffffu, v[i], mask);
            v[i] = upper ? (p - v[i]) : (v[i] + p);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) v[i] *= kHadamardNorm;
}

// Loads 4 consecutive FP16 values (8 bytes, 8-byte aligned) as floats.
__device__ __forceinline__ void load_half4(const uint16_t *p, float v[4]) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __half2 h01 = *reinterpret_cast<const __half2 *>(&raw.x);
    const __half2 h23 = *reinterpret_cast<const __half2 *>(&raw.y);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    v[0] = f01.x;
    v[1] = f01.y;
    v[2] = f23.x;
    v[3] = f23.y;
}

__device__ __forceinline__ void store_half4(uint16_t *p, const float v[4]) {
    const __half2 h01 = __floats2half2_rn(v[0], v[1]);
    const __half2 h23 = __floats2half2_rn(v[2], v[3]);
    uint2 raw;
    raw.x = *reinterpret_cast<const uint32_t *>(&h01);
    raw.y = *reinterpret_cast<const uint32_t *>(&h23);
    *reinterpret_cast<uint2 *>(p) = raw;
}

// One 128-block of x rotated by a warp into FP16 (nearest even), lane l storing outputs
// 4l .. 4l+3 of the block.  kPerm: 0 natural order; 8: each 8 consecutive outputs in the
// order [0, 4, 1, 5, 2, 6, 3, 7]; 16: each 16 in the order [0, 8, 1, 9, ..., 7, 15].  The
// prefill GEMM expands its PQ2_0 (8) or Q1_0 (16) weights in the same order within each
// block (a contraction does not depend on the order of its terms), which lets it build
// two FP16 weights with one byte permute.
// rotate_store_f16 takes the lane's four inputs already loaded (as load_half4 gives them).
template <int kPerm>
__device__ __forceinline__ void rotate_store_f16(float (&v)[4], uint16_t *__restrict__ out, int64_t blk, int lane) {
    fwht128_warp(v, lane);
    float o[4];
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
        o[0] = odd ? a[2] : a[0];
        o[1] = odd ? b[2] : b[0];
        o[2] = odd ? a[3] : a[1];
        o[3] = odd ? b[3] : b[1];
    } else if (kPerm == 8) {
        // lanes 2b, 2b + 1 hold outputs 8b .. 8b + 7; the even lane stores
        // (0, 4, 1, 5), the odd one (2, 6, 3, 7)
        const bool odd = lane & 1;
        const float r0 = __shfl_xor_sync(0xffffffffu, odd ? v[0] : v[2], 1);
        const float r1 = __shfl_xor_sync(0xffffffffu, odd ? v[1] : v[3], 1);
        if (odd) {
            o[0] = r0, o[1] = v[2], o[2] = r1, o[3] = v[3];
        } else {
            o[0] = v[0], o[1] = r0, o[2] = v[1], o[3] = r1;
        }
    } else {
        o[0] = v[0], o[1] = v[1], o[2] = v[2], o[3] = v[3];
    }
    store_half4(out + blk * kGroup + 4 * lane, o);
}

template <int kPerm>
__device__ __forceinline__ void rotate_block_f16(const uint16_t *__restrict__ x, uint16_t *__restrict__ out,
                                                 int64_t blk, int lane) {
    float v[4];
    load_half4(x + blk * kGroup + 4 * lane, v);
    rotate_store_f16<kPerm>(v, out, blk, lane);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace bonsai
