// gemm_tcgen05.cu -- prefill ternary GEMM on the 5th-generation tensor cores.
//
// y[m][n] = sum_k x'[m][k] * s[n][k/128] * t[n][k] for M tokens at once: a dense
// contraction (2*M*N*K FLOP), so it runs as an FP16 x FP16 -> FP32 tcgen05 MMA with the
// accumulator in tensor memory.  Sources: "27B 模型压到 5.95GB，推理能力还保住 98%"
// (allhereai.com): method paragraph (trits, FP16 scale per 128 weights, block
// Hadamard), packings paragraph (PQ2_0 wins prompt processing); "Bonsai 2，把27B压进6个G"
// (10100.com), section 它怎么做到的 (the input takes the matching transform).
//
// Two launches per call:
//  1. the block-Hadamard rotation x -> x' (FP16, round to nearest) into the workspace
//     (hadamard.cu).  Rotating inside the GEMM would redo each 128 x 128 A tile's FWHT
//     for every one of the N/256 column tiles; as a pass it costs one read and one
//     write of x, under 1% of the GEMM's time at these shapes.
//  2. this kernel.  A CTA computes one 128 x 256 tile of y over all of K in 64-wide
//     stages (4-stage ring):
//     - warp 0 (one thread): TMA loads of the x' tile (128 rows x 64, 128-byte swizzle);
//     - warp 1: allocates 256 TMEM columns; one thread issues tcgen05.mma
//       (M=128, N=256, K=16, kind::f16, FP32 accumulate) and commits each stage back;
//     - warps 2..9 (256 threads, one weight row each): expand the packed trits of a
//       128-weight group times its FP16 scale into two 64-wide FP16 B stages, written
//       in the same 128-byte-swizzled K-major layout the MMA descriptors describe
//       (t * s is exact in FP16); then the epilogue: tcgen05.ld of the accumulator,
//       FP32 -> FP16 (nearest even), stores to y.
// Every wait is bounded: if one gives up, the CTA stops issuing work, waits for the
// copies and MMAs it started, frees its tensor memory and writes NaN to its tile.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace bonsai {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;  // BM: rows of one MMA / one TMEM accumulator
constexpr int kExpandWarps = 8;
constexpr int kThreads = (2 + kExpandWarps) * 32;  // 320
constexpr int B_STAGE_BYTES = BN * BK * 2;         // 32 KB

// Tile configuration: kAcc accumulators of 128 rows each share every B stage (the
// expanded weights), so the CTA covers 128 * kAcc rows of y.
template <int kAcc>
struct Cfg {
    static constexpr int kStages = kAcc == 2 ? 3 : 4;
    static constexpr int kTileM = BM * kAcc;
    static constexpr int kAStage = kTileM * BK * 2;  // 16 or 32 KB
    static constexpr int kTmemCols = 256 * kAcc;
    // shared memory: [A stages][B stages][barriers][tmem slot][abort flag][PTQ1_0 LUT]
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kStages * kAStage;
    static constexpr int kOffBar = kOffB + kStages * B_STAGE_BYTES;
    static constexpr int kNumBars = 3 * kStages + 1;  // full_a, full_b, empty, done
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 8;
    static constexpr int kOffLut = kOffAbort + 8;
    static constexpr int kSmemBytes = kOffLut + 256 * 4 + 1024;  // + slack for the 1024-B tile base
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle: rows of
// 128 bytes, 8-row atoms 1024 bytes apart (SBO), version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                 // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: next 8-row atom
    d |= (uint64_t)1 << 46;                 // descriptor version
    d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor: D F32, A and B F16, both K-major, N = BN, M = BM.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- trit expansion

// One 32-bit word of 2-bit codes (code c_i = trit + 1 at bits 2i, weights w0 .. w0+15)
// times the scale, as two 16-byte chunks of FP16: out[0..3] = weights w0..w0+7,
// out[4..7] = weights w0+8..w0+15.  A code placed in the mantissa of 1024.0
// (0x6400) reads as 1024 + c; subtracting 1025 gives the trit exactly and the
// multiply by the FP16 scale is exact (the product is 0 or +-s).
__device__ __forceinline__ void expand_word(uint32_t w, __half2 s2, uint32_t (&out)[8]) {
    const __half2 bias = __halves2half2(__ushort_as_half(0x6401), __ushort_as_half(0x6401));  // 1025
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        // low half: code i, high half: code i + 8
        const uint32_t m = ((w >> (2 * i)) & 0x00030003u) | 0x64006400u;
        __half2 v = __hsub2(*reinterpret_cast<const __half2 *>(&m), bias);
        v = __hmul2(v, s2);
        h[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        out[i] = __byte_perm(h[2 * i], h[2 * i + 1], 0x5410);      // low halves: codes 2i, 2i+1
        out[4 + i] = __byte_perm(h[2 * i], h[2 * i + 1], 0x7632);  // high halves: codes 2i+8, 2i+9
    }
}

// Stores one 16-byte chunk (8 halves) of row r of a B stage at its swizzled place.
__device__ __forceinline__ void st_chunk(uint8_t *stage, int r, int chunk, const uint32_t *v) {
    uint4 *p = reinterpret_cast<uint4 *>(stage + r * 128 + ((chunk ^ (r & 7)) << 4));
    *p = make_uint4(v[0], v[1], v[2], v[3]);
}

// Raw packed bytes of one 128-weight group of row n (PQ2_0: 32 bytes; PTQ1_0: 26 bytes
// in 7 words) and its FP16 scale, loaded a group ahead of their decode.
struct GroupRaw {
    uint32_t w[8];
    uint16_t scale;
};

template <int kFmt>
__device__ __forceinline__ void load_group(const uint8_t *packed, const uint16_t *scales, int64_t n, int64_t G,
                                           int64_t g, GroupRaw &raw) {
    raw.scale = __ldg(scales + n * G + g);
    if (kFmt == 2) {
        const uint4 *p = reinterpret_cast<const uint4 *>(packed + (n * G + g) * kPq2GroupBytes);
        const uint4 a = __ldg(p), b = __ldg(p + 1);
        raw.w[0] = a.x, raw.w[1] = a.y, raw.w[2] = a.z, raw.w[3] = a.w;
        raw.w[4] = b.x, raw.w[5] = b.y, raw.w[6] = b.z, raw.w[7] = b.w;
    } else {
        // 26 bytes at an even address: 6 aligned words and one aligned half-word
        const uint8_t *src = packed + (n * G + g) * kPtq1GroupBytes;
        if ((reinterpret_cast<uintptr_t>(src) & 3u) == 0) {
            const uint32_t *q = reinterpret_cast<const uint32_t *>(src);
#pragma unroll
            for (int i = 0; i < 6; i++) raw.w[i] = __ldg(q + i);
            raw.w[6] = __ldg(reinterpret_cast<const unsigned short *>(src + 24));
        } else {
            const uint32_t lo = __ldg(reinterpret_cast<const unsigned short *>(src));
            const uint32_t *q = reinterpret_cast<const uint32_t *>(src + 2);
            uint32_t t[6];
#pragma unroll
            for (int i = 0; i < 6; i++) t[i] = __ldg(q + i);
            raw.w[0] = lo | (t[0] << 16);
#pragma unroll
            for (int i = 1; i < 6; i++) raw.w[i] = __funnelshift_r(t[i - 1], t[i], 16);
            raw.w[6] = t[5] >> 16;
        }
        raw.w[7] = 0u;
    }
}

// Codes of the group as 8 words (word i: weights 16i .. 16i+15, code = trit + 1).
template <int kFmt>
__device__ __forceinline__ void group_codes(const GroupRaw &raw, const uint32_t *lut, uint32_t (&cw)[8]) {
    if (kFmt == 2) {
#pragma unroll
        for (int i = 0; i < 8; i++) cw[i] = raw.w[i];
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) cw[i] = 0u;
        // byte b's five digits become codes 5b .. 5b+4 (2 bits each, bit 10b of the
        // 256-bit code stream); the padding digits of byte 25 fall past bit 255
#pragma unroll
        for (int b = 0; b < kPtq1GroupBytes; b++) {
            const uint32_t f = lut[(raw.w[b >> 2] >> (8 * (b & 3))) & 0xFFu];
            const int pos = 10 * b, wi = pos >> 5, sh = pos & 31;
            cw[wi] |= f << sh;
            if (sh > 22 && wi + 1 < 8) cw[wi + 1] |= f >> (32 - sh);
        }
    }
}

// ---------------------------------------------------------------- kernel

template <int kFmt, int kAcc>
__global__ void __launch_bounds__(kThreads, 1) gemm_tcgen05_kernel(
    const __grid_constant__ CUtensorMap a_map, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, int M, int N, int K) {
    using C = Cfg<kAcc>;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the tile area (128-byte swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + C::kOffA;
    uint8_t *sB = smem + C::kOffB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *full_a = bars, *full_b = bars + STAGES, *empty = bars + 2 * STAGES, *done = bars + 3 * STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem + C::kOffLut);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile_m = blockIdx.x, tile_n = blockIdx.y;
    const int num_k = K / BK;
    const int64_t G = K / kGroup;

    if (tid == 0) {
        for (int st = 0; st < STAGES; st++) {
            mbar_init(full_a + st, 1);
            mbar_init(full_b + st, kExpandWarps);
            mbar_init(empty + st, 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (kFmt == 1) {  // byte -> its five base-3 digits as 2-bit codes (code i at bits 2i)
        for (int b = tid; b < 256; b += kThreads) {
            uint32_t f = 0;
            int v = b < 243 ? b : 0;
            for (int i = 0; i < 5; i++) {
                f |= (uint32_t)(v % 3) << (2 * i);
                v /= 3;
            }
            lut[b] = f;
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                     "r"(C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (x' tiles)
        if (lane == 0) {
            int issued = 0;
            for (int ks = 0; ks < num_k; ks++) {
                const int st = ks % STAGES;
                const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
                if (*abort_flag || !mbar_wait(empty + st, ph ^ 1u)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full_a + st, C::kAStage);
#pragma unroll
                for (int a = 0; a < kAcc; a++)
                    tma_load_2d(sA + st * C::kAStage + a * (BM * BK * 2), &a_map, full_a + st, ks * BK,
                                tile_m * C::kTileM + a * BM);
                issued = ks + 1;
            }
            // the copies this thread started land before the CTA may exit
            for (int ks = issued - STAGES < 0 ? 0 : issued - STAGES; ks < issued; ks++)
                mbar_wait(full_a + (ks % STAGES), (uint32_t)(ks / STAGES) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int ks = 0; ks < num_k; ks++) {
                const int st = ks % STAGES;
                const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
                if (*abort_flag || !mbar_wait(full_a + st, ph) || !mbar_wait(full_b + st, ph)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t b0 = saddr(sB + st * B_STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; kk++) {
                    const uint64_t bdesc = desc_sw128(b0 + kk * 32);
#pragma unroll
                    for (int a = 0; a < kAcc; a++) {
                        const uint32_t a0 = saddr(sA + st * C::kAStage + a * (BM * BK * 2));
                        mma_f16(tmem + (uint32_t)(a * 256), desc_sw128(a0 + kk * 32), bdesc,
                                (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(empty + st);  // frees the stage when these MMAs have read it
            }
            mma_commit(done);  // all MMAs issued by this thread are complete
        }
    } else {
        // ------------------------------------------------ trit expansion (one row per thread)
        const int r = tid - 64;                      // 0 .. 255: row of the B tile
        const int64_t n = (int64_t)tile_n * BN + r;  // weight row
        const bool valid = n < N;
        GroupRaw cur, nxt;
        if (valid) load_group<kFmt>(packed, scales, n, G, 0, cur);
        uint32_t cw[8];
        __half2 s2 = __float2half2_rn(0.f);
        for (int ks = 0; ks < num_k; ks++) {
            const int g = ks >> 1, hf = ks & 1;  // a 128-weight group fills two 64-wide stages
            if (hf == 0) {
                if (valid && g + 1 < (int)G) load_group<kFmt>(packed, scales, n, G, g + 1, nxt);  // in flight
                if (valid) {
                    group_codes<kFmt>(cur, lut, cw);
                    const __half sh = __ushort_as_half(cur.scale);
                    s2 = __halves2half2(sh, sh);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; i++) cw[i] = 0x55555555u;  // all trits zero
                }
            }
            const int st = ks % STAGES;
            const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
            // every lane acquires the stage itself; the verdict is made warp-uniform
            const bool free_ok = !*abort_flag && mbar_wait(empty + st, ph ^ 1u);
            if (!__all_sync(0xffffffffu, free_ok)) {
                *abort_flag = 1;
                break;
            }
            uint8_t *stage = sB + st * B_STAGE_BYTES;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                uint32_t out[8];
                expand_word(hf ? cw[4 + i] : cw[i], s2, out);  // weights 64hf + 16i .. +15
                st_chunk(stage, r, 2 * i, out);
                st_chunk(stage, r, 2 * i + 1, out + 4);
            }
            // make the generic-proxy stores visible to the tensor core, then signal
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(full_b + st);
            if (hf == 1) cur = nxt;
        }

        // ------------------------------------------------ epilogue
        const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0)) && !*abort_flag;
        tc_fence_after();
        const int q = warp & 3;            // TMEM lane quadrant this warp may read
        const int half = (warp - 2) >> 2;  // which 128 columns
#pragma unroll 1
        for (int a = 0; a < kAcc; a++) {
            const int m = tile_m * C::kTileM + a * BM + 32 * q + lane;
#pragma unroll 1
            for (int c = 0; c < 4; c++) {
                const int col = half * 128 + 32 * c;
                uint32_t v[32];
                __syncwarp();
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256 + col), v);
                if (m >= M) continue;
                const int64_t n0 = (int64_t)tile_n * BN + col;
                uint16_t *yr = y + (int64_t)m * N + n0;
                if (ok && n0 + 32 <= N && (N & 7) == 0) {
                    uint32_t h[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const __half2 p2 =
                            __floats2half2_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        h[i] = *reinterpret_cast<const uint32_t *>(&p2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(yr);
#pragma unroll
                    for (int i = 0; i < 4; i++) dst[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
                } else {
                    for (int i = 0; i < 32; i++)
                        if (n0 + i < N) yr[i] = ok ? float_to_half_bits(__uint_as_float(v[i])) : (uint16_t)0x7E00u;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------- host side

}  // namespace

bool gemm_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    (void)fmt;
    // TMA coordinates and the grid are 32-bit; the rows of x' must be 16-byte multiples
    return M >= 1 && M < (int64_t)1 << 30 && N < (int64_t)1 << 30 && K % kGroup == 0 && K < (int64_t)1 << 30;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt) {
    (void)N;
    (void)fmt;
    return (size_t)M * (size_t)K * 2;  // x' in FP16
}

cudaError_t launch_gemm(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int tile_hint,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    uint16_t *xr = reinterpret_cast<uint16_t *>(ws.data);
    cudaError_t err = launch_hadamard_f16(x, xr, M, K, s, dev);
    if (err != cudaSuccess) return err;

    EncodeTiledFn encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, BM};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    // one or two 128-row accumulators per CTA: two halve the trit expansion per FLOP; pick
    // the one whose grid wastes less of the last wave
    const int64_t nt = (N + BN - 1) / BN;
    auto wave_eff = [&](int64_t tiles) {
        const int64_t waves = (tiles + dev.sm_count - 1) / dev.sm_count;
        return (double)tiles / (double)(waves * dev.sm_count);
    };
    const int64_t t1 = ((M + BM - 1) / BM) * nt, t2 = ((M + 2 * BM - 1) / (2 * BM)) * nt;
    const bool two = tile_hint == 2 || (tile_hint != 1 && M > BM && wave_eff(t2) * 1.35 >= wave_eff(t1));
    auto go = [&](auto kern, int acc, int smem) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const dim3 grid((unsigned)((M + (int64_t)BM * acc - 1) / ((int64_t)BM * acc)), (unsigned)nt);
        kern<<<grid, kThreads, smem, s>>>(map, packed, scales, y, (int)M, (int)N, (int)K);
        return cudaGetLastError();
    };
    if (fmt == 1)
        return two ? go(gemm_tcgen05_kernel<1, 2>, 2, Cfg<2>::kSmemBytes) : go(gemm_tcgen05_kernel<1, 1>, 1, Cfg<1>::kSmemBytes);
    return two ? go(gemm_tcgen05_kernel<2, 2>, 2, Cfg<2>::kSmemBytes) : go(gemm_tcgen05_kernel<2, 1>, 1, Cfg<1>::kSmemBytes);
}

}  // namespace bonsai
