// skinny_mma.cu -- ternary linear layer for small batches (1 <= M <= 16 tokens): PQ2_0
// with one FP16 scale per 128 or per 64 weights, and the 1-bit Q1_0 packing.
//
// y[m][n] = sum_g s[n][g] * sum_j t[n][128g+j] * x'[m][128g+j].  Sources: "27B 模型压到
// 5.95GB，推理能力还保住 98%" (allhereai.com): method paragraph (trits, FP16 group
// scale, block Hadamard) and packings paragraph (PQ2_0: one trit per 2-bit slot).
//
// With M >= 2 every weight byte is used by several tokens, which takes the work past
// what FP32 FMAs can do at HBM speed, so the products run on the tensor cores
// (mma.sync m16n8k16, FP16 in, FP32 accumulate) with the weights dequantised in
// registers -- nothing but x' goes through shared memory.
//
// * Codes as FP16 subnormals.  A PQ2_0 byte holds codes c = t + 1 of 4 weights.  One
//   byte permute copies byte t of a weight word into both halves of a register; two
//   masks (0x000C0003, 0x00C00030) then leave codes (c0, c1) and (c2, c3) in place,
//   where an FP16 bit pattern with a zero exponent reads as c * 4^j * 2^-24.  The
//   matching activations are stored pre-scaled by 4^-j (exact), so each MMA adds
//   2^-24 * sum c * x' in FP32.  The lane's k slots are permuted (the same
//   permutation on both operands) so that its four slots are one byte of a word.
// * Per 128-weight group the MMA starts from zero; the epilogue adds
//   s[n][g] * (2^24 * D - sum_j x'[m][j]) (the second term turns codes into trits).
// * Each lane reads only the 8 bytes of a row's group that its MMA slots use (words 2tq,
//   2tq + 1).  With K a multiple of 1024 (PQ2_0, g64, Q1_0) the weights and scales come
//   by TMA into a ring of two stages of 8 groups per warp (4 KB of codes, 128-byte
//   swizzle), so the copies in flight hold no registers and no per-thread load slots;
//   otherwise (and for PTQ1_0) the lane keeps kRing groups in flight in a ring of
//   registers whose slots are addressed by constants.
// * x' (FWHT prepass, FP16) of the CTA's K chunk sits in shared memory as
//   [k-step][token][16 halves], 4^-(k mod 4)-scaled and in the MMAs' K order, so a
//   lane's B fragment is one 8-byte load from a contiguous 256-byte row.
// * A warp owns 16 weight rows; a CTA 128 rows and one K chunk.  Split-K: chunks
//   write FP32 partials; the warp that brings a row block's last chunk sums them in
//   chunk order (deterministic) and writes y.
// * 64-weight scales (PQ2_0 g64, the Q2_0_g64 files of "Bonsai把 27B 大模型塞进手机的极端
//   量化方案到底靠不靠谱" (wmrh.cn), sections 快速上手 and 后端支持现状): lane quad member tq
//   takes words tq and tq + 4 of the group instead of 2tq and 2tq + 1, so that MMAs 0-3
//   cover the group's first 64 weights and MMAs 4-7 the last 64; each half has its own
//   accumulator, scale and sum of x'.
// * Q1_0 (weights +-1 as bits, "Bonsai把 27B 大模型塞进手机的极端量化方案到底靠不靠谱"
//   (wmrh.cn), sections 核心观点 and 关键机制): lane quad member tq takes word tq of the
//   16-byte group; MMA i uses nibble i & 1 of byte i >> 1, bits left in place as FP16
//   subnormals b * 2^j * 2^-24 (j = 0..7 within the byte) against x' pre-scaled by 2^-j,
//   and the epilogue adds s * (2 * 2^24 * D - sum x'), which turns bits b into 2b - 1.
// * PTQ1_0 (5 trits per base-3 byte, 26 bytes per 128-weight group; the allhereai.com
//   page's packings paragraph).  A byte's base-3 digits are the trits plus one, i.e.
//   PQ2_0's codes, so a 256-entry shared-memory table turns each byte into its five 2-bit
//   codes and the lane assembles the same two code words (weights 32tq .. 32tq + 31) the
//   PQ2_0 path loads; everything after that is PQ2_0's.  The lane's 7 or 8 bytes of a row's
//   group (from byte 32tq / 5) come as three aligned 32-bit loads.
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tma.cuh"  // kSpinLimit: the bound of every wait; TMA and mbarrier wrappers

namespace bonsai {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerCta = kWarps * 16;
constexpr int kRing = 8;  // groups of weights in flight per warp (register ring)

// groups of x' staged in shared memory at a time: 96 KB for either token tile count
template <int NT>
constexpr int sub_groups() { return NT == 1 ? 48 : 24; }

// TMA ring (PQ2_0, g64, Q1_0 with K a multiple of 1024): per warp kTStages stages of
// kTGroups groups of its 16 rows, each stage one mbarrier; x' staged 32 KB at a time.
constexpr int kTStages = 2;
constexpr int kTGroups = 8;
template <int NT>
constexpr int sub_groups_tma() { return NT == 1 ? 16 : 8; }
template <int kFmt>
constexpr int tma_wstage() { return 16 * kTGroups * (kFmt == 3 ? 16 : 32); }  // weight bytes per stage
template <int kFmt>
constexpr int tma_sstage() { return 16 * kTGroups * 2 * (kFmt == 4 ? 2 : 1); }  // scale bytes per stage

// One 128-weight group of the warp's rows r0 = gid and r1 = gid + 8, as lane (gid, tq)
// holds it: words 2tq and 2tq + 1 (g64: tq and tq + 4) of each row, and the rows' FP16
// scales (g64: both halves' scales, the first in the low 16 bits).
struct Grp {
    uint2 a, b;
    uint32_t s0, s1;
    uint32_t a2, b2;  // PTQ1_0: the third raw word of each row (a, b hold the first two)
};

// PTQ1_0: the first of the group's bytes that hold lane quad member tq's weights 32tq ..
// 32tq + 31, and the digit of that byte where weight 32tq sits.
__device__ __forceinline__ int ptq1_first_byte(int tq) { return (32 * tq) / 5; }
__device__ __forceinline__ int ptq1_first_digit(int tq) { return (32 * tq) % 5; }

// PTQ1_0 -> the lane's two PQ2_0 code words: w0..w2 are the aligned 32-bit words that hold
// its bytes from byte offset `shift` on; lut[b] holds the five 2-bit codes (digits) of byte b.
__device__ __forceinline__ uint2 ptq1_codes(uint32_t w0, uint32_t w1, uint32_t w2, int shift, int tq,
                                            const uint16_t *lut) {
    const uint32_t lo = __funnelshift_r(w0, w1, 8 * shift), hi = __funnelshift_r(w1, w2, 8 * shift);
    const uint64_t v0 = (uint64_t)lut[lo & 0xffu] | ((uint64_t)lut[(lo >> 8) & 0xffu] << 10) |
                        ((uint64_t)lut[(lo >> 16) & 0xffu] << 20) | ((uint64_t)lut[lo >> 24] << 30) |
                        ((uint64_t)lut[hi & 0xffu] << 40) | ((uint64_t)lut[(hi >> 8) & 0xffu] << 50);
    const uint64_t v1 = (uint64_t)lut[(hi >> 16) & 0xffu] | ((uint64_t)lut[hi >> 24] << 10);
    const int off = 2 * ptq1_first_digit(tq);  // bits of the digits before weight 32tq
    const uint64_t r = (v0 >> off) | (v1 << (60 - off));
    return make_uint2((uint32_t)r, (uint32_t)(r >> 32));
}

// 32-bit word at byte offset o (a multiple of 4) of a plane of `end` bytes (even): the bytes
// past the end read as zero and are never accessed.
__device__ __forceinline__ uint32_t ld_word_clamped(const uint8_t *p, int64_t o, int64_t end) {
    if (o + 4 <= end) return __ldcs(reinterpret_cast<const unsigned int *>(p + o));
    if (o + 2 <= end) return (uint32_t)__ldcs(reinterpret_cast<const unsigned short *>(p + o));
    return 0u;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(d[2]), "f"(d[3]));
}

// K order of the MMAs: MMA i of a group takes, from lane quad member tq, byte (i & 3) of
// group word 2tq + (i >> 2), i.e. the four weights 32tq + 16(i >> 2) + 4(i & 3) + c,
// c = 0..3, which sit at B slots 4tq + c of the MMA's 16-half row of x'.  g64: byte
// (i & 3) of word tq + 4(i >> 2), weights 64(i >> 2) + 16tq + 4(i & 3) + c.  Q1_0:
// nibble i & 1 of byte i >> 1 of word tq, weights 32tq + 4i + c.
template <int kFmt>
__device__ __forceinline__ int64_t skinny_k(int64_t group, int step, int tq) {
    return kFmt == 4   ? group * kGroup + 64 * (step >> 2) + 16 * tq + 4 * (step & 3)
           : kFmt == 3 ? group * kGroup + 32 * tq + 4 * step
                       : group * kGroup + 32 * tq + 16 * (step >> 2) + 4 * (step & 3);
}

// The rotation pass of this kernel: one warp per (group g, token m < MT).  It writes x'
// (FP16, nearest) of the block in the layout the MMAs read, [g][step][token][16] with
// slot 4tq + c = element skinny_k(g, step, tq) + c scaled by 4^-c (Q1_0: by 2^-c for an
// even step, 2^-(4 + c) for an odd one), zeros for the padding
// tokens m >= M, and the FP32 sum of the block's FP16 x' values to gsum[g][m] (g64: the
// sums of its two 64-element halves to gsum[g][h][m]).
template <int MT, int kFmt>
__device__ __forceinline__ void prep_task(const uint16_t *__restrict__ x, uint16_t *__restrict__ xs,
                                          float *__restrict__ gsum, int M, int64_t K, int64_t w, int lane) {
    const int64_t g = w / MT;  // (g, m) = (w / MT, w % MT)
    const int m = (int)(w % MT);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (m < M) {
        load_half4(x + (int64_t)m * K + g * kGroup + 4 * lane, v);
        fwht128_warp(v, lane);
    }
    const __half2 h01 = __floats2half2_rn(v[0], v[1]), h23 = __floats2half2_rn(v[2], v[3]);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    constexpr bool kG64 = kFmt == 4;
    float sum = (f01.x + f01.y) + (f23.x + f23.y);
    if (kG64) {  // lanes 0..15 hold the first 64 elements, 16..31 the last 64
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    } else {
        sum = warp_sum(sum);
    }
    // lane l holds elements 4l .. 4l+3 = skinny_k(g, i, tq) + c with tq = l >> 3 and
    // i = 4 ((l >> 2) & 1) + (l & 3) (g64: tq = (l >> 2) & 3, i = 4 (l >> 4) + (l & 3);
    // Q1_0: tq = l >> 3, i = l & 7)
    const int tq = kG64 ? (lane >> 2) & 3 : lane >> 3;
    const int i = kG64 ? 4 * (lane >> 4) + (lane & 3) : (kFmt == 3 ? lane & 7 : 4 * ((lane >> 2) & 1) + (lane & 3));
    __half2 s01, s23;
    if (kFmt == 3) {  // 2^-c, or 2^-(4 + c) for the high nibble (odd step)
        const float f = (i & 1) ? 0.0625f : 1.f;
        s01 = __hmul2(h01, __floats2half2_rn(f, 0.5f * f));
        s23 = __hmul2(h23, __floats2half2_rn(0.25f * f, 0.125f * f));
    } else {
        s01 = __hmul2(h01, __floats2half2_rn(1.f, 0.25f));
        s23 = __hmul2(h23, __floats2half2_rn(0.0625f, 0.015625f));
    }
    uint2 out;
    out.x = *reinterpret_cast<const uint32_t *>(&s01);
    out.y = *reinterpret_cast<const uint32_t *>(&s23);
    *reinterpret_cast<uint2 *>(xs + ((g * 8 + i) * MT + m) * 16 + 4 * tq) = out;
    if (kG64) {
        if ((lane & 15) == 0) gsum[(g * 2 + (lane >> 4)) * MT + m] = sum;
    } else if (lane == 0) {
        gsum[g * MT + m] = sum;
    }
}

template <int MT, int kFmt>
__global__ void __launch_bounds__(256) skinny_prep_kernel(const uint16_t *__restrict__ x, uint16_t *__restrict__ xs,
                                                          float *__restrict__ gsum, int M, int64_t K) {
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= (K / kGroup) * MT) return;
    prep_task<MT, kFmt>(x, xs, gsum, M, K, w, threadIdx.x & 31);
}


// kFmt: 2 PQ2_0, 4 PQ2_0 g64 (64-weight scales), 3 Q1_0, 1 PTQ1_0 (transcoded to PQ2_0 codes)
//
// x != nullptr: the rotation is the kernel's first phase.  Every CTA rotates its share of
// the (group, token) blocks into the staged layout (as the rotation pass does), counts
// itself in the workspace's call counter (ctl) and requests its first weights; before
// staging x' it waits (bounded) until the last CTA has advanced the counter.  The grid
// is then resident at once (the launcher checks the occupancy).  If that wait gives up,
// the CTA writes NaN and sets the status bit.
//
// kTma: the weights and scales come by TMA into a ring of kTStages stages per warp (the
// warp's 16 rows x kTGroups groups, 128-byte swizzle; scales unswizzled), one mbarrier
// per stage, instead of the register ring: the copies in flight then do not hold
// registers or load slots.  wmap and smap are the packed plane's and the scale plane's
// tensor maps (unused otherwise).  Needs K a multiple of 1024 and chunks of whole stages.
template <int NT, int kFmt, bool kTma>  // n8 token tiles: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kThreads) skinny_kernel(
    uint16_t *__restrict__ xsg, float *__restrict__ gsg, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, float *__restrict__ partials,
    unsigned int *__restrict__ counters, int M, int64_t N, int64_t K, int S, int gpc,
    const uint16_t *__restrict__ x, unsigned int *__restrict__ ctl, const __grid_constant__ CUtensorMap wmap,
    const __grid_constant__ CUtensorMap smap) {
    constexpr int MT = NT * 8;  // tokens padded
    static_assert(sub_groups<NT>() % kRing == 0, "ring slots follow the group index");
    static_assert(!kTma || (kFmt != 1 && sub_groups_tma<NT>() % kTGroups == 0), "TMA stages follow the group index");
    // groups staged at a time: the whole chunk when it fits (shared memory is sized so)
    constexpr int kSubMax = kTma ? sub_groups_tma<NT>() : sub_groups<NT>();
    const int kSub = gpc < kSubMax ? gpc : kSubMax;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    constexpr bool kG64 = kFmt == 4, kQ1 = kFmt == 3, kP1 = kFmt == 1;
    constexpr int kHalves = kG64 ? 2 : 1;  // scale groups per 128 weights
    constexpr int kWStage = tma_wstage<kFmt>(), kSStage = tma_sstage<kFmt>();
    __shared__ uint16_t lut3[kP1 ? 256 : 1];  // PTQ1_0: byte -> its five digits as 2-bit codes
    // kTma: [weight ring kWarps x kTStages x kWStage, 1024-byte aligned][scale ring
    // kWarps x kTStages x kSStage][x'][group sums][stage barriers]; otherwise [x'][group sums]
    uint8_t *smem = kTma ? smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u) : smem_raw;
    uint8_t *wring = smem;
    uint8_t *sring = smem + (kTma ? kWarps * kTStages * kWStage : 0);
    uint8_t *xbase = sring + (kTma ? kWarps * kTStages * kSStage : 0);
    uint16_t *xs = reinterpret_cast<uint16_t *>(xbase);  // [kSub * 8 steps][MT][16]
    float *gsum = reinterpret_cast<float *>(xbase + kSub * 8 * MT * 32);  // [MT][kSub][kHalves]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int64_t G = K / kGroup;
    const int chunk = blockIdx.y;
    const int g_begin = chunk * gpc;
    const int g_end = (int)((int64_t)(chunk + 1) * gpc < G ? (int64_t)(chunk + 1) * gpc : G);
    const int64_t n0 = (int64_t)blockIdx.x * kRowsPerCta + warp * 16;
    const int64_t r0 = n0 + gid, r1 = n0 + gid + 8;
    const bool v0 = r0 < N, v1 = r1 < N;

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 4; e++) acc[nt][e] = 0.f;

    // ---- the rotation phase and this CTA's arrival (fused launch)
    unsigned long long arrival = 0;
    if (x != nullptr) {
        const int64_t ncta = (int64_t)gridDim.x * gridDim.y;
        const int64_t b = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
        for (int64_t w = b * kWarps + warp; w < G * MT; w += ncta * kWarps)
            prep_task<MT, kFmt>(x, xsg, gsg, M, K, w, lane);
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            arrival = atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls), 1ull);
            const uint32_t calls = (uint32_t)(arrival >> 32);
            if ((uint32_t)arrival == (uint32_t)ncta - 1u) {  // the last CTA releases the others
                const unsigned long long step = calls + 1u == 0xffffffffu ? 2ull : 1ull;
                atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls),
                          (step << 32) - (unsigned long long)ncta);
            }
        }
    }

    const int64_t plane_end = N * G * kPtq1GroupBytes;  // PTQ1_0 plane size
    // PTQ1_0: the three aligned words holding the lane's bytes of row r's group g
    auto row_words3 = [&](int64_t r, int g, uint2 &w01, uint32_t &w2) {
        const int64_t a = ((r * G + g) * kPtq1GroupBytes + ptq1_first_byte(tq)) & ~(int64_t)3;
        if (a + 12 <= plane_end) {
            const unsigned int *p = reinterpret_cast<const unsigned int *>(packed + a);
            w01 = make_uint2(__ldcs(p), __ldcs(p + 1));
            w2 = __ldcs(p + 2);
        } else {  // the plane's last group
            w01 = make_uint2(ld_word_clamped(packed, a, plane_end), ld_word_clamped(packed, a + 4, plane_end));
            w2 = ld_word_clamped(packed, a + 8, plane_end);
        }
    };
    auto row_words = [&](int64_t r, int g) -> uint2 {
        if (kQ1)  // word tq of the row's 16-byte group
            return make_uint2(__ldcs(reinterpret_cast<const unsigned int *>(packed + (r * G + g) * kQ1GroupBytes) + tq),
                              0u);
        const uint8_t *p = packed + (r * G + g) * kPq2GroupBytes;
        if (kG64)
            return make_uint2(__ldcs(reinterpret_cast<const unsigned int *>(p) + tq),
                              __ldcs(reinterpret_cast<const unsigned int *>(p) + tq + 4));
        return __ldcs(reinterpret_cast<const uint2 *>(p) + tq);
    };
    auto row_scales = [&](int64_t r, int g) -> uint32_t {
        if (kG64) return __ldg(reinterpret_cast<const unsigned int *>(scales + r * 2 * G + 2 * g));
        return __ldg(scales + r * G + g);
    };
    auto load = [&](int g, Grp &q) {
        if (v0) {
            if (kP1)
                row_words3(r0, g, q.a, q.a2);
            else
                q.a = row_words(r0, g);
            q.s0 = row_scales(r0, g);
        } else {
            q.a = make_uint2(0x55555555u, 0x55555555u), q.s0 = 0u;  // trits 0
            q.a2 = 0u;
        }
        if (v1) {
            if (kP1)
                row_words3(r1, g, q.b, q.b2);
            else
                q.b = row_words(r1, g);
            q.s1 = row_scales(r1, g);
        } else {
            q.b = make_uint2(0x55555555u, 0x55555555u), q.s1 = 0u;
            q.b2 = 0u;
        }
    };
    if (kP1) {  // the byte -> codes table; the barrier before the first staging of x' publishes it
        for (int b = tid; b < 256; b += kThreads) {
            uint32_t f = 0;
            int v = b < 243 ? b : 0;
            for (int i = 0; i < 5; i++) {
                f |= (uint32_t)(v % 3) << (2 * i);
                v /= 3;
            }
            lut3[b] = (uint16_t)f;
        }
    }

    // Register ring: group g of the chunk lives in slot (g - g_begin) % kRing; the first
    // kRing are requested before x' is staged.  TMA ring: stage q (groups g_begin + 8q ..)
    // in slot q % kTStages of the warp's ring, its barrier completing with phase q / 2 & 1;
    // the first kTStages are requested before x' is staged.  A stage past the chunk's end
    // reads groups it does not use (zeros past the row).
    Grp ring[kTma ? 1 : kRing];
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        xbase + kSub * 8 * MT * 32 + ((MT * kSub * kHalves * 4 + 7) & ~7)) + warp * kTStages;
    const int nstages = kTma ? (g_end - g_begin + kTGroups - 1) / kTGroups : 0;
    int n_issued = 0;
    auto issue = [&](int q) {
        if (q >= nstages) return;
        const int slot = q % kTStages;
        if (lane == 0) {
            uint64_t *bar = bars + slot;
            uint8_t *wdst = wring + (warp * kTStages + slot) * kWStage;
            const int g = g_begin + q * kTGroups;
            mbar_arrive_expect_tx(bar, (uint32_t)(kWStage + kSStage));
            if (kQ1) {  // 8 groups x 16 bytes: one 128-byte box per row
                tma_load_2d(wdst, &wmap, bar, g * 16, (int)n0);
            } else {    // 8 groups x 32 bytes: two boxes of 4 groups
                tma_load_2d(wdst, &wmap, bar, g * 32, (int)n0);
                tma_load_2d(wdst + kWStage / 2, &wmap, bar, g * 32 + 128, (int)n0);
            }
            tma_load_2d(sring + (warp * kTStages + slot) * kSStage, &smap, bar, g * kHalves, (int)n0);
        }
        n_issued++;
    };
    if constexpr (kTma) {
        if (lane == 0) {
            for (int st = 0; st < kTStages; st++) mbar_init(bars + st, 1);
            mbar_init_fence();
        }
        __syncwarp();
        for (int q = 0; q < kTStages; q++) issue(q);
    } else {
#pragma unroll
        for (int u = 0; u < kRing; u++)
            if (g_begin + u < g_end) load(g_begin + u, ring[u]);
    }

    bool barrier_ok = true;
    bool copies_ok = true;  // (kTma) every stage waited for has landed
    int n_waited = 0;
    if (x != nullptr) {  // every CTA's x' is staged once the counter has moved on
        __shared__ int ok_s;
        if (tid == 0) {
            const uint32_t calls = (uint32_t)(arrival >> 32);
            uint32_t i = 0;
            for (; i < kSpinLimit; i++) {
                uint32_t hi;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(hi) : "l"(ctl + kCtlCalls + 1) : "memory");
                if (hi != calls) break;
                __nanosleep(32);
            }
            ok_s = i < kSpinLimit;
            if (i == kSpinLimit) atomicOr(ctl + kCtlStatus, kDevStatusSkinnyTimeout);
        }
        __syncthreads();
        barrier_ok = ok_s != 0;
    }

    for (int sub = g_begin; sub < g_end; sub += kSub) {
        const int nsub = g_end - sub < kSub ? g_end - sub : kSub;
        __syncthreads();  // the previous sub-chunk's x' is no longer read
        // the sub-chunk's x' (laid out by the rotation pass as read here) and group sums
        {
            const uint8_t *src = reinterpret_cast<const uint8_t *>(xsg + (int64_t)sub * 8 * MT * 16);
            const int bytes = nsub * 8 * MT * 32;
            for (int off = tid * 16; off < bytes; off += kThreads * 16)
                cp_async16(reinterpret_cast<uint8_t *>(xs) + off, src + off);
            cp_async_commit();
            for (int idx = tid; idx < nsub * MT * kHalves; idx += kThreads) {
                const int gh = idx / MT, m = idx % MT;  // gh = kHalves * gl + h
                // (through L2: in the fused launch other CTAs wrote these sums)
                gsum[m * kSub * kHalves + gh] = __ldcg(gsg + ((int64_t)sub * kHalves + gh) * MT + m);
            }
            cp_async_wait_all();
        }
        __syncthreads();

        // one group of the warp's rows: decode, MMAs, fold into acc
        auto consume = [&](Grp &cur, int gl) {
            if (kP1) {  // base-3 bytes -> the PQ2_0 code words of weights 32tq .. 32tq + 31
                const int g = sub + gl;
                const int sh0 = (int)(((r0 * G + g) * kPtq1GroupBytes + ptq1_first_byte(tq)) & 3);
                const int sh1 = (int)(((r1 * G + g) * kPtq1GroupBytes + ptq1_first_byte(tq)) & 3);
                if (v0) cur.a = ptq1_codes(cur.a.x, cur.a.y, cur.a2, sh0, tq, lut3);
                if (v1) cur.b = ptq1_codes(cur.b.x, cur.b.y, cur.b2, sh1, tq, lut3);
            }
            float d[kHalves][NT][4];  // g64: MMAs 0-3 and 4-7 fill the two halves
#pragma unroll
            for (int h = 0; h < kHalves; h++)
#pragma unroll
                for (int nt = 0; nt < NT; nt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) d[h][nt][e] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                // byte (i & 3) of the lane's word i >> 2, in both halves: (c0, c1) and
                // (c2, c3) left in place as FP16 subnormals c * 4^j * 2^-24.  Q1_0: byte
                // i >> 1 of the word, bits 4(i & 1) + (0, 1) and + (2, 3) left in place
                const int byte = kQ1 ? i >> 1 : i & 3;
                const uint32_t sel = 0x4040u | (uint32_t)byte | ((uint32_t)byte << 8);
                const uint32_t w0 = kQ1 ? cur.a.x : ((i >> 2) ? cur.a.y : cur.a.x);
                const uint32_t w1 = kQ1 ? cur.b.x : ((i >> 2) ? cur.b.y : cur.b.x);
                const uint32_t p0 = __byte_perm(w0, 0u, sel);
                const uint32_t p1 = __byte_perm(w1, 0u, sel);
                const uint32_t m01 = kQ1 ? ((i & 1) ? 0x00200010u : 0x00020001u) : 0x000C0003u;
                const uint32_t m23 = kQ1 ? ((i & 1) ? 0x00800040u : 0x00080004u) : 0x00C00030u;
                const uint32_t a0 = p0 & m01, a1 = p1 & m01;
                const uint32_t a2 = p0 & m23, a3 = p1 & m23;
                const int ks = gl * 8 + i;
#pragma unroll
                for (int nt = 0; nt < NT; nt++) {
                    const uint2 b = *reinterpret_cast<const uint2 *>(xs + ((ks * MT + nt * 8 + gid) * 16 + tq * 4));
                    mma16816(d[kG64 ? i >> 2 : 0][nt], a0, a1, a2, a3, b.x, b.y);
                }
            }
#pragma unroll
            for (int h = 0; h < kHalves; h++) {
                const float cs0 = half_bits_to_float((uint16_t)(cur.s0 >> (16 * h)));
                const float cs1 = half_bits_to_float((uint16_t)(cur.s1 >> (16 * h)));
#pragma unroll
                for (int nt = 0; nt < NT; nt++) {
                    const int m0 = nt * 8 + 2 * tq;
                    const float gs0 = gsum[m0 * kSub * kHalves + gl * kHalves + h];
                    const float gs1 = gsum[(m0 + 1) * kSub * kHalves + gl * kHalves + h];
                    // d[h][nt][0], [1]: row r0, tokens m0, m0+1; [2], [3]: row r1.  Codes c
                    // give sum c x' - sum x'; Q1_0 bits b give 2 sum b x' - sum x'
                    constexpr float kUnit = kQ1 ? 33554432.f : 16777216.f;
                    acc[nt][0] = fmaf(cs0, fmaf(d[h][nt][0], kUnit, -gs0), acc[nt][0]);
                    acc[nt][1] = fmaf(cs0, fmaf(d[h][nt][1], kUnit, -gs1), acc[nt][1]);
                    acc[nt][2] = fmaf(cs1, fmaf(d[h][nt][2], kUnit, -gs0), acc[nt][2]);
                    acc[nt][3] = fmaf(cs1, fmaf(d[h][nt][3], kUnit, -gs1), acc[nt][3]);
                }
            }
        };
        if constexpr (kTma) {
            for (int gs = 0; gs < nsub; gs += kTGroups) {
                const int q = (sub - g_begin + gs) / kTGroups;  // the stage
                const int slot = q % kTStages;
                if (copies_ok) {  // warp-uniform outcome
                    copies_ok = __all_sync(0xffffffffu, mbar_wait(bars + slot, (uint32_t)(q / kTStages) & 1u));
                    if (copies_ok)
                        n_waited++;
                    else if (lane == 0 && ctl != nullptr)
                        atomicOr(ctl + kCtlStatus, kDevStatusSkinnyTimeout);
                }
                const uint8_t *wst = wring + (warp * kTStages + slot) * kWStage;
                const uint8_t *sst = sring + (warp * kTStages + slot) * kSStage;
#pragma unroll
                for (int u = 0; u < kTGroups; u++) {
                    if (gs + u >= nsub) break;
                    // rows gid and gid + 8 of the stage (both in swizzle phase gid); the
                    // lane's words as the register ring would load them
                    Grp cur;
                    if (kQ1) {  // word tq of the 16-byte group u: logical chunk u
                        const int c = (u ^ gid) << 4;
                        cur.a = make_uint2(*reinterpret_cast<const uint32_t *>(wst + gid * 128 + c + 4 * tq), 0u);
                        cur.b = make_uint2(*reinterpret_cast<const uint32_t *>(wst + (gid + 8) * 128 + c + 4 * tq), 0u);
                    } else {
                        const uint8_t *b0 = wst + (u >> 2) * (kWStage / 2) + gid * 128;  // box of groups 4(u/4) ..
                        const uint8_t *b1 = b0 + 8 * 128;
                        const int qg = u & 3;
                        if (kG64) {  // words tq and tq + 4: logical chunks 2qg and 2qg + 1
                            const int c0 = ((2 * qg) ^ gid) << 4, c1 = ((2 * qg + 1) ^ gid) << 4;
                            cur.a = make_uint2(*reinterpret_cast<const uint32_t *>(b0 + c0 + 4 * tq),
                                               *reinterpret_cast<const uint32_t *>(b0 + c1 + 4 * tq));
                            cur.b = make_uint2(*reinterpret_cast<const uint32_t *>(b1 + c0 + 4 * tq),
                                               *reinterpret_cast<const uint32_t *>(b1 + c1 + 4 * tq));
                        } else {  // words 2tq, 2tq + 1: logical chunk 2qg + tq / 2
                            const int c = ((2 * qg + (tq >> 1)) ^ gid) << 4;
                            cur.a = *reinterpret_cast<const uint2 *>(b0 + c + (tq & 1) * 8);
                            cur.b = *reinterpret_cast<const uint2 *>(b1 + c + (tq & 1) * 8);
                        }
                    }
                    if (kG64) {
                        cur.s0 = reinterpret_cast<const uint32_t *>(sst)[gid * kTGroups + u];
                        cur.s1 = reinterpret_cast<const uint32_t *>(sst)[(gid + 8) * kTGroups + u];
                    } else {
                        cur.s0 = reinterpret_cast<const uint16_t *>(sst)[gid * kTGroups + u];
                        cur.s1 = reinterpret_cast<const uint16_t *>(sst)[(gid + 8) * kTGroups + u];
                    }
                    cur.a2 = cur.b2 = 0u;
                    consume(cur, gs + u);
                }
                __syncwarp();  // every lane has read the stage
                if (copies_ok) {
                    if (lane == 0) fence_proxy_async();
                    issue(q + kTStages);  // refill the slot
                }
            }
        } else {
            for (int gl0 = 0; gl0 < nsub; gl0 += kRing) {
#pragma unroll
                for (int u = 0; u < kRing; u++) {
                    const int gl = gl0 + u;
                    if (gl >= nsub) break;
                    Grp &cur = ring[u];
                    consume(cur, gl);
                    const int g = sub + gl;
                    if (g + kRing < g_end) load(g + kRing, cur);  // refill the slot
                }
            }
        }
    }

    if (kTma && !copies_ok && lane == 0) {  // the copies already started land before the CTA exits
        for (int q = n_waited; q < n_issued; q++) mbar_wait(bars + q % kTStages, (uint32_t)(q / kTStages) & 1u);
    }
    if (!barrier_ok || !copies_ok)
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) acc[nt][e] = __int_as_float(0x7fc00000);
    // ---- output (warps wholly past N do nothing; every CTA of the row block agrees)
    if (n0 >= N) return;
    if (S == 1) {
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int m = nt * 8 + 2 * tq + (e & 1);
                const int64_t r = e < 2 ? r0 : r1;
                if (m < M && r < N) y[(int64_t)m * N + r] = float_to_half_bits(acc[nt][e]);
            }
        return;
    }
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int m = nt * 8 + 2 * tq + (e & 1);
            const int64_t r = e < 2 ? r0 : r1;
            if (m < M && r < N) partials[((int64_t)chunk * M + m) * N + r] = acc[nt][e];
        }
    __threadfence();
    __syncwarp();
    const int64_t rb = n0 / 16;  // this warp's 16-row block
    unsigned int arrived = 0;
    if (lane == 0) arrived = atomicAdd(counters + rb, 1u);
    arrived = __shfl_sync(0xffffffffu, arrived, 0);
    if (arrived != (unsigned int)(S - 1)) return;
    __threadfence();
    // last chunk of this row block: sum the partials in chunk order
    for (int idx = lane; idx < 16 * M; idx += 32) {
        const int m = idx / 16;
        const int64_t r = n0 + (idx & 15);
        if (r >= N) continue;
        float a = 0.f;
        for (int c = 0; c < S; c++) a += __ldcg(partials + ((int64_t)c * M + m) * N + r);
        y[(int64_t)m * N + r] = float_to_half_bits(a);
    }
    if (lane == 0) counters[rb] = 0u;
}

// The TMA ring takes PQ2_0, g64 and Q1_0 when a row's groups come in whole stages (its
// plane rows and scale rows are then multiples of 16 bytes, as tensor maps need).
bool use_tma(int64_t K, int fmt) { return fmt != 1 && (K / kGroup) % kTGroups == 0; }

int smem_bytes(int NT, int gpc, int fmt, bool tma) {
    const bool g64 = fmt == 4;
    int sub = tma ? (NT == 1 ? sub_groups_tma<1>() : sub_groups_tma<2>()) : (NT == 1 ? sub_groups<1>() : sub_groups<2>());
    sub = gpc < sub ? gpc : sub;
    const int xs = sub * 8 * NT * 8 * 32, gs = NT * 8 * sub * 4 * (g64 ? 2 : 1);
    if (!tma) return xs + gs;
    const int ws = fmt == 3 ? tma_wstage<3>() : tma_wstage<2>();
    const int ss = g64 ? tma_sstage<4>() : tma_sstage<2>();
    return 1024 + kWarps * kTStages * (ws + ss) + xs + ((gs + 7) & ~7) + kWarps * kTStages * 8;
}

// K chunks: about as many CTAs as fit on the GPU at once (one wave; a CTA's registers
// allow two per SM), unless split_k (> 0) says otherwise.  With the TMA ring a chunk is
// a whole number of stages (kTGroups groups).
void choose_split(int64_t N, int64_t K, int split_k, bool tma, const DeviceInfo &dev, int *S, int *gpc) {
    const int64_t G = K / kGroup;
    const int64_t rb = (N + kRowsPerCta - 1) / kRowsPerCta;
    int64_t s = split_k > 0 ? split_k : (2 * (int64_t)dev.sm_count) / rb;
    if (s < 1) s = 1;
    if (s > G) s = G;
    int64_t per = (G + s - 1) / s;
    if (tma) per = (per + kTGroups - 1) / kTGroups * kTGroups;
    *gpc = (int)per;
    *S = (int)((G + per - 1) / per);
}

// Workspace: the staged x' ([G][8][MT][16] FP16), the group sums ([G][MT] FP32; g64
// [G][2][MT]), then the split-K partials.
size_t staged_bytes(int64_t M, int64_t K) {
    const int64_t MT = M <= 8 ? 8 : 16;
    return ((size_t)(K / kGroup) * 8 * MT * 32 + 255) / 256 * 256;
}
size_t gsum_bytes(int64_t M, int64_t K) {  // room for the g64 half sums
    const int64_t MT = M <= 8 ? 8 : 16;
    return ((size_t)(K / kGroup) * 2 * MT * 4 + 255) / 256 * 256;
}

// The kernel instance for (M, fmt, ring), its shared memory, and whether its grid is
// resident on the GPU at once (then the rotation runs inside it: one launch).
template <int NT, int kFmt, bool kTma>
cudaError_t kernel_fits(int64_t grid_ctas, int smem, const DeviceInfo &dev, bool *fits) {
    auto kern = skinny_kernel<NT, kFmt, kTma>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (err != cudaSuccess) return err;
    *fits = grid_ctas <= (int64_t)per_sm * dev.sm_count;
    return cudaSuccess;
}

template <int NT>
cudaError_t kernel_fits_fmt(int fmt, bool tma, int64_t ctas, int smem, const DeviceInfo &dev, bool *fits) {
    if (tma)
        return fmt == 4   ? kernel_fits<NT, 4, true>(ctas, smem, dev, fits)
               : fmt == 3 ? kernel_fits<NT, 3, true>(ctas, smem, dev, fits)
                          : kernel_fits<NT, 2, true>(ctas, smem, dev, fits);
    return fmt == 4   ? kernel_fits<NT, 4, false>(ctas, smem, dev, fits)
           : fmt == 3 ? kernel_fits<NT, 3, false>(ctas, smem, dev, fits)
           : fmt == 1 ? kernel_fits<NT, 1, false>(ctas, smem, dev, fits)
                      : kernel_fits<NT, 2, false>(ctas, smem, dev, fits);
}

cudaError_t grid_fits(int64_t M, int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev, bool *fits) {
    const bool tma = use_tma(K, fmt);
    int S, gpc;
    choose_split(N, K, split_k, tma, dev, &S, &gpc);
    const int64_t ctas = ((N + kRowsPerCta - 1) / kRowsPerCta) * S;
    const int NT = M <= 8 ? 1 : 2;
    const int smem = smem_bytes(NT, gpc, fmt, tma);
    return NT == 1 ? kernel_fits_fmt<1>(fmt, tma, ctas, smem, dev, fits)
                   : kernel_fits_fmt<2>(fmt, tma, ctas, smem, dev, fits);
}

}  // namespace

bool skinny_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    return fmt >= 1 && fmt <= 4 && M >= 1 && M <= 16 && K % kGroup == 0 && (N + 15) / 16 <= kMaxTiles &&
           K < ((int64_t)1 << 31);
}

size_t skinny_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    int S, gpc;
    choose_split(N, K, split_k, use_tma(K, fmt), dev, &S, &gpc);
    return staged_bytes(M, K) + gsum_bytes(M, K) + (S > 1 ? (size_t)S * (size_t)M * (size_t)N * sizeof(float) : 0);
}

int skinny_launches(int64_t M, int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    bool fits = false;
    if (grid_fits(M, N, K, fmt, split_k, dev, &fits) != cudaSuccess) return -1;
    return fits ? 1 : 2;
}

cudaError_t launch_skinny(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                          uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int split_k,
                          const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    if (fmt < 1 || fmt > 4) return cudaErrorInvalidValue;
    uint16_t *xsg = reinterpret_cast<uint16_t *>(ws.data);
    float *gsg = reinterpret_cast<float *>(ws.data + staged_bytes(M, K));
    float *partials = reinterpret_cast<float *>(ws.data + staged_bytes(M, K) + gsum_bytes(M, K));
    const bool tma = use_tma(K, fmt);
    int S, gpc;
    choose_split(N, K, split_k, tma, dev, &S, &gpc);
    const dim3 grid((unsigned)((N + kRowsPerCta - 1) / kRowsPerCta), (unsigned)S);
    const int64_t G = K / kGroup;
    // tensor maps of the packed plane (rows of G x 32 bytes, Q1_0 16; boxes of 128 bytes x
    // 16 rows, 128-byte swizzle) and of the scale plane (rows of G or 2G FP16; boxes of 8
    // or 16 scales x 16 rows), for the TMA ring; zeros otherwise (never read)
    CUtensorMap wmap, smap;
    memset(&wmap, 0, sizeof(wmap));
    memset(&smap, 0, sizeof(smap));
    if (tma) {
        EncodeTiledFn encode = encode_fn();
        if (!encode) return cudaErrorNotSupported;
        const int64_t rowb = G * (fmt == 3 ? 16 : 32), GS = G * (fmt == 4 ? 2 : 1);
        const cuuint64_t wd[2] = {(cuuint64_t)rowb, (cuuint64_t)N}, ws_[1] = {(cuuint64_t)rowb};
        const cuuint32_t wb[2] = {128, 16}, es[2] = {1, 1};
        if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), wd, ws_, wb, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        const cuuint64_t sd[2] = {(cuuint64_t)GS, (cuuint64_t)N}, ss_[1] = {(cuuint64_t)GS * 2};
        const cuuint32_t sb[2] = {(cuuint32_t)(kTGroups * (fmt == 4 ? 2 : 1)), 16};
        if (encode(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t *>(scales), sd, ss_, sb, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // one launch when the whole grid is resident at once (its CTAs meet at a barrier after
    // rotating x), else the rotation pass first
    bool fits = false;
    cudaError_t ferr = grid_fits(M, N, K, fmt, split_k, dev, &fits);
    if (ferr != cudaSuccess) return ferr;
    const bool fused = fits && ws.zeroed != nullptr && ws.zeroed_bytes >= kCtlRegionBytes;
    auto run = [&](auto prep, auto kern, int MT, int NT) -> cudaError_t {
        const int smem = smem_bytes(NT, gpc, fmt, tma);
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
        if (!fused) prep<<<(unsigned)((G * MT + 7) / 8), 256, 0, s>>>(x, xsg, gsg, (int)M, K);
        kern<<<grid, kThreads, smem, s>>>(xsg, gsg, packed, scales, y, partials, ws.counters, (int)M, N, K, S, gpc,
                                          fused ? x : nullptr, reinterpret_cast<unsigned int *>(ws.zeroed), wmap,
                                          smap);
        return cudaGetLastError();
    };
    if (M <= 8) {
        if (fmt == 4)
            return tma ? run(skinny_prep_kernel<8, 4>, skinny_kernel<1, 4, true>, 8, 1)
                       : run(skinny_prep_kernel<8, 4>, skinny_kernel<1, 4, false>, 8, 1);
        if (fmt == 3)
            return tma ? run(skinny_prep_kernel<8, 3>, skinny_kernel<1, 3, true>, 8, 1)
                       : run(skinny_prep_kernel<8, 3>, skinny_kernel<1, 3, false>, 8, 1);
        if (fmt == 1) return run(skinny_prep_kernel<8, 1>, skinny_kernel<1, 1, false>, 8, 1);
        return tma ? run(skinny_prep_kernel<8, 2>, skinny_kernel<1, 2, true>, 8, 1)
                   : run(skinny_prep_kernel<8, 2>, skinny_kernel<1, 2, false>, 8, 1);
    }
    if (fmt == 4)
        return tma ? run(skinny_prep_kernel<16, 4>, skinny_kernel<2, 4, true>, 16, 2)
                   : run(skinny_prep_kernel<16, 4>, skinny_kernel<2, 4, false>, 16, 2);
    if (fmt == 3)
        return tma ? run(skinny_prep_kernel<16, 3>, skinny_kernel<2, 3, true>, 16, 2)
                   : run(skinny_prep_kernel<16, 3>, skinny_kernel<2, 3, false>, 16, 2);
    if (fmt == 1) return run(skinny_prep_kernel<16, 1>, skinny_kernel<2, 1, false>, 16, 2);
    return tma ? run(skinny_prep_kernel<16, 2>, skinny_kernel<2, 2, true>, 16, 2)
               : run(skinny_prep_kernel<16, 2>, skinny_kernel<2, 2, false>, 16, 2);
}

}  // namespace bonsai
