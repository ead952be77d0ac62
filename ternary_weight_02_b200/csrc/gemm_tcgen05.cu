// gemm_tcgen05.cu -- prefill ternary GEMM on the 5th-generation tensor cores.
//
// y[m][n] = sum_k x'[m][k] * s[n][k/128] * t[n][k] for M tokens at once: a dense
// contraction (2*M*N*K FLOP), so it runs as an FP16 x FP16 -> FP32 tcgen05 MMA with the
// accumulator in tensor memory.  Sources: "27B 模型压到 5.95GB，推理能力还保住 98%"
// (allhereai.com): method paragraph (trits, FP16 scale per 128 weights, block
// Hadamard), packings paragraph (PQ2_0 wins prompt processing); "Bonsai 2，把27B压进6个G"
// (10100.com), section 它怎么做到的 (the input takes the matching transform).
//
// One launch per call, persistent (at most one CTA per SM, all resident at once):
//  1. every CTA rotates its share of the 128-blocks of x into x' (FP16, round to
//     nearest) in the workspace, each 8 columns (Q1_0: 16) in the K order of the expanded
//     weights.  Rotating per tile would redo each 128 x 128 x' tile's FWHT for every one
//     of the N/256 column tiles; done once, it costs one read and one write of x.  The
//     CTAs then meet at a grid-wide barrier: each counts itself in the workspace's call
//     counter with one atomic add, the last one advances the counter, and only the
//     thread that issues the TMA loads of x' waits for that (bounded), while the rest of
//     the CTA sets up its barriers and tensor memory.
//  2. the tiles: each CTA takes whole tiles in waves
//     and then an even share of the last tiles' 64-wide K stages (stream-K, below), so
//     that no SM idles in a partial last wave.  A tile is kAcc x 128 rows x 256
//     columns of y; per stage (3- or 4-deep rings):
//     - warp 0 (one thread): TMA loads of the x' tile (128 rows x 64, 128-byte swizzle);
//     - warp 1: allocates the TMEM accumulators; one thread issues tcgen05.mma
//       (M=128, N=256, K=16, kind::f16, FP32 accumulate) and commits each stage back;
//     - warps 2..9 (256 threads, one weight row each): expand the packed trits of a
//       128-weight group times its FP16 scale into two 64-wide FP16 B stages, written
//       in the same 128-byte-swizzled K-major layout the MMA descriptors describe
//       (t * s is exact in FP16; PQ2_0 g64 takes a new scale with every 64-wide
//       stage); after each piece of a tile, the epilogue:
//       tcgen05.ld of the accumulator, then FP16 (nearest even) stores to y, or the
//       FP32 hand-over of a split tile.
// Every wait is bounded: if one gives up, the CTA stops issuing work, waits for the
// copies and MMAs it started, frees its tensor memory and writes NaN to its tiles (and
// hands NaN over for a split one), and sets its bit in the device status word.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace bonsai {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;  // BM: rows of one MMA / one TMEM accumulator
constexpr int kExpandWarps = 8;
constexpr int kThreads = (2 + kExpandWarps) * 32;  // 320

// Tile configuration: kAcc accumulators of 128 rows each share every B stage (the
// expanded weights), so the CTA covers 128 * kAcc rows of y.  kPair (CTA pairs): each CTA
// holds half of a B stage (128 weight rows), so the same shared memory takes more stages,
// which the pair's longer round trip per stage (both CTAs' copies and expansions) needs.
template <int kAcc, bool kPair = false>
struct Cfg {
    static constexpr int kStages = kPair ? (kAcc == 2 ? 4 : 6) : (kAcc == 2 ? 3 : 4);
    static constexpr int kTileM = BM * kAcc;
    static constexpr int kAStage = kTileM * BK * 2;  // 16 or 32 KB
    static constexpr int kBStage = (kPair ? BN / 2 : BN) * BK * 2;   // 16 or 32 KB
    static constexpr int kCodeStage = (kPair ? BN / 2 : BN) * BK / 4;  // PQ2_0 codes of a B stage
    static constexpr int kTmemCols = 256 * kAcc;
    // shared memory: [A stages][B stages][PQ2_0 code stages][barriers][tmem slot][abort
    // flag][PTQ1_0 LUT]
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kStages * kAStage;
    static constexpr int kOffCodes = kOffB + kStages * kBStage;
    static constexpr int kOffBar = kOffCodes + kStages * kCodeStage;
    static constexpr int kNumBars = 3 * kStages + 6;  // full_a, full_b, empty, done, tmem_free, fin, 3 rotation
    static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr int kOffAbort = kOffTmemSlot + 8;
    static constexpr int kOffLut = kOffAbort + 8;
    static constexpr int kSmemBytes = kOffLut + 256 * 4 + 1024;  // + slack for the 1024-B tile base
    // the epilogue stages y through the B ring: 8 warps x 8 KB
    static_assert(kStages * kBStage >= kExpandWarps * 8192, "the B ring holds the epilogue's staging rows");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
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
// The same for a CTA pair (cta_group::2): M = 256, rows 0..127 of A and D in the even CTA
// of the pair and rows 128..255 in the odd one; B's N = 256 columns split the same way
// (columns 0..127 in the even CTA's shared memory).  Issued by the even CTA only.
constexpr uint32_t kIdesc2 = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(256 >> 4) << 24);
__device__ __forceinline__ void mma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accumulate));
}
// Arrives on the barrier at the same shared-memory offset in both CTAs of the pair once
// every MMA the pair's issuing thread started has completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(saddr(bar)), "h"((uint16_t)3)
        : "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// Bounded wait with cluster-scope acquire (arrivals from the peer CTA included).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; i++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(saddr(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(bar))
                 : "memory");
}

// 32 columns of this warp's 32 TMEM lanes, the wait in the same statement.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 64 columns of this warp's 32 TMEM lanes (lane i of the warp: TMEM lane 32q + i) in one
// load; the wait is in the same statement, so no use of r can be scheduled before it.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, "
        "%35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
        "%56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// ---------------------------------------------------------------- trit expansion

// One 32-bit word of 2-bit codes (code c_i = trit + 1 at bits 2i, weights w0 .. w0+15)
// times the scale s, as two 16-byte chunks of FP16: out[0..3] = weights w0 .. w0+7 and
// out[4..7] = weights w0+8 .. w0+15, each 8 in the order [0, 4, 1, 5, 2, 6, 3, 7] (x' is
// stored in the same order).  The value of code c is byte pair (2c, 2c+1) of the table
// {tneg = -s | 0 << 16, tpos = +s}: -s, 0 or +s, exactly t * s.  With m = the codes j,
// j+4, j+8, j+12 of the word as bytes, m * 0x22 + 0x10 per byte is the selector nibble
// pair (2c, 2c+1) of each, so one byte permute makes two weights.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t tneg, uint32_t tpos, uint32_t (&out)[8]) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t m = (w >> (2 * j)) & 0x03030303u;
        const uint32_t sel = m * 0x22u + 0x10101010u;
        out[j] = __byte_perm(tneg, tpos, sel);            // codes j, j + 4
        out[4 + j] = __byte_perm(tneg, tpos, sel >> 16);  // codes j + 8, j + 12
    }
}

// Q1_0: one 32-bit word of signs (bit i = weight w0+i, 1 for +1) times the scale s, as
// four 16-byte chunks of FP16: out[0..3] = weights [0,8,1,9,2,10,3,11], out[4..7] =
// [4,12,..,7,15], out[8..11] = 16 + [0,8,..], out[12..15] = 16 + [4,12,..] (x' is stored
// in the same order within each 16).  The value of bit b is byte pair (2b, 2b+1) of the
// table tab = -s | +s << 16.
__device__ __forceinline__ void expand_word_q1(uint32_t w, uint32_t tab, uint32_t (&out)[16]) {
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const uint32_t m = (w >> j) & 0x01010101u;  // weights j, j + 8, j + 16, j + 24
        const uint32_t sel = m * 0x22u + 0x10101010u;
        const int c = (j >> 2) * 4 + (j & 3);
        out[c] = __byte_perm(tab, 0u, sel);             // weights j, j + 8
        out[8 + c] = __byte_perm(tab, 0u, sel >> 16);   // weights j + 16, j + 24
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
    } else if (kFmt == 3) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(packed + (n * G + g) * kQ1GroupBytes));
        raw.w[0] = a.x, raw.w[1] = a.y, raw.w[2] = a.z, raw.w[3] = a.w;
        raw.w[4] = raw.w[5] = raw.w[6] = raw.w[7] = 0u;
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
    if (kFmt == 2 || kFmt == 3) {  // (Q1_0: sign words 0..3)
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

// ---------------------------------------------------------------- cross-CTA hand-over

// A tile piece's FP32 partial sums go to the CTA's own slot in the workspace; a flag
// word per CTA says that the slot is complete by holding this call's epoch (the call
// counter's value plus one), so flags never need clearing.  The writer's threads fence,
// meet at a named barrier, and one of them releases the flag; the owner acquires it
// (every lane polls, bounded) and reads the slot through L2.
__device__ __forceinline__ void flag_release(unsigned int *p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int flag_acquire(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Bounded wait of a whole warp for *p == want.
__device__ __forceinline__ bool flag_wait(const unsigned int *p, unsigned int want, uint32_t limit) {
    for (uint32_t i = 0; i < limit; i++) {
        if (__all_sync(0xffffffffu, flag_acquire(p) == want)) return true;
        __nanosleep(64);
    }
    return false;
}
__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// The eight expansion/epilogue warps (256 threads) meet here; barrier 0 is __syncthreads.
__device__ __forceinline__ void expand_warps_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// ---------------------------------------------------------------- kernel

// Work split (whole-tile waves, then stream-K).  The T tiles of y (kAcc*128 rows x 256
// columns, numbered with the row tile fastest) are taken by C persistent CTAs:
//  1. W = floor(T/C) - 1 waves of whole tiles (none if T < 2C): CTA b takes tiles b,
//     b + C, ..., so that the C tiles in flight at once are consecutive and share x' row
//     tiles and weight columns in L2;
//  2. the remaining tiles (one to two waves' worth) are cut into units of one 64-wide K
//     stage, unit u being stage u % nk of remaining tile u / nk, and CTA b takes units
//     [Ur*b/C, Ur*(b+1)/C) in order, as a run of "pieces" (its units of one tile).  Only
//     the first of these pieces can continue a tile that an earlier CTA started, and only
//     the last can be a tile's start that a later CTA continues:
//     - a whole tile is written to y directly;
//     - a continuing piece stores its FP32 sums in the CTA's slot and raises its flag;
//     - a tile's first piece (its "owner") waits for the flags of the CTAs that continue
//       the tile, adds their slots in K order, writes y and clears those flags.
// A continuing piece comes before anything else of its CTA's split share, and the owner's
// piece last: the waits are short, and they only go from a CTA to later ones, which never
// wait before they have stored (all CTAs of the grid are resident at once, one per SM).
//
// x: the un-rotated input (M x K); xr: the workspace's x' (nblocks 128-blocks).  ctl: the
// workspace's control words (call counter, status word, hand-over flags from kCtlGemmFlags
// on).  wait_limit and epoch_skew: the polls of an owner's wait for a flag and an offset
// added to the epoch it waits for (kSpinLimit and 0 except under the test hook that makes
// those waits give up).
//
// kSwiglu: the weight rows are a fused gate/up projection (gate rows 0 .. F-1, up rows
// F .. 2F-1, N = 2F) and the output is h = silu(gate) * up, M x F.  A tile's
// 256 weight rows are then gate rows 128 tn .. 128 tn + 127 followed by the matching up
// rows, so that each epilogue warp finds gate column c and up column 128 + c of the same
// output in its own accumulator lanes.
//
// kPair: the CTAs work in pairs (clusters of two) on tiles of 256 kAcc rows x 256 columns
// with tcgen05.mma.cta_group::2: CTA rank r of the pair holds x' rows a 256 + 128 r ..
// +127 of its accumulator a and expands weight rows 128 r .. 128 r + 127 of the tile's
// 256 (two threads per row, half a stage each), so each SM expands half the B operand for
// the same MMA work (each SM's tensor core still reads all of B, the peer's half from the
// peer's shared memory).  The even CTA issues the MMAs once both CTAs' stages
// are ready (its full_b barrier counts its own expansion warps and one arrival that a
// thread of the odd CTA forwards) and commits them to the barriers of both; hand-over
// slots and flags stay per CTA, work is split per pair.  Only an explicit request takes
// this mode: on the 27B-class projections it runs a few per cent behind single-CTA
// tiles, whose x' traffic per MMA it shares, so halving the expansion buys nothing there.
template <int kFmt, int kAcc, bool kSwiglu, bool kPair>
__global__ void __launch_bounds__(kThreads, 1) gemm_tcgen05_kernel(
    const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap w_map,
    const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, float *__restrict__ partials,
    const uint16_t *__restrict__ x, uint16_t *__restrict__ xr, int64_t nblocks, unsigned int *__restrict__ ctl,
    uint32_t wait_limit, uint32_t epoch_skew, int M, int N, int K, int mt, int F) {
    using C = Cfg<kAcc, kPair>;
    constexpr int STAGES = C::kStages;
    constexpr int kSlotFloats = C::kTileM * BN;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the tile area (128-byte swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + C::kOffA;
    uint8_t *sB = smem + C::kOffB;
    const uint8_t *sCodes = smem + C::kOffCodes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *full_a = bars, *full_b = bars + STAGES, *empty = bars + 2 * STAGES;
    uint64_t *done = bars + 3 * STAGES, *tmem_free = done + 1, *fin = done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    uint32_t *epoch_s = tmem_slot + 1;  // the second word of the slot's 8 bytes
    unsigned int *flags = ctl + kCtlGemmFlags;
    unsigned int *status = ctl + kCtlStatus;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem + C::kOffLut);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = K / BK;
    const int64_t G = K / kGroup;
    // PQ2_0 and its 64-weight-scale variant take their codes by TMA with the x' stage
    constexpr bool kTma = kFmt == 2 || kFmt == 4;
    const int64_t G64 = K / 64;  // PQ2_0 g64: scales per row
    const int nctas = (int)gridDim.x, cta = (int)blockIdx.x;
    // the work split's unit: a CTA, or (kPair) a pair of CTAs
    const int rank = kPair ? (int)cluster_rank() : 0;
    const int nunits = kPair ? nctas / 2 : nctas, unit = kPair ? cta / 2 : cta;
    auto cta_of = [&](int u) { return kPair ? 2 * u + rank : u; };  // this rank's CTA of unit u
    constexpr int kTileRows = kPair ? 256 * kAcc : C::kTileM;      // x' rows of a tile
    // first x' row of this CTA's accumulator a in row tile tm
    auto acc_row0 = [&](int tm, int a) { return tm * kTileRows + (kPair ? a * 256 + rank * BM : a * BM); };
    // whole-tile waves first (unit b: tiles b, b + C, ...), then the last one or two
    // waves' worth of tiles split by K stages
    const int T = mt * ((N + BN - 1) / BN);
    const int W = T / nunits >= 2 ? T / nunits - 1 : 0;
    const int Tdp = W * nunits;
    const int Ur = (T - Tdp) * nk;
    auto range_end = [&](int c) { return (int)((int64_t)Ur * (c + 1) / nunits); };
    const int u_begin = (int)((int64_t)Ur * unit / nunits), u_end = range_end(unit);
    const int n_mine = W * nk + (u_end - u_begin);  // this CTA's units
    // the piece that starts at this CTA's unit v: tile s (row tile fastest), stages
    // [kb, ke); tr: the tile's index among the split ones (-1 for a whole-tile wave)
    struct Piece {
        int s, kb, ke, tr;
    };
    auto piece_at = [&](int v) {
        Piece p;
        if (v < W * nk) {
            p.s = unit + (v / nk) * nunits;
            p.kb = 0;
            p.ke = nk;
            p.tr = -1;
        } else {
            const int u = u_begin + (v - W * nk);
            p.tr = u / nk;
            p.kb = u - p.tr * nk;
            p.ke = p.kb + (u_end - u) < nk ? p.kb + (u_end - u) : nk;
            p.s = Tdp + p.tr;
        }
        return p;
    };

    // ---- rotation of this CTA's share of x, then its arrival at the grid barrier.  The
    // CTA's 128-blocks (a contiguous run of x) stream through the tile rings' shared memory,
    // idle until the tiles start, in 64 KB bulk copies three deep; each warp rotates blocks
    // from there and stores x'.
    bool rot_fail = false;
    {
        constexpr int kWarps = kThreads / 32;
        constexpr int kRotBufBytes = 64 * 1024, kRotBufs = 3, kRotBlocks = kRotBufBytes / (kGroup * 2);
        static_assert(kRotBufs * kRotBufBytes <= C::kOffCodes, "rotation buffers lie inside the A and B rings");
        uint64_t *rot_bar = bars + 3 * STAGES + 3;
        const int64_t rb0 = nblocks * cta / nctas, rb1 = nblocks * (cta + 1) / nctas;
        const int nchunks = (int)((rb1 - rb0 + kRotBlocks - 1) / kRotBlocks);
        auto issue_chunk = [&](int c) {  // one thread
            const int64_t b = rb0 + (int64_t)c * kRotBlocks;
            const int64_t e = b + kRotBlocks < rb1 ? b + kRotBlocks : rb1;
            const uint32_t bytes = (uint32_t)((e - b) * kGroup * 2);
            mbar_arrive_expect_tx(rot_bar + c % kRotBufs, bytes);
            bulk_load(smem + (c % kRotBufs) * kRotBufBytes, x + b * kGroup, bytes, rot_bar + c % kRotBufs);
        };
        if (tid == 0) {
            for (int i = 0; i < kRotBufs; i++) mbar_init(rot_bar + i, 1);
            mbar_init_fence();
            for (int c = 0; c < kRotBufs && c < nchunks; c++) issue_chunk(c);
        }
        __syncthreads();
        int c = 0;
        for (; c < nchunks; c++) {
            const bool got = mbar_wait(rot_bar + c % kRotBufs, (uint32_t)(c / kRotBufs) & 1u);
            if (__syncthreads_or(!got)) {
                rot_fail = true;
                break;
            }
            const int64_t b = rb0 + (int64_t)c * kRotBlocks;
            const int64_t e = b + kRotBlocks < rb1 ? b + kRotBlocks : rb1;
            const uint8_t *buf = smem + (c % kRotBufs) * kRotBufBytes;
            for (int64_t blk = b + warp; blk < e; blk += kWarps) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(buf + (blk - b) * (kGroup * 2) + lane * 8);
                const float2 f01 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
                const float2 f23 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
                float v[4] = {f01.x, f01.y, f23.x, f23.y};
                rotate_store_f16<kFmt == 3 ? 16 : 8>(v, xr, blk, lane);
            }
            // these reads of the buffer before the copy that refills it
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (tid == 0 && c + kRotBufs < nchunks) issue_chunk(c + kRotBufs);
        }
        if (rot_fail && tid == 0)  // let the copies in flight land before the rings are reused
            for (int c2 = c; c2 < nchunks && c2 < c + kRotBufs; c2++)
                mbar_wait(rot_bar + c2 % kRotBufs, (uint32_t)(c2 / kRotBufs) & 1u);
        // these generic-proxy stores before the async-proxy (TMA) loads of any CTA
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
    }
    __syncthreads();
    unsigned long long arrival = 0;
    if (tid == 0) arrival = atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls), 1ull);

    if (tid == 0) {
        for (int st = 0; st < STAGES; st++) {
            mbar_init(full_a + st, 1);
            // (kPair: the even CTA's barrier also takes the odd CTA's forwarded arrival)
            mbar_init(full_b + st, kExpandWarps + (kPair && rank == 0 ? 1 : 0));
            mbar_init(empty + st, 1);
        }
        mbar_init(done, 1);
        mbar_init(tmem_free, kExpandWarps + (kPair && rank == 0 ? 1 : 0));
        mbar_init(fin, 1);
        *abort_flag = rot_fail ? 1 : 0;
        mbar_init_fence();
        // this call's epoch; the last CTA to arrive advances the counter (skipping
        // 0xffffffff, so that the epoch is never 0), which releases the barrier
        const uint32_t calls = (uint32_t)(arrival >> 32);
        *epoch_s = calls + 1u;
        if ((uint32_t)arrival == (uint32_t)nctas - 1u) {
            const unsigned long long step = calls + 1u == 0xffffffffu ? 2ull : 1ull;
            atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls),
                      (step << 32) - (unsigned long long)nctas);
        }
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
        if (kPair) {  // the same warp in both CTAs of the pair, the same slot address
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                         "r"(C::kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)),
                         "r"(C::kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    // kPair: both CTAs' barriers exist before the first arrival from the peer
    if (kPair) cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t epoch = *epoch_s;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (x' tiles)
        if (lane == 0) {
            // every CTA's x' is written: the call counter has moved past this call's arrivals
            {
                uint32_t i = 0;
                for (; i < kSpinLimit; i++) {
                    if (ld_acquire_u32(ctl + kCtlCalls + 1) != epoch - 1u) break;
                    __nanosleep(32);
                }
                if (i == kSpinLimit) *abort_flag = 1;
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            int it = 0;  // units issued: ring position
            for (int v = 0; v < n_mine && !*abort_flag;) {
                const Piece p = piece_at(v);
                const int tm = p.s % mt, tn = p.s / mt;
                for (int ks = p.kb; ks < p.ke; ks++, it++) {
                    const int st = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (*abort_flag || !mbar_wait(empty + st, ph ^ 1u)) {
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(full_a + st,
                                          C::kAStage + (kTma ? C::kCodeStage : 0));
#pragma unroll
                    for (int a = 0; a < kAcc; a++)
                        tma_load_2d(sA + st * C::kAStage + a * (BM * BK * 2), &a_map, full_a + st, ks * BK,
                                    acc_row0(tm, a));
                    // kPair: this CTA's 128 weight rows of the tile (SwiGLU: rank 0 the gate
                    // rows, rank 1 the matching up rows)
                    if (kTma && kPair)
                        tma_load_2d(const_cast<uint8_t *>(sCodes) + st * C::kCodeStage, &w_map, full_a + st,
                                    ks * (BK / 4),
                                    kSwiglu ? (rank == 0 ? tn * (BN / 2) : F + tn * (BN / 2)) : tn * BN + rank * 128);
                    // PQ2_0: the stage's codes, 16 bytes of each of the tile's 256 weight rows
                    if (kTma && !kSwiglu && !kPair)
                        tma_load_2d(const_cast<uint8_t *>(sCodes) + st * C::kCodeStage, &w_map, full_a + st,
                                    ks * (BK / 4), tn * BN);
                    if (kTma && kSwiglu && !kPair) {  // 128 gate rows, then the matching 128 up rows
                        tma_load_2d(const_cast<uint8_t *>(sCodes) + st * C::kCodeStage, &w_map, full_a + st,
                                    ks * (BK / 4), tn * (BN / 2));
                        tma_load_2d(const_cast<uint8_t *>(sCodes) + st * C::kCodeStage + C::kCodeStage / 2,
                                    &w_map, full_a + st, ks * (BK / 4), F + tn * (BN / 2));
                    }
                }
                v += p.ke - p.kb;
            }
            // the copies this thread started land before the CTA may exit
            for (int i = it - STAGES < 0 ? 0 : it - STAGES; i < it; i++)
                mbar_wait(full_a + (i % STAGES), (uint32_t)(i / STAGES) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (kPair: the even CTA)
        if (lane == 0 && rank == 0) {
            int it = 0, pc = 0;
            for (int v = 0; v < n_mine && !*abort_flag; pc++) {
                const Piece p = piece_at(v);
                v += p.ke - p.kb;
                // the accumulator is free once the previous piece's epilogue has read it (kPair:
                // the epilogues of both CTAs)
                if (pc > 0 && !(kPair ? mbar_wait_cluster(tmem_free, (uint32_t)(pc - 1) & 1u)
                                      : mbar_wait(tmem_free, (uint32_t)(pc - 1) & 1u))) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                for (int ks = p.kb; ks < p.ke; ks++, it++) {
                    const int st = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    // kPair: full_b completes once this CTA's expansion warps have written their
                    // B half and the odd CTA's forwarder has seen its half written and its x' in
                    if (*abort_flag || !mbar_wait(full_a + st, ph) ||
                        !(kPair ? mbar_wait_cluster(full_b + st, ph) : mbar_wait(full_b + st, ph))) {
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b0 = saddr(sB + st * C::kBStage);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; kk++) {
                        const uint64_t bdesc = desc_sw128(b0 + kk * 32);
#pragma unroll
                        for (int a = 0; a < kAcc; a++) {
                            const uint32_t a0 = saddr(sA + st * C::kAStage + a * (BM * BK * 2));
                            if (kPair)
                                mma_f16_pair(tmem + (uint32_t)(a * 256), desc_sw128(a0 + kk * 32), bdesc,
                                             (ks > p.kb || kk > 0) ? 1u : 0u);
                            else
                                mma_f16(tmem + (uint32_t)(a * 256), desc_sw128(a0 + kk * 32), bdesc,
                                        (ks > p.kb || kk > 0) ? 1u : 0u);
                        }
                    }
                    // frees the stage when these MMAs have read it (kPair: in both CTAs)
                    if (kPair)
                        mma_commit_pair(empty + st);
                    else
                        mma_commit(empty + st);
                }
                if (*abort_flag) break;
                // the piece's sums are complete in tensor memory
                if (kPair)
                    mma_commit_pair(done);
                else
                    mma_commit(done);
            }
            // every MMA this thread issued has completed before tensor memory is freed
            if (kPair)
                mma_commit_pair(fin);
            else
                mma_commit(fin);
            mbar_wait(fin, 0);
        } else if (kPair && lane == 0) {
            // the odd CTA: its expansion warps arrive on its own barriers, and this thread
            // forwards each completed stage (B half written, x' and codes landed) and each
            // freed accumulator to the even CTA's barriers with one cluster-scope arrival.
            // (An arrival with cluster-scope release waits for all of the arriving thread's
            // earlier memory operations; here that is one idle thread, not the expansion
            // warps with their scale and code loads in flight.)  The events come in the
            // order the expansion warps make them: a piece's stages, then its accumulator.
            const uint32_t full_b_lead = cluster_addr(full_b, 0);
            const uint32_t tmem_free_lead = cluster_addr(tmem_free, 0);
            int it = 0;
            bool ok = true;
            for (int v = 0, pc = 0; v < n_mine && ok; pc++) {
                const Piece p = piece_at(v);
                v += p.ke - p.kb;
                for (int ks = p.kb; ks < p.ke; ks++, it++) {
                    const int st = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (*abort_flag || !mbar_wait(full_b + st, ph) || !mbar_wait(full_a + st, ph)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_remote(full_b_lead + (uint32_t)(st * 8));
                }
                if (!ok || !mbar_wait(tmem_free, (uint32_t)pc & 1u)) {
                    ok = false;
                    break;
                }
                mbar_arrive_remote(tmem_free_lead);
            }
            if (!ok) *abort_flag = 1;
            // its shared memory and tensor memory serve the pair's MMAs until the even
            // CTA's last commit
            mbar_wait(fin, 0);
        }
    } else {
        // ------------------------------------------------ trit expansion (one row per thread), epilogues
        const int r = tid - 64;            // 0 .. 255
        const int q = warp & 3;            // TMEM lane quadrant this warp may read
        const int half = (warp - 2) >> 2;  // which 128 columns of the tile it writes
        // the B row this thread expands: its row rr of the CTA's B stage, row rb of the
        // tile's 256, and (kPair: two threads per row) which 32 of a stage's 64 weights
        const int rr = kPair ? (r & 127) : r;
        const int rb = kPair ? rank * 128 + rr : r;
        const int hsel = kPair ? (r >> 7) : 0;
        int it = 0, pc = 0;
        bool live = true;
        for (int v = 0; v < n_mine; pc++) {
            const Piece p = piece_at(v);
            v += p.ke - p.kb;
            const int tm = p.s % mt, tn = p.s / mt;
            const int64_t n = kSwiglu ? (rb < BN / 2 ? (int64_t)tn * (BN / 2) + rb : (int64_t)F + tn * (BN / 2) + rb - BN / 2)
                                      : (int64_t)tn * BN + rb;  // weight row
            // (SwiGLU: the last tile's gate rows past F belong to no output; their weights read as 0)
            const bool valid = kSwiglu ? (int64_t)tn * (BN / 2) + (rb & (BN / 2 - 1)) < F : n < N;
            if (live) {
                // PTQ1_0, Q1_0: the packed bytes of the group being expanded and of the next one (in
                // flight) come by plain loads; PQ2_0: the codes come with the stage's x' tiles
                // (TMA), only the scale by a plain load, one group ahead
                GroupRaw cur, nxt;
                const int g_last = (p.ke - 1) >> 1;
                uint32_t sc = 0u;
                if (!kTma && valid) load_group<kFmt>(packed, scales, n, G, p.kb >> 1, cur);
                if (kFmt == 2 && valid) sc = __ldg(scales + n * G + (p.kb >> 1));
                if (kFmt == 4 && valid) sc = __ldg(scales + n * G64 + p.kb);  // one scale per stage
                uint32_t cw[8];
                uint32_t tneg = 0u, tpos = 0u;  // the group's value table {-s, 0, +s}
                for (int ks = p.kb; ks < p.ke; ks++, it++) {
                    const int g = ks >> 1, hf = ks & 1;  // a 128-weight group fills two 64-wide stages
                    if (kFmt == 4) {  // a 64-weight scale group is one stage
                        tneg = valid ? sc ^ 0x8000u : 0u;
                        tpos = valid ? sc : 0u;
                        if (valid && ks + 1 < p.ke) sc = __ldg(scales + n * G64 + ks + 1);
                    } else if (ks == p.kb || hf == 0) {
                        if (kFmt == 2) {
                            tneg = valid ? sc ^ 0x8000u : 0u;
                            tpos = valid ? sc : 0u;
                            if (valid && g < g_last) sc = __ldg(scales + n * G + g + 1);
                        } else {
                            if (valid && g < g_last) load_group<kFmt>(packed, scales, n, G, g + 1, nxt);
                            if (valid) {
                                group_codes<kFmt>(cur, lut, cw);
                                tneg = (uint32_t)cur.scale ^ 0x8000u;
                                tpos = (uint32_t)cur.scale;
                            } else {
#pragma unroll
                                for (int i = 0; i < 8; i++) cw[i] = 0x55555555u;  // all trits zero
                            }
                            if (kFmt == 3)  // Q1_0: one table {-s, +s}
                                tneg = valid ? ((uint32_t)cur.scale ^ 0x8000u) | ((uint32_t)cur.scale << 16) : 0u;
                        }
                    }
                    const int st = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    // every lane acquires the stage itself (and, PQ2_0, its codes); the outcome
                    // is made warp-uniform
                    const bool free_ok = !*abort_flag && mbar_wait(empty + st, ph ^ 1u) &&
                                         (!kTma || mbar_wait(full_a + st, ph));
                    if (!__all_sync(0xffffffffu, free_ok)) {
                        *abort_flag = 1;
                        live = false;
                        break;
                    }
                    uint32_t w4[4];
                    if (kTma) {
                        const uint4 c4 = *reinterpret_cast<const uint4 *>(sCodes + st * C::kCodeStage + rr * 16);
                        w4[0] = c4.x, w4[1] = c4.y, w4[2] = c4.z, w4[3] = c4.w;
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; i++) w4[i] = hf ? cw[4 + i] : cw[i];
                    }
                    uint8_t *stage = sB + st * C::kBStage;
                    if (kFmt == 3) {
                        const uint32_t wq[2] = {hf ? cw[2] : cw[0], hf ? cw[3] : cw[1]};  // no dynamic index
#pragma unroll
                        for (int i = 0; i < (kPair ? 1 : 2); i++) {
                            const int ii = kPair ? hsel : i;  // (kPair: this thread's 32 weights)
                            uint32_t out[16];
                            expand_word_q1(ii ? wq[1] : wq[0], tneg, out);  // weights 64ks + 32ii .. +31
#pragma unroll
                            for (int c = 0; c < 4; c++) st_chunk(stage, rr, 4 * ii + c, out + 4 * c);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < (kPair ? 2 : 4); i++) {
                            const int wi = kPair ? 2 * hsel + i : i;  // (kPair: this thread's 32 weights)
                            const uint32_t wv = kPair ? (hsel ? w4[2 + i] : w4[i]) : w4[i];
                            uint32_t out[8];
                            expand_word(wv, tneg, tpos, out);  // weights 64ks + 16wi .. +15
                            st_chunk(stage, rr, 2 * wi, out);
                            st_chunk(stage, rr, 2 * wi + 1, out + 4);
                        }
                    }
                    // make the generic-proxy accesses (these stores, the code loads) ordered
                    // before later async-proxy ones, then signal
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full_b + st);
                    if (!kTma && hf == 1) cur = nxt;
                }
            }

            // ---------------------------------------------- epilogue of the piece
            if (live) live = __all_sync(0xffffffffu, mbar_wait(done, (uint32_t)pc & 1u)) && !*abort_flag;
            const bool ok = live;
            tc_fence_after();
            const bool continues = p.kb > 0;                  // a later piece of a tile
            const bool owner = p.kb == 0 && p.ke < nk;        // first piece, others follow
            const int tile_end = (p.tr + 1) * nk;  // in split units
            bool got = true;  // the later pieces all arrived (owner)
            if (owner)  // (the same rank's CTA of each later unit: its half of the tile)
                for (int c2 = unit + 1, s = u_end; s < tile_end; s = range_end(c2), c2++)
                    got = flag_wait(flags + cta_of(c2), epoch + epoch_skew, wait_limit) && got;
            if (!got && r == 0) atomicOr(status, kDevStatusGemmTimeout);
            const int w8 = warp - 2;
            if constexpr (kSwiglu) {
                // h columns [64 half, +64) of the tile's 128: gate accumulator columns
                // 64 half + 32 cc and up columns 128 + 64 half + 32 cc.  Hand-over slots are
                // in the order (accumulator a, TMEM quadrant q, 32-column chunk of 256, float4 i,
                // lane): writer and owner use the same mapping.
                auto sw_slot = [&](int c2, int a, int ch) {
                    return reinterpret_cast<float4 *>(partials + (size_t)c2 * kSlotFloats) +
                           ((size_t)((a * 4 + q) * 8 + ch) * 8) * 32 + lane;
                };
                uint8_t *stage_h = sB + w8 * 4096;  // 32 rows x 64 FP16, 16-byte chunks swizzled by the row
#pragma unroll 1
                for (int a = 0; a < kAcc; a++) {
#pragma unroll 1
                    for (int cc = 0; cc < 2; cc++) {
                        const int cg = 2 * half + cc, cu = 4 + cg;  // 32-column chunks of the 256
                        uint32_t vg[32], vu[32];
                        __syncwarp();
                        if (ok) {
                            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256 + 32 * cg), vg);
                            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256 + 32 * cu), vu);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; i++) vg[i] = vu[i] = 0x7fc00000u;
                        }
                        if (continues) {
                            float4 *dg = sw_slot(cta, a, cg), *du = sw_slot(cta, a, cu);
#pragma unroll
                            for (int i = 0; i < 8; i++) {
                                dg[32 * i] = make_float4(__uint_as_float(vg[4 * i]), __uint_as_float(vg[4 * i + 1]),
                                                         __uint_as_float(vg[4 * i + 2]), __uint_as_float(vg[4 * i + 3]));
                                du[32 * i] = make_float4(__uint_as_float(vu[4 * i]), __uint_as_float(vu[4 * i + 1]),
                                                         __uint_as_float(vu[4 * i + 2]), __uint_as_float(vu[4 * i + 3]));
                            }
                            continue;
                        }
                        if (owner) {
                            for (int c2 = unit + 1, s = u_end; s < tile_end; s = range_end(c2), c2++) {
                                const float4 *sg = sw_slot(cta_of(c2), a, cg), *su = sw_slot(cta_of(c2), a, cu);
#pragma unroll
                                for (int i = 0; i < 8; i++) {
                                    const float4 wg = __ldcg(sg + 32 * i), wu = __ldcg(su + 32 * i);
                                    vg[4 * i] = __float_as_uint(__uint_as_float(vg[4 * i]) + wg.x);
                                    vg[4 * i + 1] = __float_as_uint(__uint_as_float(vg[4 * i + 1]) + wg.y);
                                    vg[4 * i + 2] = __float_as_uint(__uint_as_float(vg[4 * i + 2]) + wg.z);
                                    vg[4 * i + 3] = __float_as_uint(__uint_as_float(vg[4 * i + 3]) + wg.w);
                                    vu[4 * i] = __float_as_uint(__uint_as_float(vu[4 * i]) + wu.x);
                                    vu[4 * i + 1] = __float_as_uint(__uint_as_float(vu[4 * i + 1]) + wu.y);
                                    vu[4 * i + 2] = __float_as_uint(__uint_as_float(vu[4 * i + 2]) + wu.z);
                                    vu[4 * i + 3] = __float_as_uint(__uint_as_float(vu[4 * i + 3]) + wu.w);
                                }
                            }
                            if (!got)
#pragma unroll
                                for (int i = 0; i < 32; i++) vg[i] = 0x7fc00000u;
                        }
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            uint32_t hw[4];
#pragma unroll
                            for (int e = 0; e < 4; e++) {
                                float hv[2];
#pragma unroll
                                for (int k2 = 0; k2 < 2; k2++) {
                                    const float g = __uint_as_float(vg[8 * j + 2 * e + k2]);
                                    hv[k2] = g / (1.f + expf(-g)) * __uint_as_float(vu[8 * j + 2 * e + k2]);
                                }
                                const __half2 p2 = __floats2half2_rn(hv[0], hv[1]);
                                hw[e] = *reinterpret_cast<const uint32_t *>(&p2);
                            }
                            *reinterpret_cast<uint4 *>(stage_h + lane * 128 + (((4 * cc + j) ^ (lane & 7)) << 4)) =
                                make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        }
                    }
                    if (continues) continue;
                    __syncwarp();
                    // four rows of 128 bytes per instruction: lane (row within four, 16-byte chunk)
                    const int ch = lane & 7;
                    const int64_t f0 = (int64_t)tn * (BN / 2) + half * 64 + ch * 8;
#pragma unroll 4
                    for (int i = 0; i < 8; i++) {
                        const int row = 4 * i + (lane >> 3);
                        const int m = acc_row0(tm, a) + 32 * q + row;
                        const uint4 val = *reinterpret_cast<const uint4 *>(stage_h + row * 128 + ((ch ^ (row & 7)) << 4));
                        if (m >= M || f0 >= F) continue;
                        uint16_t *hr = y + (int64_t)m * F + f0;
                        if (f0 + 8 <= F && (F & 7) == 0) {
                            *reinterpret_cast<uint4 *>(hr) = val;
                        } else {
                            const uint32_t wv[4] = {val.x, val.y, val.z, val.w};
                            for (int e = 0; e < 8 && f0 + e < F; e++) hr[e] = (uint16_t)(wv[e >> 1] >> (16 * (e & 1)));
                        }
                    }
                    __syncwarp();
                }
            } else {
            // Hand-over slots are kept in the order of the accumulator fragments (accumulator a,
            // warp, 32-column chunk c, float4 i, lane), so that writer and owner, which use the
            // same thread mapping, both move 512 contiguous bytes per warp instruction.
            auto slot_at = [&](int c2, int a, int c) {
                return reinterpret_cast<float4 *>(partials + (size_t)c2 * kSlotFloats) +
                       ((size_t)((a * kExpandWarps + w8) * 4 + c) * 8) * 32 + lane;
            };
            // y goes out through this warp's 8 KB of the B ring (idle until the next piece's
            // expansion): 32 rows x 128 FP16 columns, 16-byte chunks swizzled by the row.
            uint8_t *stage_y = sB + w8 * 8192;
#pragma unroll 1
            for (int a = 0; a < kAcc; a++) {
#pragma unroll 1
                for (int cp = 0; cp < 2; cp++) {
                    uint32_t v[64];
                    __syncwarp();
                    if (ok) {
                        tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256 + half * 128 + 64 * cp), v);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; i++) v[i] = 0x7fc00000u;
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; cc++) {
                        const int c = 2 * cp + cc;  // 32-column chunk of this warp's 128 columns
                        uint32_t *vc = v + 32 * cc;
                        if (continues) {
                            float4 *dst = slot_at(cta, a, c);
#pragma unroll
                            for (int i = 0; i < 8; i++)
                                dst[32 * i] = make_float4(__uint_as_float(vc[4 * i]), __uint_as_float(vc[4 * i + 1]),
                                                          __uint_as_float(vc[4 * i + 2]), __uint_as_float(vc[4 * i + 3]));
                            continue;
                        }
                        if (owner) {
                            for (int c2 = unit + 1, s = u_end; s < tile_end; s = range_end(c2), c2++) {
                                const float4 *src = slot_at(cta_of(c2), a, c);
                                float4 w[8];
#pragma unroll
                                for (int i = 0; i < 8; i++) w[i] = __ldcg(src + 32 * i);
#pragma unroll
                                for (int i = 0; i < 8; i++) {
                                    vc[4 * i] = __float_as_uint(__uint_as_float(vc[4 * i]) + w[i].x);
                                    vc[4 * i + 1] = __float_as_uint(__uint_as_float(vc[4 * i + 1]) + w[i].y);
                                    vc[4 * i + 2] = __float_as_uint(__uint_as_float(vc[4 * i + 2]) + w[i].z);
                                    vc[4 * i + 3] = __float_as_uint(__uint_as_float(vc[4 * i + 3]) + w[i].w);
                                }
                            }
                            if (!got)
#pragma unroll
                                for (int i = 0; i < 32; i++) vc[i] = 0x7fc00000u;
                        }
                        // FP16 (nearest even) into the staging row of this lane
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            uint32_t h[4];
#pragma unroll
                            for (int e = 0; e < 4; e++) {
                                const __half2 p2 = __floats2half2_rn(__uint_as_float(vc[8 * j + 2 * e]),
                                                                     __uint_as_float(vc[8 * j + 2 * e + 1]));
                                h[e] = *reinterpret_cast<const uint32_t *>(&p2);
                            }
                            *reinterpret_cast<uint4 *>(stage_y + lane * 256 + (((4 * c + j) ^ (lane & 7)) << 4)) =
                                make_uint4(h[0], h[1], h[2], h[3]);
                        }
                    }
                }
                if (continues) continue;
                __syncwarp();
                // two rows of 256 bytes per instruction: lane (row parity, 16-byte chunk)
                const int ch = lane & 15;
                const int64_t n0 = (int64_t)tn * BN + half * 128 + ch * 8;
#pragma unroll 4
                for (int i = 0; i < 16; i++) {
                    const int row = 2 * i + (lane >> 4);
                    const int m = acc_row0(tm, a) + 32 * q + row;
                    const uint4 val = *reinterpret_cast<const uint4 *>(stage_y + row * 256 + ((ch ^ (row & 7)) << 4));
                    if (m >= M || n0 >= N) continue;
                    uint16_t *yr = y + (int64_t)m * N + n0;
                    if (n0 + 8 <= N && (N & 7) == 0) {
                        *reinterpret_cast<uint4 *>(yr) = val;
                    } else {
                        const uint32_t wv[4] = {val.x, val.y, val.z, val.w};
                        for (int e = 0; e < 8 && n0 + e < N; e++) yr[e] = (uint16_t)(wv[e >> 1] >> (16 * (e & 1)));
                    }
                }
                __syncwarp();  // the staging rows are rewritten by the next accumulator
            }
            }  // kSwiglu
            // tensor memory has been read: the next piece's MMAs may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_free);
            if (continues) {
                __threadfence();
                expand_warps_sync();
                if (r == 0) flag_release(flags + cta, epoch);
            } else if (owner) {
                expand_warps_sync();  // every warp has read the later pieces and its staging rows
            } else {
                // the next piece's expansion writes the B ring, where other warps may still
                // be reading their staging rows
                expand_warps_sync();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(status, kDevStatusGemmTimeout);
    // kPair: neither CTA leaves (or frees its tensor memory) while the other may still
    // arrive on its barriers or the pair's MMAs may still use its memory
    if (kPair) cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if (kPair)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                         : "memory");
    }
}

// ---------------------------------------------------------------- host side

// Tile and grid of one call.  Stream-K leaves no partial last wave, so two 128-row
// accumulators (half the trit expansion per FLOP) are used whenever M > 128.
// tile_hint 3: CTA pairs (cta_group::2), tiles of 256 acc rows, acc = 2 when M > 256;
// the caller caps the pairs at the clusters that fit on the GPU at once.
struct GemmPlan {
    int acc, mt, nt, nk, ctas;
    bool pair;
    int64_t units;
};
GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, int tile_hint, int sm_count) {
    GemmPlan p;
    p.pair = tile_hint == 3;
    if (p.pair) {
        p.acc = M > 2 * BM ? 2 : 1;
        const int64_t rows = (int64_t)2 * BM * p.acc;
        p.mt = (int)((M + rows - 1) / rows);
        p.nt = (int)((N + BN - 1) / BN);
        p.nk = (int)(K / BK);
        p.units = (int64_t)p.mt * p.nt * p.nk;
        int64_t pairs = (p.units + 3) / 4;
        pairs = pairs < sm_count / 2 ? pairs : sm_count / 2;
        p.ctas = (int)(2 * (pairs > 0 ? pairs : 1));
        return p;
    }
    p.acc = tile_hint == 1 ? 1 : tile_hint == 2 ? 2 : (M > BM ? 2 : 1);
    p.mt = (int)((M + (int64_t)BM * p.acc - 1) / ((int64_t)BM * p.acc));
    p.nt = (int)((N + BN - 1) / BN);
    p.nk = (int)(K / BK);
    p.units = (int64_t)p.mt * p.nt * p.nk;
    // at least kMinUnits stages per CTA, at most one CTA per SM (all resident at once)
    constexpr int64_t kMinUnits = 4;
    int64_t c = (p.units + kMinUnits - 1) / kMinUnits;
    c = c < sm_count ? c : sm_count;
    p.ctas = (int)(c > 0 ? c : 1);
    return p;
}

constexpr size_t kSlotBytes = (size_t)2 * BM * BN * 4;  // one CTA's FP32 partial tile (two accumulators)

size_t x_rot_bytes(int64_t M, int64_t K) { return (((size_t)M * (size_t)K * 2) + 255) / 256 * 256; }

}  // namespace

bool gemm_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    if (fmt < 1 || fmt > 4) return false;
    // TMA coordinates are 32-bit; the unit count of the work split must fit an int
    if (!(M >= 1 && M < (int64_t)1 << 30 && N >= 1 && N < (int64_t)1 << 30 && K % kGroup == 0 &&
          K < (int64_t)1 << 30))
        return false;
    return ((M + BM - 1) / BM) * ((N + BN - 1) / BN) * (K / BK) < ((int64_t)1 << 31) / 4;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, const DeviceInfo &dev) {
    (void)N;
    (void)fmt;
    // x' in FP16, then one partial tile per CTA
    return x_rot_bytes(M, K) + (size_t)dev.sm_count * kSlotBytes;
}

cudaError_t launch_gemm(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int tile_hint,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev, int64_t swiglu_f) {
    const bool swiglu = swiglu_f > 0;
    if (swiglu && N != 2 * swiglu_f) return cudaErrorInvalidValue;
    GemmPlan plan = gemm_plan(M, N, K, tile_hint, dev.sm_count);
    if (ws.data_bytes < gemm_workspace_bytes(M, N, K, fmt, dev) || plan.ctas > kCtlGemmMaxCtas ||
        ws.zeroed_bytes < kCtlRegionBytes)
        return cudaErrorInvalidValue;
    uint16_t *xr = reinterpret_cast<uint16_t *>(ws.data);
    float *partials = reinterpret_cast<float *>(ws.data + x_rot_bytes(M, K));
    unsigned int *ctl = reinterpret_cast<unsigned int *>(ws.zeroed);
    const int64_t nblocks = M * (K / kGroup);
    const uint32_t limit = dev.force_wait_timeouts ? kForcedWaitPolls : kSpinLimit;
    const uint32_t skew = dev.force_wait_timeouts ? 0x80000000u : 0u;

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

    // PQ2_0 codes: rows of K/4 bytes, a box of 16 bytes x 256 rows per 64-wide stage
    CUtensorMap wmap = map;  // (unused by PTQ1_0)
    if (fmt == 2 || fmt == 4) {
        const cuuint64_t wdims[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
        const cuuint64_t wstrides[1] = {(cuuint64_t)(K / 4)};
        const cuuint32_t wbox[2] = {(cuuint32_t)(BK / 4), (cuuint32_t)(swiglu || plan.pair ? BN / 2 : BN)};
        if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), wdims, wstrides, wbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    auto go = [&](auto kern, int smem) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (!plan.pair) {
            kern<<<plan.ctas, kThreads, smem, s>>>(map, wmap, packed, scales, y, partials, x, xr, nblocks, ctl, limit,
                                                   skew, (int)M, (int)N, (int)K, plan.mt, (int)swiglu_f);
            return cudaGetLastError();
        }
        // clusters of two; only as many pairs as fit at once (the rotation phase's grid
        // barrier and the hand-over of split tiles wait on every CTA of the grid)
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)plan.ctas);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
        if (plan.ctas > 2 * clusters) cfg.gridDim = dim3((unsigned)(2 * clusters));
        return cudaLaunchKernelEx(&cfg, kern, map, wmap, packed, scales, y, partials, x, xr, nblocks, ctl, limit, skew,
                                  (int)M, (int)N, (int)K, plan.mt, (int)swiglu_f);
    };
    auto pick = [&](auto k1, auto k2) {
        if (plan.pair) return plan.acc == 2 ? go(k2, Cfg<2, true>::kSmemBytes) : go(k1, Cfg<1, true>::kSmemBytes);
        return plan.acc == 2 ? go(k2, Cfg<2>::kSmemBytes) : go(k1, Cfg<1>::kSmemBytes);
    };
    if (plan.pair) {
        if (swiglu) {
            if (fmt == 1) return pick(gemm_tcgen05_kernel<1, 1, true, true>, gemm_tcgen05_kernel<1, 2, true, true>);
            if (fmt == 3) return pick(gemm_tcgen05_kernel<3, 1, true, true>, gemm_tcgen05_kernel<3, 2, true, true>);
            if (fmt == 4) return pick(gemm_tcgen05_kernel<4, 1, true, true>, gemm_tcgen05_kernel<4, 2, true, true>);
            return pick(gemm_tcgen05_kernel<2, 1, true, true>, gemm_tcgen05_kernel<2, 2, true, true>);
        }
        if (fmt == 1) return pick(gemm_tcgen05_kernel<1, 1, false, true>, gemm_tcgen05_kernel<1, 2, false, true>);
        if (fmt == 3) return pick(gemm_tcgen05_kernel<3, 1, false, true>, gemm_tcgen05_kernel<3, 2, false, true>);
        if (fmt == 4) return pick(gemm_tcgen05_kernel<4, 1, false, true>, gemm_tcgen05_kernel<4, 2, false, true>);
        return pick(gemm_tcgen05_kernel<2, 1, false, true>, gemm_tcgen05_kernel<2, 2, false, true>);
    }
    if (swiglu) {
        if (fmt == 1) return pick(gemm_tcgen05_kernel<1, 1, true, false>, gemm_tcgen05_kernel<1, 2, true, false>);
        if (fmt == 3) return pick(gemm_tcgen05_kernel<3, 1, true, false>, gemm_tcgen05_kernel<3, 2, true, false>);
        if (fmt == 4) return pick(gemm_tcgen05_kernel<4, 1, true, false>, gemm_tcgen05_kernel<4, 2, true, false>);
        return pick(gemm_tcgen05_kernel<2, 1, true, false>, gemm_tcgen05_kernel<2, 2, true, false>);
    }
    if (fmt == 1) return pick(gemm_tcgen05_kernel<1, 1, false, false>, gemm_tcgen05_kernel<1, 2, false, false>);
    if (fmt == 3) return pick(gemm_tcgen05_kernel<3, 1, false, false>, gemm_tcgen05_kernel<3, 2, false, false>);
    if (fmt == 4) return pick(gemm_tcgen05_kernel<4, 1, false, false>, gemm_tcgen05_kernel<4, 2, false, false>);
    return pick(gemm_tcgen05_kernel<2, 1, false, false>, gemm_tcgen05_kernel<2, 2, false, false>);
}

}  // namespace bonsai
