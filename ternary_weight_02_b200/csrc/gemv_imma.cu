// gemv_imma.cu -- batch-1 and batch-2 (M <= 2) ternary GEMV for PQ2_0 (one FP16 scale per
// 128 or per 64 weights) on the integer tensor cores, with the block Hadamard rotation of
// x fused in.
//
// Operation: y[n] = sum_g s[n][g] * sum_j t[n][128g+j] * x'[128g+j], x' = blockdiag(Hn) x;
// with 64-weight scale groups each 128-group's sum splits into two halves, each with its
// own scale (PQ2_0 g64, the Q2_0_g64 files of "Bonsai把 27B 大模型塞进手机的极端量化方案
// 到底靠不靠谱" (wmrh.cn), sections 快速上手 and 后端支持现状).
// Sources: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com): method paragraph
// (trits, FP16 scale per 128 weights, block Hadamard), paragraph on running the files
// (activation-side Hadamard), paragraph on the two packings (PQ2_0: one trit per 2-bit
// slot); "Bonsai 2，把27B压进6个G" (10100.com), section 它怎么做到的.
//
// Design (B200, HBM-bound: 34 bytes per 128 weights):
//
// * At ~6.5 TB/s an SM must take in ~22 weight bytes per clock.  mma.sync issues at
//   ~0.38 per clock per SM on this part, so one MMA has to cover well over 64 bytes.
//   The u8 x s8 m16n8k32 MMA covers 16 rows x 32 weights = 128 bytes once its eight
//   columns are used for (4 scale groups) x (high byte, low byte) of the activations:
//   the weights of group gl meet a B operand that is non-zero in columns 2gl, 2gl+1
//   only, so four groups accumulate side by side in one fragment.
// * Activations as 16-bit block fixed point.  Per 128-group, x~ = rint(x' * 2^e) with
//   the power of two chosen so that the group's largest |x'| * 2^e lies in [2^13, 2^14),
//   stored as signed bytes hi * 256 + lo.  With c = t + 1 the PQ2_0 code of a weight, the
//   MMA gives sum c*hi and sum c*lo exactly in int32, so sum t*x~ = 256*Dhi + Dlo - sum x~
//   exactly; one FP32 multiply by s * 2^-e per (row, group) follows.  The rounding of x'
//   to x~ is the only approximation: every element is off by at most half a step 2^-e,
//   2^-15 to 2^-14 of the group's largest element.  That is finer than FP16 for the
//   group's elements above about 1/8 of its largest and coarser for those below (an
//   element 1000 times smaller than the group's largest keeps about 4 significant bits).
//   With 64-weight scales the MMA chain runs over the group's first two 32-weight
//   subslots, is folded with the first half's sum of x~ and scale, then over the last
//   two: the same accumulator registers, one more fold per group.
// * One launch.  16 warps per CTA, each feeding its own ring of item buffers (a TMA
//   box of trits, and the item's scales by cp.async).  After waiting for the previous
//   kernel, every CTA loads all of x (each CTA starting at a different group quad), then
//   starts its weight copies, then rotates and quantises x into x~ fragments in shared
//   memory (8 lanes per group) while the first items arrive.
// * Decode.  A 32-bit weight word holds 16 codes; (w >> 2j) & 0x03030303 is code j of
//   its four bytes as four u8 lanes of an A register.  The three shifts are done as
//   multiply-high by 2^(32-2j) (FMA pipe), the masks on the ALU pipe.
// * A work item is 32 rows x 512 weights: one TMA box of the trit plane (4 KB, 128-byte
//   swizzle).  MMA row gid reads shared-memory row 2*gid (gid < 4) or 2*gid - 7, so
//   that the eight rows one 64-bit load touches fall in distinct swizzle phases (no
//   bank conflicts).
// * Work split.  Items are ordered (row tile, K chunk); each CTA takes one contiguous
//   range, dealt round-robin to its consumer warps.  Every item's 32 row sums go to a
//   slot in shared memory; the warp that completes the CTA's part of a row tile adds its
//   slots in K order.  A tile shared with the following CTAs goes through 64-bit
//   (value, epoch) pairs in the workspace: the CTA holding the tile's first item adds
//   the later pieces in K order (deterministic).  The epoch is a call number kept in
//   the workspace's control words, so stored pairs never need clearing and a late pair
//   can never be taken for a later call's.
// * Several tokens (kM = 2 or 3; g64: 2).  The batch-1 layout spends an MMA's eight
//   columns on four groups x (high, low byte), and the loop is bound by the rate of
//   mma.sync, so more tokens there would mean more MMAs.  Instead one MMA covers one
//   group's 32 weights of one code slot (each lane of a quad 8 bytes of the group, the
//   same bytes for the four slots), and its columns carry (token, high/low byte); with
//   64-weight scales (half, token, high/low byte), a column meeting only its half's
//   weights.  The MMAs per item stay 32, the masks 128.  Each token has its own x~
//   fragments, sums and exponents, so shared memory limits K (max_k).
// * Every wait is bounded.  A warp whose mbarrier wait gives up stops refilling, turns
//   its results into NaN (keeping the partial-sum protocol intact) and, before the
//   CTA exits, waits (again bounded) for the copies it had started; an owner whose wait
//   for a later piece gives up writes NaN for that tile.  Both set a bit in the
//   workspace's device status word.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace bonsai {
namespace {

constexpr int kConsumers = 16;                          // warps; each feeds its own ring
constexpr int kThreads = kConsumers * 32;
constexpr int kItemRows = 32;
constexpr int kItemK = 512;
constexpr int kItemRowBytes = kItemK / 4;               // 128 bytes of PQ2_0 codes
constexpr int kItemBytes = kItemRows * kItemRowBytes;   // 4096
constexpr int kScaleRingBytes = kItemRows * 16;         // per stage: the item's 4 (g64: 8) scales of each row
constexpr int kXHalfBytes = 144;                        // one part (hi or lo) of a group's fragments, padded
constexpr int kXGroupBytes = 2 * kXHalfBytes;
constexpr int kStages = 2;
// Items each warp requests before building x~; the rest of its ring after: every
// warp's first item then arrives in the first half of the start-up burst.
constexpr int kFirstIssue = 1;
constexpr int kMaxCtaItems = 96;                        // slot buffer: 96 x 32 floats
constexpr int kMaxCtaTiles = kMaxCtaItems + 2;          // row tiles one CTA's items touch
constexpr int64_t kMaxK = 24576;   // the layout below then fits the 227 KB a CTA may use
constexpr int64_t kMaxK2 = 12288;  // the same with two tokens' x~
constexpr int64_t kMaxK3 = 6144;   // three tokens
__host__ __device__ constexpr int64_t max_k(int M) { return M == 1 ? kMaxK : M == 2 ? kMaxK2 : kMaxK3; }
constexpr uint32_t kCodeMask = 0x03030303u;

// Shared memory, from a 1024-byte aligned base (each 4 KB weight buffer stays 1024-byte
// aligned, as the 128-byte swizzle of its TMA box requires):
// [weight rings: kConsumers x kStages x 4096][scale rings: kConsumers x kStages x 512]
// [x~ fragments G4 x 288][(64 sum x~, 2^-e / 64) x G4][64 sum of the first 64 x~ x G4]
// [slots kMaxCtaItems x 128][row-tile counts][256 zero bytes][full barriers]
struct Layout {
    int sring, xfrag, sxf, sxl, slots, tcnt, zero, full, total;
};

// Alignment: the weight buffers 1024 bytes (swizzled TMA destinations), the fragment,
// slot and zero areas 16 bytes (128-bit loads), the barriers 8 bytes.
// (M tokens: M copies of the x~ areas, token-major, and M floats per item row in the slots.)
__host__ __device__ inline Layout make_layout(int K, int M) {
    Layout L;
    const int G4 = ((K + kItemK - 1) / kItemK) * 4;
    L.sring = kConsumers * kStages * kItemBytes;
    L.xfrag = L.sring + kConsumers * kStages * kScaleRingBytes;
    L.sxf = L.xfrag + M * G4 * kXGroupBytes;
    L.sxl = L.sxf + M * G4 * 8;
    L.slots = L.sxl + ((M * G4 * 4 + 15) & ~15);
    L.tcnt = L.slots + kMaxCtaItems * kItemRows * 4 * M;
    L.zero = (L.tcnt + kMaxCtaTiles * 4 + 15) & ~15;  // 128-bit loads read the zero bytes
    L.full = L.zero + 256;
    L.total = L.full + kConsumers * kStages * 8 + 16 + 1024;  // + the epoch word, room to align the base
    return L;
}


// D += A * B, A 16 x 32 u8 (row-major fragments), B 32 x 8 s8, D int32.
__device__ __forceinline__ void imma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                     uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B (C = 0): the first MMA of an accumulator chain, so no register is zeroed.
__device__ __forceinline__ void imma0(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// ---------------------------------------------------------------- x -> x~ fragments

// Loads the 32 bytes of x lane l of group g holds (zeros past the last group).
__device__ __forceinline__ void load_x8(const uint16_t *__restrict__ x, int g, int G, int l, uint4 &r0, uint4 &r1) {
    if (g < G) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)g * kGroup + 16 * l);
        r0 = src[0];
        r1 = src[1];
    } else {
        r0 = r1 = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Eight lanes per 128-group, four groups per warp; lane l (0..7) of a group holds
// elements k = 16l + m, m = 0..15.  Fragment layout of group g, part p (0: high byte,
// 1: low byte), B-operand slot (s, j) of the MMA that meets code slot j of the weights'
// 8-byte subslot s: element k = 32*s + 16*hb + 4*i + j is byte (8*(j & 1) + 4*hb + i) of
// 16-byte chunk 2*s + (j >> 1) in the 144-byte half-block (2g + p).  The 16 bytes of
// padding per half-block put the eight lanes that load one chunk of four consecutive
// groups on distinct shared-memory banks.  Lane l = 2*s + hb writes whole words.  With
// several tokens the half-blocks of token m sit at 288 m within a group's gstride bytes.
// Rotates and quantises group g (its x in r0, r1 of the group's 8 lanes) into the
// fragment area, (64 * sum x~, 2^-e / 64) into sxf[g] and 64 * the sum of its first 64
// x~ (lanes 0..3 of the group) into sxl[g].
__device__ __forceinline__ void build_group8(uint4 r0, uint4 r1, uint8_t *xfrag, int gstride, int2 *sxf, int *sxl,
                                             int g, int lane) {
    const int l = lane & 7;
    const unsigned int gmask = 0xffu << (lane & 24);
    float v[16];
    {
        const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    // index bits 0..3 inside the lane
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int i = 0; i < 16; i++)
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
    // index bits 4..6 are lane bits 0..2
#pragma unroll
    for (int b = 0; b < 3; b++) {
        const int mask = 1 << b;
        const float sgn = (l & mask) ? -1.f : 1.f;  // upper half: partner - own; lower: own + partner
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float p = __shfl_xor_sync(gmask, v[i], mask);
            v[i] = fmaf(sgn, v[i], p);  // exact sign flip, one rounding: same as the add or subtract
        }
    }
    // v holds the unnormalised transform: 1/sqrt(128) is folded into the quantisation
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i++) am = fmaxf(am, fabsf(v[i]));
#pragma unroll
    for (int b = 1; b < 8; b <<= 1) am = fmaxf(am, __shfl_xor_sync(gmask, am, b));
    const uint32_t mb = __float_as_uint(am * kHadamardNorm);  // max |x'| of the group
    const int E = (int)(mb >> 23) - 127;  // max |x'| < 2^(E+1)
    int e = mb == 0u ? 0 : 13 - E;        // max |x'| * 2^e < 2^14
    e = e < -126 ? -126 : (e > 100 ? 100 : e);
    const float sc = __int_as_float((e + 127) << 23) * kHadamardNorm;
    // 2^-e / 64: the GEMV's sums come out 64 times too large (code slots weighted 4^(3-j))
    const float f = E == 128 ? __int_as_float(0x7fc00000) : __int_as_float((121 - e) << 23);  // Inf/NaN -> NaN
    // q = rint(v * sc) by the magic-number rounding: v*sc + (1.5*2^23 + 128) lands in
    // [2^23, 2^24), where floats are the integers, so its bits minus those of 1.5*2^23
    // are q + 128 (|q| <= 2^14 + 1).  Then the high byte hi = (q + 128) >> 8 is byte 1
    // of qa = q + 128 and the low byte lo = q - 256 hi is byte 0 of qa with its top bit
    // flipped.
    int qa[16];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        qa[i] = (int)(__float_as_uint(fmaf(v[i], sc, 12583040.0f)) - 0x4B400000u);
        sum += qa[i];
    }
    sum += __shfl_xor_sync(gmask, sum, 1);
    sum += __shfl_xor_sync(gmask, sum, 2);
    const int sum_lo = sum - 128 * (kGroup / 2);  // lane 0: elements 0..63
    sum += __shfl_xor_sync(gmask, sum, 4);
    sum -= 128 * kGroup;  // the 128 added to each of the group's q
    // lane l = 2s + hb: chunk 2s + (j >> 1), byte 8 (j & 1) + 4 hb + i (element 16l + 4i + j)
    uint8_t *dst = xfrag + g * gstride + (l >> 1) * 32 + (l & 1) * 4;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t a0 = (uint32_t)qa[j], a1 = (uint32_t)qa[4 + j];
        const uint32_t a2 = (uint32_t)qa[8 + j], a3 = (uint32_t)qa[12 + j];
        const uint32_t whi = __byte_perm(__byte_perm(a0, a1, 0x0051), __byte_perm(a2, a3, 0x0051), 0x5410);
        const uint32_t wlo =
            __byte_perm(__byte_perm(a0, a1, 0x0040), __byte_perm(a2, a3, 0x0040), 0x5410) ^ 0x80808080u;
        const int off = (j >> 1) * 16 + (j & 1) * 8;
        *reinterpret_cast<uint32_t *>(dst + off) = whi;
        *reinterpret_cast<uint32_t *>(dst + kXHalfBytes + off) = wlo;
    }
    if (l == 0) {
        sxf[g] = make_int2(sum * 64, __float_as_int(f));
        sxl[g] = sum_lo * 64;
    }
}

// ---------------------------------------------------------------- the GEMV

// A later piece's partial sums travel as 64-bit (value, epoch) pairs, one per row: an
// aligned 64-bit access is single-copy atomic, so a reader that sees this call's epoch
// sees the value stored with it -- no fence on either side.
__device__ __forceinline__ void st_pair(uint64_t *p, float v, uint32_t epoch) {
    const uint64_t w = (uint64_t)__float_as_uint(v) | ((uint64_t)epoch << 32);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_pair(const uint64_t *p) {
    uint64_t w;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}
// Bounded wait, by the whole warp, for the 32 pairs at p (one per lane) to carry the
// epoch `want`; returns this lane's value, or NaN (and sets the status bit) if they did
// not all come within `limit` polls.  The pairs are written by a CTA with a higher index,
// which writes them before it waits on anything itself.
__device__ __forceinline__ float wait_pairs(const uint64_t *p, int lane, uint32_t want, uint32_t limit,
                                            unsigned int *status) {
    for (uint32_t i = 0; i < limit; i++) {
        const uint64_t w = ld_pair(p + lane);
        if (__all_sync(0xffffffffu, (uint32_t)(w >> 32) == want)) return __uint_as_float((uint32_t)w);
        __nanosleep(32);
    }
    if (lane == 0) atomicOr(status, kDevStatusGemvPieceTimeout);
    return __int_as_float(0x7fc00000);
}



// kAsyncScales: K is a multiple of 512, so an item's four (g64: eight) scales of a row are
// 8 (16) aligned bytes, copied with cp.async as part of the item's copy; otherwise each
// lane loads the scales it needs when it processes the item.
//
// kG64: one scale per 64 weights (scales N x K/64).
//
// kSwiglu: the rows are a fused gate/up projection (gate rows 0 .. F-1, up rows F .. 2F-1,
// N = 2F) and the output is h = silu(gate) * up (F values).  Row tile v then holds gate
// rows 16v .. 16v+15 in its rows 0..15 and up rows F + 16v .. in rows 16..31 (two 16-row
// TMA boxes), so that the lane that finishes row r < 16 of the tile finds the matching up
// row in lane r + 16.  (When F % 16 != 0 the last tile's rows past gate row F - 1 belong to
// no output and are not written; its up box reads zeros past row 2F - 1.)
//
// ctl: the workspace's control words: the 64-bit call counter (calls counted so far in
// its high half, CTAs of the running call that have read it in its low half) and the
// sticky status bits.  wait_limit and epoch_skew are the polls of a wait for a later piece
// and an offset added to the epoch it waits for: kSpinLimit and 0, except under the test
// hook that makes those waits give up.
//
// kM: tokens (1 to 3; g64 1 or 2); x is kM x K and y kM x N (kSwiglu: kM x F), row-major.
template <bool kAsyncScales, bool kSwiglu, bool kG64, int kM>
__global__ void __launch_bounds__(kThreads, 1) gemv_imma_kernel(
    const __grid_constant__ CUtensorMap wmap, const uint16_t *__restrict__ x, const uint16_t *__restrict__ scales,
    uint16_t *__restrict__ y, uint64_t *__restrict__ partials, unsigned int *__restrict__ ctl, int N, int K, int F,
    uint32_t wait_limit, uint32_t epoch_skew) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    static_assert(kM == 1 || (kM <= 3 && (!kG64 || kM == 2)), "several tokens: up to 3 (g64: 2)");
    const Layout L = make_layout(K, kM);
    const int G = K / kGroup;
    const int GS = kG64 ? 2 * G : G;  // scales per row
    const int KC = (K + kItemK - 1) / kItemK;
    const int G4 = KC * 4;
    const int RT = (N + kItemRows - 1) / kItemRows;
    const int I = RT * KC;  // items (host-checked to fit)
    const int C = gridDim.x;
    // weight row of row lr (0 .. 31) of row tile rt
    auto row_of = [&](int rt, int lr) {
        return kSwiglu ? (lr < 16 ? 16 * rt + lr : F + 16 * rt + (lr - 16)) : rt * kItemRows + lr;
    };
    const int c0 = (int)((int64_t)I * blockIdx.x / C), c1 = (int)((int64_t)I * (blockIdx.x + 1) / C);
    const int nq = c1 - c0 > warp ? (c1 - c0 - warp + kConsumers - 1) / kConsumers : 0;  // this warp's items

    uint8_t *wring = smem + warp * kStages * kItemBytes;
    uint8_t *sring = smem + L.sring + warp * kStages * kScaleRingBytes;  // [stage][item row][16 bytes]
    uint8_t *xf = smem + L.xfrag;
    const int2 *sxf = reinterpret_cast<const int2 *>(smem + L.sxf);
    float *slots = reinterpret_cast<float *>(smem + L.slots);
    int *tile_cnt = reinterpret_cast<int *>(smem + L.tcnt);  // items done, per row tile of the range
    uint8_t *zero = smem + L.zero;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.full) + warp * kStages;
    uint32_t *epoch_s = reinterpret_cast<uint32_t *>(smem + L.full + kConsumers * kStages * 8);
    unsigned int *status = ctl + kCtlStatus;

    // item q of this warp: c0 + warp + q * kConsumers -> ring stage q % kStages.  Lane 0
    // starts the TMA box; lane r copies the item's four scales of row r (cp.async); one
    // cp.async group per item (empty past the end) keeps the group count in step.
    // (row tile, K chunk) of an item, advanced by kConsumers items per step
    const int step_rt = kConsumers / KC, step_kc = kConsumers - step_rt * KC;
    auto advance = [&](int &rt, int &kc) {
        kc += step_kc;
        rt += step_rt;
        if (kc >= KC) kc -= KC, rt++;
    };
    int n_issued = 0;
    int i_rt = (c0 + warp) / KC, i_kc = (c0 + warp) - ((c0 + warp) / KC) * KC;  // next item to issue
    auto issue = [&](int q) {
        if (q < nq) {
            const int rt = i_rt, kc = i_kc;
            advance(i_rt, i_kc);
            const int st = q % kStages;
            if (lane == 0) {
                mbar_arrive_expect_tx(full + st, kItemBytes);
                if (kSwiglu) {  // gate rows, then the matching up rows (16-row boxes)
                    tma_load_2d(wring + st * kItemBytes, &wmap, full + st, kc * kItemRowBytes, 16 * rt);
                    tma_load_2d(wring + st * kItemBytes + kItemBytes / 2, &wmap, full + st, kc * kItemRowBytes,
                                F + 16 * rt);
                } else {
                    tma_load_2d(wring + st * kItemBytes, &wmap, full + st, kc * kItemRowBytes, rt * kItemRows);
                }
            }
            if (kAsyncScales) {
                const int row = row_of(rt, lane);
                const bool v = row < N;
                if (kG64)
                    cp_async16_zfill(sring + st * kScaleRingBytes + lane * 16, scales + (v ? (int64_t)row * GS + kc * 8 : 0), v);
                else
                    cp_async8_zfill(sring + st * kScaleRingBytes + lane * 16, scales + (v ? (int64_t)row * GS + kc * 4 : 0), v);
            }
            n_issued++;
        }
        if (kAsyncScales) cp_async_commit();
    };

    if (lane == 0) {
        for (int st = 0; st < kStages; st++) mbar_init(full + st, 1);
        mbar_init_fence();
    }
    if (tid < 64) reinterpret_cast<uint32_t *>(zero)[tid] = 0u;
    for (int i = tid; i < kMaxCtaTiles; i += kThreads) tile_cnt[i] = 0;
    __syncthreads();
    // Nothing is requested before the wait: a CTA that starts late (its SM freed late by
    // the previous kernel) would otherwise queue its x loads behind its own weight copies,
    // and the call's time is set by its slowest CTA (measured: faster on every shape).
    pdl_launch_dependents();
    pdl_wait();  // x, y and the workspace may belong to the previous kernel
    // This call's epoch is one more than the calls counted so far.  One atomic add reads the
    // count and counts this CTA in the same 64-bit word, so every CTA sees the same count;
    // the last CTA to arrive advances it for the next call (its result is needed only after
    // the x~ build, which hides its latency).
    unsigned long long ctr = 0;
    if (tid == 0) ctr = atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls), 1ull);
    // x -> x~ fragments, four groups (a quad) per warp and round: all of this warp's x
    // first (token by token).  Every CTA reads all of x at the same moment, so each starts
    // at a different quad: the simultaneous requests spread over the lines of x instead of
    // piling up.
#pragma unroll
    for (int m = 0; m < kM; m++) {
        constexpr int kRounds = (int)((max_k(kM) / kItemK) * 4 / 4 + kConsumers - 1) / kConsumers;
        const int nquads = G4 / 4;
        const int rot = (int)(blockIdx.x % (unsigned)nquads);
        const uint16_t *xm = x + (int64_t)m * K;
        uint4 xr[kRounds][2];
#pragma unroll
        for (int r = 0; r < kRounds; r++) {
            const int quad = warp + r * kConsumers;
            int pq = quad + rot;
            if (pq >= nquads) pq -= nquads;
            if (quad < nquads) load_x8(xm, pq * 4 + (lane >> 3), G, lane & 7, xr[r][0], xr[r][1]);
        }
        if (m == 0)
            for (int q = 0; q < kFirstIssue; q++) issue(q);
#pragma unroll
        for (int r = 0; r < kRounds; r++) {
            const int quad = warp + r * kConsumers;
            int pq = quad + rot;
            if (pq >= nquads) pq -= nquads;
            if (quad < nquads)  // whole warps
                build_group8(xr[r][0], xr[r][1], xf + m * kXGroupBytes, kM * kXGroupBytes,
                             reinterpret_cast<int2 *>(smem + L.sxf) + m * G4,
                             reinterpret_cast<int *>(smem + L.sxl) + m * G4, pq * 4 + (lane >> 3), lane);
        }
    }
    for (int q = kFirstIssue; q < kStages; q++) issue(q);
    if (tid == 0) {
        const uint32_t calls = (uint32_t)(ctr >> 32);
        *epoch_s = calls + 1u;  // the count skips 0xffffffff, so the epoch is never 0
        if ((uint32_t)ctr == (uint32_t)C - 1u) {  // the last CTA: every CTA has its epoch
            const unsigned long long step = calls + 1u == 0xffffffffu ? 2ull : 1ull;
            atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlCalls), (step << 32) - (unsigned long long)C);
        }
    }
    __syncthreads();
    const uint32_t epoch = *epoch_s;

    // Lane (gid, tig) works on scale group tig of the item: MMA rows gid and gid + 8 of
    // each 16-row tile t are shared-memory rows r = 16t + gid (+ 8), whose group tig is
    // logical 16-byte chunks 2tig and 2tig + 1, stored at chunk ^ (r & 7) = chunk ^ gid.
    const uint32_t loff0 = (uint32_t)(gid * kItemRowBytes + (((2 * tig) ^ gid) << 4));
    const uint32_t loff1 = (uint32_t)(gid * kItemRowBytes + (((2 * tig + 1) ^ gid) << 4));
    // B columns 2gq, 2gq + 1 carry group gq's high and low bytes; lane (gid, tig) supplies
    // column gid for the k of lane quad tig, i.e. group tig: non-zero iff gid >> 1 == tig.
    const bool bactive = (gid >> 1) == tig;
    const uint8_t *xb_lane = bactive ? xf + (2 * tig + (gid & 1)) * kXHalfBytes : zero;
    const int xb_stride = bactive ? kXGroupBytes : 0;
    const int R = 8 * tig + gid;  // the item row this lane reports: (t, h) = (tig >> 1, tig & 1)

    bool ok = true;
    int n_waited = 0;
    int st = 0;
    uint32_t phase = 0;
    int rt = (c0 + warp) / KC, kc = (c0 + warp) - ((c0 + warp) / KC) * KC;
    // Row tiles split between CTAs: the CTA holding a tile's first item owns the tile and
    // adds the other pieces, which the CTAs that follow store as (value, epoch) pairs.  The
    // owner reaches its piece last (the end of its range), while the later pieces open
    // their CTAs' ranges and are stored as soon as their items are done.  Waits only go
    // from a CTA to higher ones, which store before they wait on anything: all CTAs of the
    // grid fit on the GPU at once (one per SM).
    const int rt_first = c0 / KC;
    // One warp per tile, one lane per row: add the CTA's items of tile rt ([a, b)) in K
    // order, then write y (whole tile), store the piece (a later piece) or collect the
    // later pieces and write y (owned); token by token.  Slots and pairs hold kM values
    // per item row, token-major within an item.
    auto finish_tile = [&](int rt, int a, int b) {
        const int tile_first = rt * KC, tile_end = tile_first + KC;
#pragma unroll
        for (int m = 0; m < kM; m++) {
            float sum = 0.f;
            for (int i = a; i < b; i++) sum += slots[((i - c0) * kM + m) * kItemRows + lane];
            if (a > tile_first) {
                st_pair(partials + ((int64_t)a * kM + m) * kItemRows + lane, sum, epoch);
                continue;
            }
            int s = b, c2 = (int)blockIdx.x + 1;
            while (s < tile_end) {
                int e2 = (int)((int64_t)I * (c2 + 1) / C);  // the piece of CTA c2 is [s, e2)
                e2 = e2 < tile_end ? e2 : tile_end;
                sum += wait_pairs(partials + ((int64_t)s * kM + m) * kItemRows, lane, epoch + epoch_skew, wait_limit,
                                  status);
                s = e2;
                c2++;
            }
            if (kSwiglu) {  // h = silu(gate) * up: lanes 0..15 hold gate rows, 16..31 the up rows
                const float up = __shfl_down_sync(0xffffffffu, sum, 16);
                const int f = 16 * rt + lane;
                if (lane < 16 && f < F) y[(int64_t)m * F + f] = float_to_half_bits(sum / (1.f + expf(-sum)) * up);
                continue;
            }
            const int row = rt * kItemRows + lane;
            if (row < N) y[(int64_t)m * N + row] = float_to_half_bits(sum);
        }
    };

    auto process = [&](int q) {
        const int i = c0 + warp + q * kConsumers;
        if (ok) {
            ok = __all_sync(0xffffffffu, mbar_wait(full + st, phase));
            if (ok)
                n_waited++;
            else if (lane == 0)
                atomicOr(status, kDevStatusGemvCopyTimeout);
        }
        const uint8_t *sb = wring + st * kItemBytes;
        uint4 raw[2][2][2];  // [t][h][16-byte half of the lane's 32 bytes]
        // (several tokens) [t][h][group]: bytes 8 tig .. 8 tig + 7 of each of the item's
        // four groups of row 16t + 8h + gid
        uint2 rawg[2][2][4];
        if constexpr (kM == 1) {
#pragma unroll
            for (int t = 0; t < 2; t++)
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    raw[t][h][0] = *reinterpret_cast<const uint4 *>(sb + loff0 + 2048 * t + 1024 * h);
                    raw[t][h][1] = *reinterpret_cast<const uint4 *>(sb + loff1 + 2048 * t + 1024 * h);
                }
        } else {
#pragma unroll
            for (int t = 0; t < 2; t++)
#pragma unroll
                for (int h = 0; h < 2; h++)
#pragma unroll
                    for (int g = 0; g < 4; g++)  // logical chunk 2g + tig / 2, swizzled by the row
                        rawg[t][h][g] = *reinterpret_cast<const uint2 *>(
                            sb + 2048 * t + 1024 * h + gid * kItemRowBytes + (((2 * g + (tig >> 1)) ^ gid) << 4) +
                            (tig & 1) * 8);
        }
        const int g0 = kc * 4;
        // (t, h) = (e >> 1, e & 1): scale of row 16t + 8h + gid, group g0 + tig (g64: the
        // group's two half scales, first half in the low 16 bits)
        uint32_t sc[4];
        // (several tokens) [t][h]: the four (g64: eight) scales of row 16t + 8h + gid in
        // this item, two to a word, the first in the low half
        uint32_t scw[2][2][kG64 ? 4 : 2];
        if (kAsyncScales) {
            cp_async_wait<kStages - 1>();  // this item's scales have landed (own copies)
            __syncwarp();                  // ... and every lane's
            if constexpr (kM == 1) {
                const uint8_t *sp = sring + st * kScaleRingBytes + gid * 16 + tig * (kG64 ? 4 : 2);
#pragma unroll
                for (int e = 0; e < 4; e++)
                    sc[e] = kG64 ? *reinterpret_cast<const uint32_t *>(sp + e * 128)
                                 : (uint32_t)*reinterpret_cast<const uint16_t *>(sp + e * 128);
            } else {
#pragma unroll
                for (int t = 0; t < 2; t++)
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint8_t *sp = sring + st * kScaleRingBytes + (16 * t + 8 * h + gid) * 16;
                        if constexpr (kG64) {
                            const uint4 u = *reinterpret_cast<const uint4 *>(sp);
                            scw[t][h][0] = u.x, scw[t][h][1] = u.y, scw[t][h][2] = u.z, scw[t][h][3] = u.w;
                        } else {
                            const uint2 u = *reinterpret_cast<const uint2 *>(sp);
                            scw[t][h][0] = u.x, scw[t][h][1] = u.y;
                        }
                    }
            }
        } else if constexpr (kM == 1) {
            const int g = g0 + tig;
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int row = row_of(rt, 8 * e + gid);
                const bool v = row < N && g < G;
                if (kG64)
                    sc[e] = v ? (uint32_t)__ldg(scales + (int64_t)row * GS + 2 * g) |
                                    ((uint32_t)__ldg(scales + (int64_t)row * GS + 2 * g + 1) << 16)
                              : 0u;
                else
                    sc[e] = v ? (uint32_t)__ldg(scales + (int64_t)row * GS + g) : 0u;
            }
        } else {
            constexpr int kPer = kG64 ? 8 : 4;  // scales of a row in one item
#pragma unroll
            for (int t = 0; t < 2; t++)
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    const int row = row_of(rt, 16 * t + 8 * h + gid);
#pragma unroll
                    for (int w = 0; w < kPer / 2; w++) {
                        const int q0 = kPer * kc + 2 * w;  // the row's scale index
                        const uint32_t lo = row < N && q0 < GS ? (uint32_t)__ldg(scales + (int64_t)row * GS + q0) : 0u;
                        const uint32_t hi =
                            row < N && q0 + 1 < GS ? (uint32_t)__ldg(scales + (int64_t)row * GS + q0 + 1) : 0u;
                        scw[t][h][w] = lo | (hi << 16);
                    }
                }
        }
        __syncwarp();
        if (ok) {  // refill this buffer with the warp's item q + kStages
            if (lane == 0) fence_proxy_async();
            issue(q + kStages);
        } else if (kAsyncScales) {
            cp_async_commit();
        }

        // Codes stay in place: (w & 0x03030303 << 2j) gives code slot j of the four bytes of
        // a word as u8 values c * 4^j.  One accumulator per (tile, j); the 4^j factors are
        // undone once per fold (the sums come out 64 times too large, folded into 2^-e).
        // One fold per group, or (g64) one per 64-weight half: subslots 0, 1 then 2, 3.
        constexpr int kFolds = kG64 ? 2 : 1, kSubPerFold = 4 / kFolds;
        // sum over the four groups (lanes of the quad) and leave (t, h) = (tig >> 1, tig & 1)
        // in lane tig: keep the pair whose h is the lane's, then the t
        auto quad_sum = [&](const float (&v)[4]) {
            const bool b0 = tig & 1;
            const float k0 = b0 ? v[1] : v[0], s0 = b0 ? v[0] : v[1];
            const float k1 = b0 ? v[3] : v[2], s1 = b0 ? v[2] : v[3];
            const float u0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 1);  // t = 0
            const float u1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 1);  // t = 1
            const bool b1 = tig & 2;
            const float kk = b1 ? u1 : u0, ss = b1 ? u0 : u1;
            return kk + __shfl_xor_sync(0xffffffffu, ss, 2);
        };
        if constexpr (kM == 1) {
        int d[2][4][4];
        const uint8_t *xb = xb_lane + g0 * xb_stride;
        const int2 sf = sxf[g0 + tig];  // (64 * sum x~, 2^-e / 64)
        const float fg = __int_as_float(sf.y);
        const int sfl = kG64 ? reinterpret_cast<const int *>(smem + L.sxl)[g0 + tig] : 0;  // first half's
        float v[4] = {0.f, 0.f, 0.f, 0.f};  // (t, h) = (e >> 1, e & 1)
#pragma unroll
        for (int fold = 0; fold < kFolds; fold++) {
#pragma unroll
        for (int s = fold * kSubPerFold; s < (fold + 1) * kSubPerFold; s++) {
            const uint4 b01 = *reinterpret_cast<const uint4 *>(xb + 32 * s);       // code slots 0, 1
            const uint4 b23 = *reinterpret_cast<const uint4 *>(xb + 32 * s + 16);  // code slots 2, 3
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t mask = kCodeMask << (2 * j);
                const uint32_t bx = j == 0 ? b01.x : (j == 1 ? b01.z : (j == 2 ? b23.x : b23.z));
                const uint32_t by = j == 0 ? b01.y : (j == 1 ? b01.w : (j == 2 ? b23.y : b23.w));
#pragma unroll
                for (int t = 0; t < 2; t++) {
                    // subslot s: bytes 8s..8s+7 of the group; a0/a2 = row gid bytes 0-3 / 4-7, a1/a3 = row gid + 8
                    const uint4 &r0 = raw[t][0][s >> 1], &r1 = raw[t][1][s >> 1];
                    const uint32_t w0 = (s & 1) ? r0.z : r0.x, w2 = (s & 1) ? r0.w : r0.y;
                    const uint32_t w1 = (s & 1) ? r1.z : r1.x, w3 = (s & 1) ? r1.w : r1.y;
                    if (s == fold * kSubPerFold)
                        imma0(d[t][j], w0 & mask, w1 & mask, w2 & mask, w3 & mask, bx, by);
                    else
                        imma(d[t][j], w0 & mask, w1 & mask, w2 & mask, w3 & mask, bx, by);
                }
            }
        }
        // lane (gid, tig) holds columns 2tig (hi) and 2tig+1 (lo): group g0 + tig (g64: its
        // half `fold`) of rows gid (d[t][j][0..1]) and gid + 8 (d[t][j][2..3])
        const int sx = kG64 ? (fold == 0 ? sfl : sf.x - sfl) : sf.x;  // 64 * sum of the fold's x~
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int t = e >> 1, h = e & 1;
            const int H = ((d[t][0][2 * h] * 4 + d[t][1][2 * h]) * 4 + d[t][2][2 * h]) * 4 + d[t][3][2 * h];
            const int Lo = ((d[t][0][2 * h + 1] * 4 + d[t][1][2 * h + 1]) * 4 + d[t][2][2 * h + 1]) * 4 +
                           d[t][3][2 * h + 1];
            const int T64 = H * 256 + Lo - sx;
            const uint16_t sbits = (uint16_t)(kG64 && fold == 1 ? sc[e] >> 16 : sc[e]);
            v[e] = fmaf((float)T64, half_bits_to_float(sbits) * fg, v[e]);
        }
        }
        float mine = quad_sum(v);
        if (!ok) mine = __int_as_float(0x7fc00000);
        slots[(i - c0) * kItemRows + R] = mine;
        } else {
            // Several tokens: MMA (t, g, j) meets code slot j of group g0 + g of tile t with
            // B columns (token, high/low byte) -- g64: (half, token, high/low byte), where a
            // column meets only its half's weights (the k of lane quads 2 hf, 2 hf + 1).
            // Lane (gid, tig) holds columns 2 tig, 2 tig + 1: token mt (g64: half ht).
            const int mt = kG64 ? (tig & 1) : tig;
            const int ht = kG64 ? (tig >> 1) : 0;
            const bool valid = mt < kM;
            const int mc = valid ? mt : 0;  // (the addresses an unused lane reads)
            // the B column this lane supplies: column gid, for the k of lane quad tig
            const int bm = kG64 ? ((gid >> 1) & 1) : (gid >> 1);
            const bool bact = bm < kM && (!kG64 || (gid >> 2) == (tig >> 1));
            const uint8_t *xbq = bact ? xf + bm * kXGroupBytes + (gid & 1) * kXHalfBytes + tig * 32 : zero;
            const int xq_stride = bact ? kM * kXGroupBytes : 0;
            const int2 *sxm = sxf + mc * G4;
            const int *sxlm = reinterpret_cast<const int *>(smem + L.sxl) + mc * G4;
            float v[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // [t][h]: row 16t + 8h + gid, token mt
#pragma unroll
            for (int g = 0; g < 4; g++) {
                const uint8_t *xb = xbq + (g0 + g) * xq_stride;
                const uint4 b01 = *reinterpret_cast<const uint4 *>(xb);       // code slots 0, 1
                const uint4 b23 = *reinterpret_cast<const uint4 *>(xb + 16);  // code slots 2, 3
                const int2 sf = sxm[g0 + g];  // (64 * sum x~, 2^-e / 64) of token mc
                const float fg = __int_as_float(sf.y);
                // 64 * the sum of x~ over the weights the lane's columns meet
                const int sx = kG64 ? (ht == 0 ? sxlm[g0 + g] : sf.x - sxlm[g0 + g]) : sf.x;
#pragma unroll
                for (int t = 0; t < 2; t++) {
                    const uint2 r0 = rawg[t][0][g], r1 = rawg[t][1][g];
                    int d[4][4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const uint32_t mask = kCodeMask << (2 * j);
                        const uint32_t bx = j == 0 ? b01.x : (j == 1 ? b01.z : (j == 2 ? b23.x : b23.z));
                        const uint32_t by = j == 0 ? b01.y : (j == 1 ? b01.w : (j == 2 ? b23.y : b23.w));
                        imma0(d[j], r0.x & mask, r1.x & mask, r0.y & mask, r1.y & mask, bx, by);
                    }
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const int H = ((d[0][2 * h] * 4 + d[1][2 * h]) * 4 + d[2][2 * h]) * 4 + d[3][2 * h];
                        const int Lo =
                            ((d[0][2 * h + 1] * 4 + d[1][2 * h + 1]) * 4 + d[2][2 * h + 1]) * 4 + d[3][2 * h + 1];
                        const int T64 = H * 256 + Lo - sx;
                        const int q = kG64 ? 2 * g + ht : g;  // the scale's index in the row's item
                        const uint16_t sbits = (uint16_t)(scw[t][h][q >> 1] >> (16 * (q & 1)));
                        v[t][h] = fmaf((float)T64, half_bits_to_float(sbits) * fg, v[t][h]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 2; t++)
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    if (kG64) v[t][h] += __shfl_xor_sync(0xffffffffu, v[t][h], 2);  // the other half
                    if (valid && ht == 0)
                        slots[((i - c0) * kM + mt) * kItemRows + 16 * t + 8 * h + gid] =
                            ok ? v[t][h] : __int_as_float(0x7fc00000);
                }
        }
        // the warp that completes the CTA's part of a row tile finalises it
        __syncwarp();
        int done = 0;
        if (lane == 0) {
            __threadfence_block();  // this warp's slot stores before the count
            done = atomicAdd(tile_cnt + (rt - rt_first), 1) + 1;
            __threadfence_block();  // the other warps' slot stores before the reads below
        }
        done = __shfl_sync(0xffffffffu, done, 0);
        const int tile_first = rt * KC;
        const int a = c0 > tile_first ? c0 : tile_first;
        const int b = c1 < tile_first + KC ? c1 : tile_first + KC;
        if (done == b - a) finish_tile(rt, a, b);
        if (++st == kStages) st = 0, phase ^= 1u;
        advance(rt, kc);
    };

    for (int q = 0; q < nq; q++) process(q);
    if (kAsyncScales) cp_async_wait_all();
    // after a wait gave up: let the box copies already started land before the CTA exits
    if (!ok && lane == 0) {
        int dst = n_waited % kStages;
        uint32_t dph = (uint32_t)((n_waited / kStages) & 1);
        for (int q = n_waited; q < n_issued; q++) {
            mbar_wait(full + dst, dph);
            if (++dst == kStages) dst = 0, dph ^= 1u;
        }
    }
}

struct Shape {
    int KC, G4, RT, I, grid;
};

Shape shape_of(int64_t N, int64_t K, int sm_count) {
    Shape s;
    s.KC = (int)((K + kItemK - 1) / kItemK);
    s.G4 = s.KC * 4;
    s.RT = (int)((N + kItemRows - 1) / kItemRows);
    s.I = s.RT * s.KC;
    int64_t grid = (s.I + kMaxCtaItems - 1) / kMaxCtaItems;  // every CTA's slots fit
    const int64_t want = (s.I + kConsumers - 1) / kConsumers;  // no idle consumer warps
    int64_t g2 = want < sm_count ? want : sm_count;
    if (grid < g2) grid = g2;
    s.grid = (int)grid;
    return s;
}

}  // namespace

static_assert(kConsumers * kStages * (kItemBytes + kScaleRingBytes) + (kMaxK / kItemK) * 4 * (kXGroupBytes + 12) +
                  kMaxCtaItems * kItemRows * 4 + kMaxCtaTiles * 4 + 15 + 256 + kConsumers * kStages * 8 + 16 + 1024 <=
                  232448,
              "shared-memory layout exceeds the per-CTA limit at the largest K");
static_assert(kConsumers * kStages * (kItemBytes + kScaleRingBytes) + 2 * (kMaxK2 / kItemK) * 4 * (kXGroupBytes + 12) +
                  2 * kMaxCtaItems * kItemRows * 4 + kMaxCtaTiles * 4 + 15 + 256 + kConsumers * kStages * 8 + 16 +
                  1024 <=
                  232448,
              "two-token shared-memory layout exceeds the per-CTA limit at its largest K");
static_assert(kConsumers * kStages * (kItemBytes + kScaleRingBytes) + 3 * (kMaxK3 / kItemK) * 4 * (kXGroupBytes + 12) +
                  3 * kMaxCtaItems * kItemRows * 4 + kMaxCtaTiles * 4 + 15 + 256 + kConsumers * kStages * 8 + 16 +
                  1024 <=
                  232448,
              "three-token shared-memory layout exceeds the per-CTA limit at its largest K");

bool gemv_imma_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    if ((fmt != 2 && fmt != 4) || M < 1 || M > (fmt == 4 ? 2 : 3) || N < 1 || K < kGroup || K % kGroup != 0 ||
        K > max_k((int)M))
        return false;
    const int64_t RT = (N + kItemRows - 1) / kItemRows;
    return RT * ((K + kItemK - 1) / kItemK) < ((int64_t)1 << 30);
}

// True when the call's grid fits on the GPU at once (at most one CTA per SM), which the
// hand-over between CTAs assumes: a CTA holds at most kMaxCtaItems items, so shapes with
// more than sm_count x kMaxCtaItems items are left to the other batch-1 kernels by the
// automatic choice.
bool gemv_imma_grid_fits(int64_t N, int64_t K, const DeviceInfo &dev) {
    return shape_of(N, K, dev.sm_count).grid <= dev.sm_count;
}

// the zero-initialised workspace region: the control words, then the (value, epoch) pairs
// of the pieces of row tiles split between CTAs, indexed by the piece's first item:
// items x M x 32 x 8 bytes.
size_t gemv_imma_zeroed_bytes(int64_t M, int64_t N, int64_t K) {
    const int64_t KC = (K + kItemK - 1) / kItemK;
    const int64_t items = ((N + kItemRows - 1) / kItemRows) * KC;
    return kCtlRegionBytes + (size_t)items * (size_t)M * kItemRows * sizeof(uint64_t);
}

cudaError_t launch_gemv_imma(const uint16_t *x, const uint8_t *packed, const uint16_t *scales, uint16_t *y,
                             int64_t M, int64_t N, int64_t K, int fmt, const Workspace &ws, cudaStream_t s,
                             const DeviceInfo &dev, int64_t swiglu_f) {
    if ((fmt != 2 && fmt != 4) || !gemv_imma_supported(M, N, K, fmt)) return cudaErrorInvalidValue;
    const bool swiglu = swiglu_f > 0;
    if (swiglu && N != 2 * swiglu_f) return cudaErrorInvalidValue;
    const Layout lay = make_layout((int)K, (int)M);
    if (lay.total > dev.smem_optin) return cudaErrorInvalidValue;
    // the kernel's 128-bit and barrier accesses rely on these alignments
    if ((lay.sring | lay.xfrag | lay.sxf | lay.slots | lay.zero) % 16 != 0 || lay.full % 8 != 0)
        return cudaErrorInvalidValue;
    EncodeTiledFn encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap wmap;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K / 4)};
        const cuuint32_t box[2] = {(cuuint32_t)kItemRowBytes, (cuuint32_t)(swiglu ? kItemRows / 2 : kItemRows)};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const Shape sh = shape_of(N, K, dev.sm_count);
    if (ws.zeroed_bytes < gemv_imma_zeroed_bytes(M, N, K)) return cudaErrorInvalidValue;
    unsigned int *ctl = reinterpret_cast<unsigned int *>(ws.zeroed);
    uint64_t *partials = reinterpret_cast<uint64_t *>(ws.zeroed + kCtlRegionBytes);
    // K a multiple of 512: an item's scales of a row are 8 (g64: 16) aligned bytes, copied
    // with the item
    using Kern = decltype(&gemv_imma_kernel<true, true, true, 1>);
    const bool async = K % kItemK == 0;
    Kern kern;
    if (M == 3) {
        kern = async ? (swiglu ? gemv_imma_kernel<true, true, false, 3> : gemv_imma_kernel<true, false, false, 3>)
                     : (swiglu ? gemv_imma_kernel<false, true, false, 3> : gemv_imma_kernel<false, false, false, 3>);
    } else if (M == 2) {
        if (fmt == 4)
            kern = async ? (swiglu ? gemv_imma_kernel<true, true, true, 2> : gemv_imma_kernel<true, false, true, 2>)
                         : (swiglu ? gemv_imma_kernel<false, true, true, 2> : gemv_imma_kernel<false, false, true, 2>);
        else
            kern = async ? (swiglu ? gemv_imma_kernel<true, true, false, 2> : gemv_imma_kernel<true, false, false, 2>)
                         : (swiglu ? gemv_imma_kernel<false, true, false, 2> : gemv_imma_kernel<false, false, false, 2>);
    } else if (fmt == 4) {
        kern = async ? (swiglu ? gemv_imma_kernel<true, true, true, 1> : gemv_imma_kernel<true, false, true, 1>)
                     : (swiglu ? gemv_imma_kernel<false, true, true, 1> : gemv_imma_kernel<false, false, true, 1>);
    } else {
        kern = async ? (swiglu ? gemv_imma_kernel<true, true, false, 1> : gemv_imma_kernel<true, false, false, 1>)
                     : (swiglu ? gemv_imma_kernel<false, true, false, 1> : gemv_imma_kernel<false, false, false, 1>);
    }
    // the attribute is set to the largest layout any K takes, so that launches of several
    // sizes captured into one graph all stay within it
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         make_layout((int)max_k((int)M), (int)M).total);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sh.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint32_t limit = dev.force_wait_timeouts ? kForcedWaitPolls : kSpinLimit;
    const uint32_t skew = dev.force_wait_timeouts ? 0x80000000u : 0u;
    return cudaLaunchKernelEx(&cfg, kern, wmap, x, scales, y, partials, ctl, (int)N, (int)K, (int)swiglu_f, limit,
                              skew);
}

}  // namespace bonsai
