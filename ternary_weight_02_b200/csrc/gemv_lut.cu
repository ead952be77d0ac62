// gemv_lut.cu -- batch-1 (M == 1) ternary GEMV for the packings, with the block
// Hadamard rotation of x fused in.  Q1_0 (1-bit, "Bonsai把 27B 大模型塞进手机的极端量化方案
// 到底靠不靠谱" (wmrh.cn), sections 核心观点 and 关键机制): a byte holds 8 signs, so its
// table covers 8 activations and a 128-byte row slice covers 1024 (split mode only).
// PQ2_0 g64 (one scale per 64 weights, the Q2_0_g64 files of the same wmrh.cn page,
// sections 快速上手 and 后端支持现状): PQ2_0's tables, with 4 lanes per scale group (split
// mode only; batch-1 calls take the integer GEMV by default, this kernel on request).
//
// Operation: y[n] = sum_g s[n][g] * sum_j t[n][128g+j] * x'[128g+j], x' = blockdiag(Hn) x.
// Sources: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com): method paragraph
// (trits, FP16 scale per 128 weights, block Hadamard), paragraph on running the files
// (activation-side Hadamard), paragraph on the two packings (PTQ1_0, PQ2_0 and their
// decode cost); "Bonsai 2，把27B压进6个G" (10100.com), section 它怎么做到的.
//
// Design (B200, HBM-bound: PQ2_0 moves 34 B and PTQ1_0 28 B per 128 weights):
//
// * Activation lookup tables.  The decode arithmetic, not the bytes, is the limit at
//   batch 1: at ~6.5 TB/s an SM must consume ~90 weights per clock.  So every weight
//   byte is used as an index into a table of signed partial sums of the activations
//   it covers: PQ2_0 byte (4 two-bit codes) -> sum_i (c_i - 1) x'_i over 4
//   activations; PTQ1_0 byte (base-3 number, 5 digits) -> sum_i (d_i - 1) x'_i over 5
//   (3 in the last byte of a group).  One byte costs a byte permute (which forms the
//   absolute shared-memory address) and one shared load, plus the FP32 adds.
// * K is cut into 512-wide slices (4 scale groups); one slice's tables are 128 tables
//   x 256 FP32 entries = 128 KB of shared memory.
// * Bank-conflict-free lookups: lane l of every warp reads only tables stored in bank
//   l, so the 32 random lookups of one instruction hit 32 different banks.  Lane l
//   owns bytes 4l..4l+3 of a 128-byte PQ2_0 row slice (one 32-bit load per lane); for
//   PTQ1_0 the 8 lanes of a scale group load 7 aligned words covering the group's 26
//   bytes (the 2 bytes of a neighbouring group and the 8th lane map to all-zero
//   "phantom" tables), so each group is again exactly 8 lanes.
// * A warp task is 16 rows of one slice, loaded in natural order (each 32-bit load
//   instruction reads one row's contiguous slice segment), with further tasks' words
//   and scales in flight.  A transpose-reduction over the 8 lanes of a scale group is
//   followed by the scale multiply and two more shuffle stages.
// * Two schedules:
//   - rows mode (on request): a CTA owns a range of rows, rotates all of x once, and
//     walks the K slices, rebuilding the tables per slice and keeping each row's sum
//     in registers.  No split-K, but ten table builds per CTA for K = 5120.
//   - split mode (the default): a CTA owns one slice and a range of rows and writes FP32
//     partials; a small second kernel (launched behind it with programmatic dependent
//     launch) sums each row's partials in slice order (deterministic) and writes y.
//     In this mode x is loaded before the weight prefetch, so that its few loads are
//     not queued behind the CTA's weight traffic.
// * Programmatic dependent launch: a kernel lets the next kernel on the stream start
//   at once; the next kernel prefetches its own weights and then waits for this one to
//   finish before it reads x, the workspace or y.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSliceK = 512;         // activations per K slice
constexpr int kRows = 16;            // rows per warp task
constexpr int kTableRegion = 65536;  // 256 entries x 256 bytes
// Shared-memory layout.  The tables live at shared-window addresses [0x10000, 0x30000)
// so that a byte permute alone forms a lookup's absolute address (byte 2 = 1 + region,
// byte 1 = the weight byte, byte 0 = lane slot).  The dynamic allocation starts at a
// small window address b (after the per-block reserved area) and spans 0x30000 bytes,
// which covers the table range for any b <= 0x10000 - kMiscBytes; x' (FP32) lives at
// its start: one slice in split mode, all of K in rows mode.
constexpr uint32_t kTableAddr = 0x10000u;
constexpr int kMiscBytes = 0x10000 - 2048;  // room for x' below the tables
constexpr int kSmemBytes = 0x30000;
constexpr int kRowsModeMaxK = 12288;        // x' of all K must fit below the tables
constexpr int kMaxTasksPerWarp = 32;        // split mode: row blocks per warp (host-checked)


template <int kFmt>
struct Fmt;

template <>
struct Fmt<2> {  // PQ2_0
    static constexpr int kSliceK = 512;       // activations per K slice
    static constexpr int kLanesPerGroup = 8;  // lanes whose words cover one scale group
    static constexpr int kScaleGroup = 128;   // weights per FP16 scale
    static constexpr int kSliceBytes = 128;
    __device__ static int64_t row_bytes(int64_t K) { return K / 4; }
    // byte offset of the lane's word inside a row's slice segment
    __device__ static int lane_offset(int lane) { return 4 * lane; }
};

template <>
struct Fmt<1> {  // PTQ1_0
    static constexpr int kSliceK = 512;
    static constexpr int kLanesPerGroup = 8;
    static constexpr int kScaleGroup = 128;
    static constexpr int kSliceBytes = 4 * kPtq1GroupBytes;  // 104
    __device__ static int64_t row_bytes(int64_t K) { return (K / kGroup) * kPtq1GroupBytes; }
    // the 8th lane of a group reads a valid word too; its tables are all zero
    __device__ static int lane_offset(int lane) {
        const int g = lane >> 3, k = lane & 7;
        return kPtq1GroupBytes * g - 2 * (g & 1) + 4 * (k == 7 ? 0 : k);  // 4-byte aligned
    }
};

template <>
struct Fmt<3> {  // Q1_0: a byte holds 8 signs, so a 128-byte row slice covers 1024 activations
    static constexpr int kSliceK = 1024;
    static constexpr int kLanesPerGroup = 4;
    static constexpr int kScaleGroup = 128;
    static constexpr int kSliceBytes = 128;
    __device__ static int64_t row_bytes(int64_t K) { return K / 8; }
    __device__ static int lane_offset(int lane) { return 4 * lane; }
};

template <>
struct Fmt<4> {  // PQ2_0 with one scale per 64 weights: PQ2_0's tables, 4 lanes per scale group
    static constexpr int kSliceK = 512;
    static constexpr int kLanesPerGroup = 4;
    static constexpr int kScaleGroup = 64;
    static constexpr int kSliceBytes = 128;
    __device__ static int64_t row_bytes(int64_t K) { return K / 4; }
    __device__ static int lane_offset(int lane) { return 4 * lane; }
};

// PTQ1_0: position (inside its group) of byte slot j of lane, or -1 for a slot that
// belongs to a neighbouring group / an idle lane (a phantom slot).
__device__ __forceinline__ int ptq1_slot_pos(int lane, int j) {
    const int g = lane >> 3, k = lane & 7;
    if (k == 7) return -1;
    const int p = 4 * k - 2 * (g & 1) + j;
    return (p >= 0 && p < kPtq1GroupBytes) ? p : -1;
}

// Offset of entry e of table (lane, slot j) from the table base:
// region (j >> 1), entry row e (256 bytes), half (j & 1), bank lane.
__device__ __forceinline__ uint32_t table_offset(int lane, int j, int e) {
    return (uint32_t)((j >> 1) * kTableRegion + e * 256 + (j & 1) * 128 + lane * 4);
}

__device__ __forceinline__ float signed_term(int digit, float xv) {
    return digit == 0 ? -xv : (digit == 1 ? 0.f : xv);
}

// Q1_0: table (lane, j) belongs to byte 4 lane + j of the row slice, i.e. activations
// 8(4 lane + j) .. +7; entry e = sum_i (bit i of e ? +x'_i : -x'_i), as a sum of two
// halves L[e & 15] + H[e >> 4].  Thread t serves table (lane = t & 31, j = (t >> 5) & 3)
// and its 64 entries e >> 6 == t >> 7.
__device__ __forceinline__ void build_tables_q1(const float *xr, uint8_t *tables, int t) {
    const int lane = t & 31, j = (t >> 5) & 3, q = t >> 7;
    const float *xa = xr + 8 * (4 * lane + j);
    const float4 a = *reinterpret_cast<const float4 *>(xa), b = *reinterpret_cast<const float4 *>(xa + 4);
    const float lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {b.x, b.y, b.z, b.w};
    float L[16];
#pragma unroll
    for (int e = 0; e < 16; e++) {
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++) v += ((e >> i) & 1) ? lo[i] : -lo[i];
        L[e] = v;
    }
#pragma unroll
    for (int hh = 0; hh < 4; hh++) {
        const int h = 4 * q + hh;  // high nibble
        float H = 0.f;
#pragma unroll
        for (int i = 0; i < 4; i++) H += ((h >> i) & 1) ? hi[i] : -hi[i];
#pragma unroll
        for (int l = 0; l < 16; l++)
            *reinterpret_cast<float *>(tables + table_offset(lane, j, 16 * h + l)) = L[l] + H;
    }
}

// Builds one slice's tables from its x' (FP32 in shared memory).  Thread t serves table
// (lane = t & 31, slot j = (t >> 5) & 3) and, of that table's 3^(n-2) settings of its
// high digits, those congruent to t >> 7 (mod 4); each setting is 9 entries.
template <int kFmt>
__device__ __forceinline__ void build_tables(const float *xr, uint8_t *tables, int t) {
    if (kFmt == 3) {
        build_tables_q1(xr, tables, t);
        return;
    }
    const int lane = t & 31, j = (t >> 5) & 3, q = t >> 7;
    const float *xa;
    int n, place;  // trits in the chunk, place value of one digit (4: 2-bit slots, 3: base 3)
    if (kFmt == 2 || kFmt == 4) {
        xa = xr + 4 * (4 * lane + j);  // chunk 4*lane + j covers activations 4c .. 4c+3
        n = 4;
        place = 4;
    } else {
        const int p = ptq1_slot_pos(lane, j);
        if (p < 0) return;  // phantom slot: its table stays zero
        xa = xr + kGroup * (lane >> 3) + 5 * p;
        n = p == kPtq1GroupBytes - 1 ? 3 : 5;
        place = 3;
    }
    int combos = 1;
    for (int i = 2; i < n; i++) combos *= 3;
    float xs[5];
    if (kFmt == 2 || kFmt == 4) {
        const float4 q4 = *reinterpret_cast<const float4 *>(xa);
        xs[0] = q4.x, xs[1] = q4.y, xs[2] = q4.z, xs[3] = q4.w, xs[4] = 0.f;
    } else {
#pragma unroll
        for (int i = 0; i < 5; i++) xs[i] = i < n ? xa[i] : 0.f;
    }
    const float x0 = xs[0], x1 = xs[1];
    for (int c = q; c < combos; c += kThreads / 128) {
        float base = 0.f;
        int e = 0, rest = c, pw = place * place;
#pragma unroll
        for (int i = 2; i < 5; i++) {
            if (i < n) {
                const int d = rest % 3;
                rest /= 3;
                base += signed_term(d, xs[i]);
                e += d * pw;
                pw *= place;
            }
        }
#pragma unroll
        for (int d1 = 0; d1 < 3; d1++) {
            const float b1 = base + signed_term(d1, x1);
#pragma unroll
            for (int d0 = 0; d0 < 3; d0++)
                *reinterpret_cast<float *>(tables + table_offset(lane, j, e + d1 * place + d0)) =
                    b1 + signed_term(d0, x0);
        }
    }
}

// PTQ1_0 phantom tables (idle 8th lane of each group, slots that belong to a
// neighbouring group) must read as zero for any byte.  Each lane clears its own
// phantom tables, so every store instruction hits 32 different banks.  PQ2_0 needs
// nothing: a valid byte never reaches an unwritten entry.
template <int kFmt>
__device__ __forceinline__ void zero_phantom_tables(uint8_t *tables, int lane, int warp) {
    if constexpr (kFmt == 1) {
        for (int e = warp; e < 256; e += kWarps)
#pragma unroll
            for (int j = 0; j < 4; j++)
                if (ptq1_slot_pos(lane, j) < 0) *reinterpret_cast<float *>(tables + table_offset(lane, j, e)) = 0.f;
    }
}

// Loads one warp task: register i <- the lane's word of row n0 + i (each load
// instruction reads one row's contiguous slice segment), and the two FP16 scales the
// lane applies after the group reduction: rows (lane & 7) + 8m of group lane >> 3.
// Nothing here consumes the loaded values, so the loads stay in flight until the
// task is processed (the scales are converted only there).
// kNS = kRows / kLanesPerGroup scales per lane: rows (lane % lpg) + lpg m of group
// lane / lpg (lpg = lanes per scale group: 8, or 4 for Q1_0).
template <int kFmt, int kNS = kRows / Fmt<kFmt>::kLanesPerGroup>
__device__ __forceinline__ void load_task(uint32_t (&w)[kRows], uint16_t (&sc)[kNS], const uint8_t *slice_base,
                                          const uint16_t *scales, int64_t n0, int64_t N, int64_t G,
                                          int64_t gcol, uint32_t row_bytes, int lane_off, int lane) {
    constexpr int lpg = Fmt<kFmt>::kLanesPerGroup;
    const uint8_t *p = slice_base + n0 * row_bytes + lane_off;
    const uint16_t *sp = scales + (n0 + (lane % lpg)) * G + gcol;
    if (N - n0 >= kRows) {  // full task: no predicates
#pragma unroll
        for (int i = 0; i < kRows; i++)
            w[i] = __ldcs(reinterpret_cast<const unsigned int *>(p + (size_t)i * row_bytes));
#pragma unroll
        for (int m = 0; m < kNS; m++) sc[m] = __ldg(sp + (int64_t)lpg * m * G);
        return;
    }
    const int nvalid = (int)(N - n0);
#pragma unroll
    for (int i = 0; i < kRows; i++)
        w[i] = i < nvalid ? __ldcs(reinterpret_cast<const unsigned int *>(p + (size_t)i * row_bytes)) : 0u;
#pragma unroll
    for (int m = 0; m < kNS; m++) sc[m] = (lane % lpg) + lpg * m < nvalid ? __ldg(sp + (int64_t)lpg * m * G) : (uint16_t)0;
}

__device__ __forceinline__ float lds_abs(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// One stage of the transpose-reduction over lane bit b: of each register pair
// (2m, 2m+1) -- the same rows except row bit b -- the lane keeps the one whose row
// bit b equals its lane bit b and adds the partner lane's copy of that row.
template <int kHalf>
__device__ __forceinline__ void transpose_stage(float (&v)[kRows], int lane, int b) {
    const bool hi = (lane >> b) & 1;
#pragma unroll
    for (int m = 0; m < kHalf; m++) {
        const float keep = hi ? v[2 * m + 1] : v[2 * m];
        const float send = hi ? v[2 * m] : v[2 * m + 1];
        v[m] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << b);
    }
}

// Lookups of one task and the reduction over the 8 lanes of each scale group:
// returns, scaled, rows (lane & 7) + 8m (m = 0, 1) of this lane's group.
__device__ __forceinline__ float2 task_group_sums(const uint32_t (&w)[kRows], const uint16_t (&sc)[2],
                                                  const uint32_t (&pbase)[4], int lane) {
    float v[kRows];
#pragma unroll
    for (int i = 0; i < kRows; i++) {
        const float t0 = lds_abs(__byte_perm(w[i], pbase[0], 0x7604));
        const float t1 = lds_abs(__byte_perm(w[i], pbase[1], 0x7614));
        const float t2 = lds_abs(__byte_perm(w[i], pbase[2], 0x7624));
        const float t3 = lds_abs(__byte_perm(w[i], pbase[3], 0x7634));
        const float2 u = __fadd2_rn(make_float2(t0, t1), make_float2(t2, t3));
        v[i] = u.x + u.y;
    }
    transpose_stage<8>(v, lane, 0);
    transpose_stage<4>(v, lane, 1);
    transpose_stage<2>(v, lane, 2);
    return make_float2(v[0] * half_bits_to_float(sc[0]), v[1] * half_bits_to_float(sc[1]));
}

// Q1_0 and PQ2_0 g64 (4 lanes per scale group): lookups of one task, the reduction over
// the 4 lanes of each of the slice's 8 scale groups, the scales, then the sum over the
// groups.  Lanes L and L + 16 end with row L & 15 of the task.
__device__ __forceinline__ float task_total_4lane(const uint32_t (&w)[kRows], const uint16_t (&sc)[4],
                                               const uint32_t (&pbase)[4], int lane) {
    float v[kRows];
#pragma unroll
    for (int i = 0; i < kRows; i++) {
        const float t0 = lds_abs(__byte_perm(w[i], pbase[0], 0x7604));
        const float t1 = lds_abs(__byte_perm(w[i], pbase[1], 0x7614));
        const float t2 = lds_abs(__byte_perm(w[i], pbase[2], 0x7624));
        const float t3 = lds_abs(__byte_perm(w[i], pbase[3], 0x7634));
        const float2 u = __fadd2_rn(make_float2(t0, t1), make_float2(t2, t3));
        v[i] = u.x + u.y;
    }
    transpose_stage<8>(v, lane, 0);
    transpose_stage<4>(v, lane, 1);  // v[m]: row (lane & 3) + 4m of group lane >> 2
#pragma unroll
    for (int m = 0; m < 4; m++) v[m] *= half_bits_to_float(sc[m]);
    transpose_stage<2>(v, lane, 2);
    transpose_stage<1>(v, lane, 3);  // v[0]: row lane & 15, summed over lane bits 2, 3
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// Sum of the four groups: lanes L and L + 16 end with row L & 15 of the task.
__device__ __forceinline__ float groups_total(float2 g, int lane) {
    const bool hi = (lane >> 3) & 1;
    const float keep = hi ? g.y : g.x;
    const float send = hi ? g.x : g.y;
    const float r = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    return r + __shfl_xor_sync(0xffffffffu, r, 16);
}

__device__ __forceinline__ void make_pbase(uint32_t (&pbase)[4], int lane) {
    // byte 0 = (j & 1) * 128 + 4 * lane, byte 2 = 1 + region (absolute address 0x10000 + ...)
#pragma unroll
    for (int j = 0; j < 4; j++)
        pbase[j] = (kTableAddr + ((uint32_t)(j >> 1) << 16)) | ((uint32_t)(j & 1) << 7) | ((uint32_t)lane << 2);
}

// ---------------------------------------------------------------- split mode

template <int kFmt>
__global__ void __launch_bounds__(kThreads, 1) gemv_split_kernel(
    const uint16_t *__restrict__ x, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, float *__restrict__ partials, int64_t N,
    int64_t K, int parts) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *xr = reinterpret_cast<float *>(smem);
    const uint32_t smem_addr = (uint32_t)__cvta_generic_to_shared(smem);
    if (smem_addr + kMiscBytes > kTableAddr) return;  // layout assumption violated (host checks it)
    uint8_t *tables = smem + (kTableAddr - smem_addr);
    pdl_launch_dependents();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t G = K / Fmt<kFmt>::kScaleGroup;  // scales per row
    constexpr int kSK = Fmt<kFmt>::kSliceK, kLPG = Fmt<kFmt>::kLanesPerGroup, kNS = kRows / kLPG;
    const int S = (int)(K / kSK);
    const int64_t RB = (N + kRows - 1) / kRows;
    // CTA = (slice, part): the row blocks of one part of the rows, for one K slice
    const int slice = blockIdx.x / parts, part = blockIdx.x - slice * parts;
    const int64_t rb_begin = RB * part / parts, rb_end = RB * (part + 1) / parts;
    const uint32_t row_bytes = (uint32_t)Fmt<kFmt>::row_bytes(K);
    const int lane_off = Fmt<kFmt>::lane_offset(lane);
    const uint8_t *slice_base = packed + (int64_t)slice * Fmt<kFmt>::kSliceBytes;
    const int64_t gcol = (int64_t)slice * (kSK / Fmt<kFmt>::kScaleGroup) + lane / kLPG;

    zero_phantom_tables<kFmt>(tables, lane, warp);
    pdl_wait();  // x, the workspace and y may belong to the previous kernel
    // x first, so that its loads are not queued behind this CTA's weight loads
    float xv[4];
    if (warp < kSK / kGroup) load_half4(x + (int64_t)slice * kSK + warp * kGroup + 4 * lane, xv);
    int64_t rb = rb_begin + warp;
    uint32_t wa[kRows], wb[kRows], wc[kRows];
    uint16_t sa[kNS], sb[kNS], sc2[kNS];
    if (rb < rb_end) load_task<kFmt>(wa, sa, slice_base, scales, rb * kRows, N, G, gcol, row_bytes, lane_off, lane);
    if (rb + kWarps < rb_end)
        load_task<kFmt>(wb, sb, slice_base, scales, (rb + kWarps) * kRows, N, G, gcol, row_bytes, lane_off, lane);
    if (warp < kSK / kGroup) {  // rotate the slice of x: 4 (Q1_0: 8) blocks of 128
        fwht128_warp(xv, lane);
        *reinterpret_cast<float4 *>(xr + warp * kGroup + 4 * lane) = make_float4(xv[0], xv[1], xv[2], xv[3]);
    }
    __syncthreads();
    build_tables<kFmt>(xr, tables, tid);
    __syncthreads();
    uint32_t pbase[4];
    make_pbase(pbase, lane);

    // one slice's sums go straight to y (S == 1) or to the FP32 partials, which
    // gemv_reduce_kernel adds up in slice order
    auto task_total = [&](const uint32_t(&w)[kRows], const uint16_t(&sc)[kNS]) -> float {
        if constexpr (kLPG == 4)
            return task_total_4lane(w, sc, pbase, lane);
        else
            return groups_total(task_group_sums(w, sc, pbase, lane), lane);
    };
    auto finish = [&](float total, int64_t task_rb) {
        const int64_t n0 = task_rb * kRows;
        const int row = lane & 15;
        if (lane < 16 && n0 + row < N) {
            if (S == 1)
                y[n0 + row] = float_to_half_bits(total);
            else
                partials[(int64_t)slice * N + n0 + row] = total;
        }
    };
    // three rotating task buffers: while one task is reduced, the next two are in flight
    while (rb < rb_end) {
        if (rb + 2 * kWarps < rb_end)
            load_task<kFmt>(wc, sc2, slice_base, scales, (rb + 2 * kWarps) * kRows, N, G, gcol, row_bytes, lane_off, lane);
        finish(task_total(wa, sa), rb);
        rb += kWarps;
        if (rb >= rb_end) break;
        if (rb + 2 * kWarps < rb_end)
            load_task<kFmt>(wa, sa, slice_base, scales, (rb + 2 * kWarps) * kRows, N, G, gcol, row_bytes, lane_off, lane);
        finish(task_total(wb, sb), rb);
        rb += kWarps;
        if (rb >= rb_end) break;
        if (rb + 2 * kWarps < rb_end)
            load_task<kFmt>(wb, sb, slice_base, scales, (rb + 2 * kWarps) * kRows, N, G, gcol, row_bytes, lane_off, lane);
        finish(task_total(wc, sc2), rb);
        rb += kWarps;
    }
}

// y[n] = sum over slices s (in order) of partials[s][n]; launched right after the split
// kernel, it waits for that kernel to finish before reading.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float *__restrict__ partials,
                                                          uint16_t *__restrict__ y, int64_t N, int S) {
    pdl_launch_dependents();
    pdl_wait();
    for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < N; n += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        int s = 0;
        for (; s + 8 <= S; s += 8) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; u++) t[u] = __ldcg(partials + (int64_t)(s + u) * N + n);
#pragma unroll
            for (int u = 0; u < 8; u++) acc += t[u];
        }
        for (; s < S; s++) acc += __ldcg(partials + (int64_t)s * N + n);
        y[n] = float_to_half_bits(acc);
    }
}

// ---------------------------------------------------------------- rows mode

// A CTA owns row blocks [rb_begin, rb_end); in rounds of kWarps blocks (one per warp)
// it walks all K slices.  Each warp keeps the scaled group sums of its block in two
// registers across slices and reduces over the groups once at the end.
template <int kFmt>
__global__ void __launch_bounds__(kThreads, 1) gemv_rows_kernel(
    const uint16_t *__restrict__ x, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, int64_t N, int64_t K) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *xr = reinterpret_cast<float *>(smem);  // x' of all K (K <= kRowsModeMaxK)
    const uint32_t smem_addr = (uint32_t)__cvta_generic_to_shared(smem);
    if (smem_addr + kMiscBytes > kTableAddr) return;  // layout assumption violated (host checks it)
    uint8_t *tables = smem + (kTableAddr - smem_addr);
    pdl_launch_dependents();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t G = K / kGroup;
    const int S = (int)(K / kSliceK);
    const int64_t RB = (N + kRows - 1) / kRows;
    const int64_t rb_begin = RB * blockIdx.x / gridDim.x, rb_end = RB * (blockIdx.x + 1) / gridDim.x;
    const uint32_t row_bytes = (uint32_t)Fmt<kFmt>::row_bytes(K);
    const int lane_off = Fmt<kFmt>::lane_offset(lane);
    uint32_t pbase[4];
    make_pbase(pbase, lane);

    bool first = true;
    for (int64_t round = rb_begin; round < rb_end; round += kWarps) {
        const int64_t rb = round + warp;
        const bool active = rb < rb_end;
        // four slice buffers: slice s uses buffer s % 4, slices s+1 .. s+3 are in flight
        uint32_t wq[4][kRows];
        uint16_t sq[4][2];
        auto fetch = [&](int sl, uint32_t (&wt)[kRows], uint16_t (&st)[2]) {
            if (active && sl < S)
                load_task<kFmt>(wt, st, packed + (int64_t)sl * Fmt<kFmt>::kSliceBytes, scales, rb * kRows, N, G,
                                (int64_t)sl * (kSliceK / kGroup) + (lane >> 3), row_bytes, lane_off, lane);
        };
        fetch(0, wq[0], sq[0]);
        fetch(1, wq[1], sq[1]);
        fetch(2, wq[2], sq[2]);
        if (first) {
            zero_phantom_tables<kFmt>(tables, lane, warp);
            pdl_wait();  // x and y may belong to the previous kernel
            for (int64_t b = warp; b < G; b += kWarps) {  // rotate all of x once
                float xv[4];
                load_half4(x + b * kGroup + 4 * lane, xv);
                fwht128_warp(xv, lane);
                *reinterpret_cast<float4 *>(xr + b * kGroup + 4 * lane) = make_float4(xv[0], xv[1], xv[2], xv[3]);
            }
            first = false;
        }
        float2 acc = make_float2(0.f, 0.f);
        for (int s = 0; s < S; s += 4) {
#pragma unroll
            for (int h = 0; h < 4; h++) {
                if (s + h < S) {
                    fetch(s + h + 3, wq[(h + 3) & 3], sq[(h + 3) & 3]);
                    __syncthreads();  // the previous slice's lookups are done (and x' is written)
                    build_tables<kFmt>(xr + (int64_t)(s + h) * kSliceK, tables, tid);
                    __syncthreads();
                    if (active) {
                        const float2 gs = task_group_sums(wq[h], sq[h], pbase, lane);
                        acc.x += gs.x;
                        acc.y += gs.y;
                    }
                }
            }
        }
        const float total = groups_total(acc, lane);
        const int64_t n0 = rb * kRows;
        const int row = lane & 15;
        if (active && lane < 16 && n0 + row < N) y[n0 + row] = float_to_half_bits(total);
    }
}

// ---------------------------------------------------------------- host side

// Rows mode (no split-K) is kept for measurement: with the split-K partials summed by a
// second kernel, split mode is as fast or faster at every measured decode shape, so it
// is the default.
bool use_rows_mode(int64_t N, int64_t K, int fmt, const DeviceInfo &dev) {
    (void)N;
    (void)K;
    (void)fmt;
    (void)dev;
    return false;
}

// Split mode: rows of the weight matrix are split into `parts` ranges per K slice so that
// the grid (slices x parts) fills the SMs once.
int slice_k(int fmt) { return fmt == 3 ? Fmt<3>::kSliceK : kSliceK; }  // (PQ2_0 g64: 512)

int gemv_parts(int64_t N, int64_t K, int fmt, const DeviceInfo &dev) {
    const int64_t S = K / slice_k(fmt);
    const int64_t RB = (N + kRows - 1) / kRows;
    int64_t parts = dev.sm_count / S;
    if (parts < 1) parts = 1;
    // every warp of a CTA handles at most kMaxTasksPerWarp row blocks
    const int64_t min_parts = (RB + (int64_t)kWarps * kMaxTasksPerWarp - 1) / ((int64_t)kWarps * kMaxTasksPerWarp);
    if (parts < min_parts) parts = min_parts;
    if (parts > RB) parts = RB;
    return (int)parts;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cfg(void (*kernel)(KArgs...), int grid, int threads, int smem, cudaStream_t s,
                           Args... args) {
    if (smem > 0) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, cudaStream_t s, Args... args) {
    return launch_pdl_cfg(kernel, grid, kThreads, kSmemBytes, s, args...);
}

// Split mode: the slice kernel, then (K > 512) the in-order reduction of its partials.
cudaError_t launch_split(const uint16_t *x, const uint8_t *packed, const uint16_t *scales, uint16_t *y,
                         float *partials, int64_t N, int64_t K, int fmt, cudaStream_t s, const DeviceInfo &dev) {
    const int parts = gemv_parts(N, K, fmt, dev);
    const int64_t S = K / slice_k(fmt);
    const int64_t grid = S * parts;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    cudaError_t e = fmt == 1   ? launch_pdl(gemv_split_kernel<1>, (int)grid, s, x, packed, scales, y, partials, N, K, parts)
                    : fmt == 3 ? launch_pdl(gemv_split_kernel<3>, (int)grid, s, x, packed, scales, y, partials, N, K, parts)
                    : fmt == 4 ? launch_pdl(gemv_split_kernel<4>, (int)grid, s, x, packed, scales, y, partials, N, K, parts)
                               : launch_pdl(gemv_split_kernel<2>, (int)grid, s, x, packed, scales, y, partials, N, K, parts);
    if (e != cudaSuccess || S == 1) return e;
    const int64_t rgrid64 = (N + 255) / 256;
    const int rgrid = (int)(rgrid64 < 4 * (int64_t)dev.sm_count ? rgrid64 : 4 * (int64_t)dev.sm_count);
    return launch_pdl_cfg(gemv_reduce_kernel, rgrid, 256, 0, s, (const float *)partials, y, N, (int)S);
}

}  // namespace

bool gemv_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    if (M != 1 || fmt < 1 || fmt > 4 || K % slice_k(fmt) != 0) return false;
    if ((N + kRows - 1) / kRows > kMaxTiles) return false;
    return true;
}

// Schedule: split_k 0 = automatic, 1 = rows mode (when the shape allows it), >= 2 = split mode.
bool pick_rows_mode(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    if (fmt == 3 || fmt == 4) return false;  // Q1_0, PQ2_0 g64: split mode only
    if (split_k == 1) return K <= kRowsModeMaxK && K / kSliceK >= 2;
    if (split_k >= 2) return false;
    return use_rows_mode(N, K, fmt, dev);
}

int gemv_launches(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    if (pick_rows_mode(N, K, fmt, split_k, dev) || K / slice_k(fmt) <= 1) return 1;
    return 2;
}

size_t gemv_workspace_bytes(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    const int64_t S = K / slice_k(fmt);
    if (S <= 1 || pick_rows_mode(N, K, fmt, split_k, dev)) return 0;
    return (size_t)S * (size_t)N * sizeof(float);
}

cudaError_t launch_gemv(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t N, int64_t K, int fmt, int split_k,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    // the dynamic allocation must start below kTableAddr - kMiscBytes in the shared
    // window; it starts right after the per-block reserved area (no static shared memory)
    if (dev.smem_reserved + kMiscBytes > (int)kTableAddr) return cudaErrorNotSupported;
    if (pick_rows_mode(N, K, fmt, split_k, dev)) {
        const int64_t RB = (N + kRows - 1) / kRows;
        const int grid = (int)(RB < dev.sm_count ? RB : dev.sm_count);
        if (fmt == 1) return launch_pdl(gemv_rows_kernel<1>, grid, s, x, packed, scales, y, N, K);
        return launch_pdl(gemv_rows_kernel<2>, grid, s, x, packed, scales, y, N, K);
    }
    return launch_split(x, packed, scales, y, reinterpret_cast<float *>(ws.data), N, K, fmt, s, dev);
}

// Split-mode launch with caller-provided scratch for the FP32 partials, whatever the shape;
// used by the no-allocation entry point.  partial_floats is the space the scratch holds;
// returns cudaErrorInvalidValue if the shape needs more.
size_t gemv_split_partial_floats(int64_t N, int64_t K) {
    const int64_t S = K / kSliceK;  // PTQ1_0 / PQ2_0 (the no-allocation entry point's formats)
    return S > 1 ? (size_t)S * (size_t)N : 0;
}

cudaError_t launch_gemv_split_scratch(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                      uint16_t *y, int64_t N, int64_t K, int fmt, float *partials,
                                      size_t partial_floats, cudaStream_t s, const DeviceInfo &dev) {
    if (gemv_split_partial_floats(N, K) > partial_floats) return cudaErrorInvalidValue;
    if (dev.smem_reserved + kMiscBytes > (int)kTableAddr) return cudaErrorNotSupported;
    return launch_split(x, packed, scales, y, partials, N, K, fmt, s, dev);
}

}  // namespace bonsai
