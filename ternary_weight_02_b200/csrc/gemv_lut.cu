// gemv_lut.cu -- batch-1 (M == 1) ternary GEMV for both packings, with the block
// Hadamard rotation of x fused in.
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
//   shared-memory offset), one shared load and half a paired FP32 add.
// * K is cut into 512-wide slices (4 scale groups).  A CTA rotates its slice of x with
//   the warp FWHT (FP32, in registers), builds the slice's tables (128 tables x 256
//   FP32 entries = 128 KB), then its 16 warps stream rows of the slice.
// * Bank-conflict-free lookups: lane l of every warp reads only tables stored in bank
//   l, so the 32 random lookups of one instruction hit 32 different banks.  Lane l
//   owns bytes 4l..4l+3 of a 128-byte PQ2_0 row slice (one 32-bit load per lane); for
//   PTQ1_0 the 8 lanes of a scale group load 7 aligned words covering the group's 26
//   bytes (the 2 bytes of a neighbouring group and the 8th lane map to all-zero
//   tables), so each group is again exactly 8 lanes.
// * Reduction: a warp handles 32 rows; lane L keeps row (i XOR L) in register i, which
//   makes the 32-row transpose-reduction select-free (31 shuffles per lane).  Scales
//   are applied after the 8 lanes of a group are summed (4 multiplies per lane).
// * Split-K: each (slice, 32-row block) task writes an FP32 partial; the warp that
//   finishes a row block last (arrival counter in the workspace) sums the partials in
//   slice order (deterministic), writes FP16 y and resets the counter.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSliceK = 512;     // activations per K slice
constexpr int kRows = 32;        // rows per warp task
constexpr int kTableRegion = 65536;  // 256 entries x 256 bytes (64 banks-words per entry)
constexpr int kTableBytes = 2 * kTableRegion;
constexpr int kMiscBytes = 4096;     // x' of the slice (2 KB) + padding
constexpr int kSmemBytes = kMiscBytes + kTableBytes;

template <int kFmt>
struct Fmt;

template <>
struct Fmt<2> {  // PQ2_0
    static constexpr int kSliceBytes = 128;
    __device__ static int64_t row_bytes(int64_t K) { return K / 4; }
    // byte offset of lane's word inside the slice-row, or -1 if the lane loads nothing
    __device__ static int lane_offset(int lane) { return 4 * lane; }
};

template <>
struct Fmt<1> {  // PTQ1_0
    static constexpr int kSliceBytes = 4 * kPtq1GroupBytes;  // 104
    __device__ static int64_t row_bytes(int64_t K) { return (K / kGroup) * kPtq1GroupBytes; }
    __device__ static int lane_offset(int lane) {
        const int g = lane >> 3, k = lane & 7;
        if (k == 7) return -1;
        return kPtq1GroupBytes * g - 2 * (g & 1) + 4 * k;  // 4-byte aligned
    }
};

// PTQ1_0: position (inside its group) of byte slot j of lane, or -1 for a slot that
// belongs to a neighbouring group / an idle lane.
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

// Builds the slice's tables from x' (FP32 in shared memory).  Thread t: lane (bank)
// t & 31, slot j = (t >> 5) & 3, top digit q = t >> 7 (threads with q == 3 idle).
template <int kFmt>
__device__ __forceinline__ void build_tables(const float *xr, uint8_t *tables, int t) {
    const int lane = t & 31, j = (t >> 5) & 3, q = t >> 7;
    if (q > 2) return;
    if (kFmt == 2) {
        const int c = 4 * lane + j;  // chunk: activations 4c .. 4c+3 of the slice
        const float x0 = xr[4 * c], x1 = xr[4 * c + 1], x2 = xr[4 * c + 2], x3 = xr[4 * c + 3];
        const float base3 = q == 0 ? -x3 : (q == 1 ? 0.f : x3);
#pragma unroll
        for (int c2 = 0; c2 < 3; c2++) {
            const float b2 = base3 + (c2 == 0 ? -x2 : (c2 == 1 ? 0.f : x2));
#pragma unroll
            for (int c1 = 0; c1 < 3; c1++) {
                const float b1 = b2 + (c1 == 0 ? -x1 : (c1 == 1 ? 0.f : x1));
#pragma unroll
                for (int c0 = 0; c0 < 3; c0++) {
                    const float v = b1 + (c0 == 0 ? -x0 : (c0 == 1 ? 0.f : x0));
                    const int e = c0 | (c1 << 2) | (c2 << 4) | (q << 6);
                    *reinterpret_cast<float *>(tables + table_offset(lane, j, e)) = v;
                }
            }
        }
    } else {
        const int p = ptq1_slot_pos(lane, j);
        if (p < 0) return;
        const int g = lane >> 3;
        const float *xa = xr + kGroup * g + 5 * p;
        if (p == kPtq1GroupBytes - 1) {  // last byte of a group: three trits, digits 3,4 zero
            if (q != 0) return;
            const float x0 = xa[0], x1 = xa[1], x2 = xa[2];
#pragma unroll
            for (int d2 = 0; d2 < 3; d2++) {
                const float b2 = d2 == 0 ? -x2 : (d2 == 1 ? 0.f : x2);
#pragma unroll
                for (int d1 = 0; d1 < 3; d1++) {
                    const float b1 = b2 + (d1 == 0 ? -x1 : (d1 == 1 ? 0.f : x1));
#pragma unroll
                    for (int d0 = 0; d0 < 3; d0++) {
                        const float v = b1 + (d0 == 0 ? -x0 : (d0 == 1 ? 0.f : x0));
                        *reinterpret_cast<float *>(tables + table_offset(lane, j, d0 + 3 * d1 + 9 * d2)) = v;
                    }
                }
            }
            return;
        }
        const float x0 = xa[0], x1 = xa[1], x2 = xa[2], x3 = xa[3], x4 = xa[4];
        const float base4 = q == 0 ? -x4 : (q == 1 ? 0.f : x4);
#pragma unroll
        for (int d3 = 0; d3 < 3; d3++) {
            const float b3 = base4 + (d3 == 0 ? -x3 : (d3 == 1 ? 0.f : x3));
#pragma unroll
            for (int d2 = 0; d2 < 3; d2++) {
                const float b2 = b3 + (d2 == 0 ? -x2 : (d2 == 1 ? 0.f : x2));
#pragma unroll
                for (int d1 = 0; d1 < 3; d1++) {
                    const float b1 = b2 + (d1 == 0 ? -x1 : (d1 == 1 ? 0.f : x1));
#pragma unroll
                    for (int d0 = 0; d0 < 3; d0++) {
                        const float v = b1 + (d0 == 0 ? -x0 : (d0 == 1 ? 0.f : x0));
                        const int e = d0 + 3 * d1 + 9 * d2 + 27 * d3 + 81 * q;
                        *reinterpret_cast<float *>(tables + table_offset(lane, j, e)) = v;
                    }
                }
            }
        }
    }
}

template <int kFmt>
__global__ void __launch_bounds__(kThreads, 1) gemv_lut_kernel(
    const uint16_t *__restrict__ x, const uint8_t *__restrict__ packed,
    const uint16_t *__restrict__ scales, uint16_t *__restrict__ y, float *__restrict__ partials,
    unsigned int *__restrict__ counters, int64_t N, int64_t K) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *xr = reinterpret_cast<float *>(smem);
    uint8_t *tables = smem + kMiscBytes;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t G = K / kGroup;
    const int S = (int)(K / kSliceK);
    const int64_t RB = (N + kRows - 1) / kRows;
    const int64_t T = (int64_t)S * RB;
    const int64_t t_begin = T * blockIdx.x / gridDim.x;
    const int64_t t_end = T * (blockIdx.x + 1) / gridDim.x;
    const int64_t row_bytes = Fmt<kFmt>::row_bytes(K);
    const int lane_off = Fmt<kFmt>::lane_offset(lane);

    // zero every table once: entries that no valid byte can reach, and the tables of
    // PTQ1_0 padding slots, then stay zero for the whole launch
    for (int i = tid; i < kTableBytes / 16; i += kThreads)
        reinterpret_cast<uint4 *>(tables)[i] = make_uint4(0u, 0u, 0u, 0u);

    // per-lane byte-permute operands: byte 0 = (j & 1) * 128 + 4 * lane, byte 2 = region
    uint32_t pbase[4];
#pragma unroll
    for (int j = 0; j < 4; j++) pbase[j] = ((uint32_t)(j >> 1) << 16) | ((uint32_t)(j & 1) << 7) | ((uint32_t)lane << 2);

    for (int64_t seg = t_begin; seg < t_end;) {
        const int slice = (int)(seg / RB);
        const int64_t seg_end = ((int64_t)slice + 1) * RB < t_end ? ((int64_t)slice + 1) * RB : t_end;
        __syncthreads();  // previous slice's lookups are done (and the zeroing above)
        if (warp >= 12) {  // rotate the slice of x: 4 blocks of 128
            const int b = warp - 12;
            float v[4];
            load_half4(x + (int64_t)slice * kSliceK + b * kGroup + 4 * lane, v);
            fwht128_warp(v, lane);
            *reinterpret_cast<float4 *>(xr + b * kGroup + 4 * lane) = make_float4(v[0], v[1], v[2], v[3]);
        }
        __syncthreads();
        build_tables<kFmt>(xr, tables, tid);
        __syncthreads();

        const uint8_t *slice_base = packed + (int64_t)slice * Fmt<kFmt>::kSliceBytes;
        for (int64_t task = seg + warp; task < seg_end; task += kWarps) {
            const int64_t rb = task - (int64_t)slice * RB;
            const int64_t n0 = rb * kRows;
            const int nvalid = (int)(N - n0 < kRows ? N - n0 : kRows);
            const uint8_t *lane_base = slice_base + n0 * row_bytes + lane_off;

            uint32_t w[kRows];
#pragma unroll
            for (int i = 0; i < kRows; i++) {
                const int r = i ^ lane;
                w[i] = 0u;
                if (lane_off >= 0 && r < nvalid)
                    w[i] = __ldcs(reinterpret_cast<const unsigned int *>(lane_base + (int64_t)r * row_bytes));
            }
            float v[kRows];
#pragma unroll
            for (int i = 0; i < kRows; i++) {
                const float t0 = *reinterpret_cast<const float *>(tables + __byte_perm(w[i], pbase[0], 0x7604));
                const float t1 = *reinterpret_cast<const float *>(tables + __byte_perm(w[i], pbase[1], 0x7614));
                const float t2 = *reinterpret_cast<const float *>(tables + __byte_perm(w[i], pbase[2], 0x7624));
                const float t3 = *reinterpret_cast<const float *>(tables + __byte_perm(w[i], pbase[3], 0x7634));
                v[i] = (t0 + t2) + (t1 + t3);
            }
            // sum over the 8 lanes of each scale group (lane bits 0..2 <-> row bits 0..2)
#pragma unroll
            for (int b = 0; b < 3; b++) {
#pragma unroll
                for (int i = 0; i < kRows; i++)
                    if ((i & ((2 << b) - 1)) == 0) v[i] += __shfl_xor_sync(0xffffffffu, v[i | (1 << b)], 1 << b);
            }
            // scale: register i (i in {0, 8, 16, 24}) holds row i ^ lane of group lane >> 3
            const int64_t gcol = (int64_t)slice * (kSliceK / kGroup) + (lane >> 3);
#pragma unroll
            for (int i = 0; i < kRows; i += 8) {
                const int r = i ^ lane;
                const float sc = r < nvalid ? half_bits_to_float(__ldg(scales + (n0 + r) * G + gcol)) : 0.f;
                v[i] *= sc;
            }
            // sum over the 4 groups (lane bits 3, 4 <-> row bits 3, 4)
            v[0] += __shfl_xor_sync(0xffffffffu, v[8], 8);
            v[16] += __shfl_xor_sync(0xffffffffu, v[24], 8);
            v[0] += __shfl_xor_sync(0xffffffffu, v[16], 16);
            // lane L now holds row n0 + L
            const bool mine = lane < nvalid;
            if (S == 1) {
                if (mine) y[n0 + lane] = float_to_half_bits(v[0]);
                continue;
            }
            if (mine) partials[(int64_t)slice * N + n0 + lane] = v[0];
            __threadfence();
            __syncwarp();
            unsigned int arrived = 0;
            if (lane == 0) arrived = atomicAdd(counters + rb, 1u);
            arrived = __shfl_sync(0xffffffffu, arrived, 0);
            if (arrived == (unsigned int)(S - 1)) {
                __threadfence();
                float acc = 0.f;
                if (mine)
                    for (int s = 0; s < S; s++) acc += __ldcg(partials + (int64_t)s * N + n0 + lane);
                if (mine) y[n0 + lane] = float_to_half_bits(acc);
                if (lane == 0) counters[rb] = 0u;
            }
        }
        seg = seg_end;
    }
}

}  // namespace

bool gemv_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    if (M != 1 || K % kSliceK != 0) return false;
    if ((N + kRows - 1) / kRows > kMaxTiles) return false;
    (void)fmt;
    return true;
}

size_t gemv_workspace_bytes(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    (void)fmt;
    (void)split_k;
    (void)dev;
    const int64_t S = K / kSliceK;
    return S > 1 ? (size_t)S * (size_t)N * sizeof(float) : 0;
}

cudaError_t launch_gemv(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t N, int64_t K, int fmt, int split_k,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    (void)split_k;  // the K split is fixed by the 512-wide table slice
    const int64_t tasks = (K / kSliceK) * ((N + kRows - 1) / kRows);
    const int grid = (int)(tasks < dev.sm_count ? tasks : dev.sm_count);
    float *partials = reinterpret_cast<float *>(ws.data);
    cudaError_t err;
    if (fmt == 1) {
        err = cudaFuncSetAttribute(gemv_lut_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (err != cudaSuccess) return err;
        gemv_lut_kernel<1><<<grid, kThreads, kSmemBytes, s>>>(x, packed, scales, y, partials, ws.counters, N, K);
    } else {
        err = cudaFuncSetAttribute(gemv_lut_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (err != cudaSuccess) return err;
        gemv_lut_kernel<2><<<grid, kThreads, kSmemBytes, s>>>(x, packed, scales, y, partials, ws.counters, N, K);
    }
    return cudaGetLastError();
}

}  // namespace bonsai
