// skinny_mma.cu -- ternary linear layer for small batches (1 <= M <= 16 tokens), PQ2_0.
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
//   permutation on both operands) so that its four slots are one byte of the word.
// * Per 128-weight group the MMA starts from zero; the epilogue adds
//   s[n][g] * (2^24 * D - sum_j x'[m][j]) (the second term turns codes into trits).
// * x' (FWHT prepass, FP16) of the CTA's K chunk sits in shared memory as
//   [k-step][token][16 halves], 4^-(k mod 4)-scaled, so a lane's B fragment is one
//   8-byte load from a contiguous 256-byte row.
// * A warp owns 16 weight rows; a CTA 128 rows and one K chunk.  Split-K: chunks
//   write FP32 partials; the warp that brings a row block's last chunk sums them in
//   chunk order (deterministic) and writes y.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerCta = kWarps * 16;
constexpr int kSubGroups = 16;  // groups of x' staged in shared memory at a time

struct Raw {
    uint4 a, b;  // 32 bytes: one 128-weight group of one row
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]), "f"(d[2]), "f"(d[3]));
}

__device__ __forceinline__ uint32_t word_of(const Raw &r, int i) {
    const uint4 &v = i < 4 ? r.a : r.b;
    const int j = i & 3;
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

template <int NT>  // n8 token tiles: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kThreads) skinny_kernel(
    const uint16_t *__restrict__ xr, const uint8_t *__restrict__ packed, const uint16_t *__restrict__ scales,
    uint16_t *__restrict__ y, float *__restrict__ partials, unsigned int *__restrict__ counters, int M, int64_t N,
    int64_t K, int S, int gpc) {
    constexpr int MT = NT * 8;  // tokens padded
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem);  // [kSubGroups * 8 k-steps][MT][16]
    float *gsum = reinterpret_cast<float *>(smem + kSubGroups * 8 * MT * 32);  // [MT][kSubGroups]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int64_t G = K / kGroup;
    const int chunk = blockIdx.y;
    const int g_begin = chunk * gpc;
    const int g_end = (int)((int64_t)(chunk + 1) * gpc < G ? (int64_t)(chunk + 1) * gpc : G);
    const int64_t n0 = (int64_t)blockIdx.x * kRowsPerCta + warp * 16;
    const int64_t r0 = n0 + gid, r1 = n0 + gid + 8;
    const bool v0 = r0 < N, v1 = r1 < N;
    const uint32_t sel = 0x4040u | (uint32_t)tq | ((uint32_t)tq << 8);  // [byte tq, 0, byte tq, 0]

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 4; e++) acc[nt][e] = 0.f;

    auto load_raw = [&](int g, Raw &ra, Raw &rb, float &s0, float &s1) {
        const uint4 z = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);  // trits 0
        if (v0) {
            const uint4 *p = reinterpret_cast<const uint4 *>(packed + (r0 * G + g) * kPq2GroupBytes);
            ra.a = __ldcs(p);
            ra.b = __ldcs(p + 1);
            s0 = half_bits_to_float(__ldg(scales + r0 * G + g));
        } else {
            ra.a = z, ra.b = z, s0 = 0.f;
        }
        if (v1) {
            const uint4 *p = reinterpret_cast<const uint4 *>(packed + (r1 * G + g) * kPq2GroupBytes);
            rb.a = __ldcs(p);
            rb.b = __ldcs(p + 1);
            s1 = half_bits_to_float(__ldg(scales + r1 * G + g));
        } else {
            rb.a = z, rb.b = z, s1 = 0.f;
        }
    };

    Raw ca, cb, na, nb;
    float cs0 = 0.f, cs1 = 0.f, ns0 = 0.f, ns1 = 0.f;
    if (g_begin < g_end) load_raw(g_begin, ca, cb, cs0, cs1);

    for (int sub = g_begin; sub < g_end; sub += kSubGroups) {
        const int nsub = g_end - sub < kSubGroups ? g_end - sub : kSubGroups;
        __syncthreads();  // the previous sub-chunk's x' is no longer read
        // stage x'[m][128*sub .. 128*(sub+nsub)) as [k-step][token][16], element k scaled 4^-(k mod 4)
        for (int idx = tid; idx < nsub * 8 * MT * 4; idx += kThreads) {
            const int q4 = idx & 3;            // which 4 halves of the 16
            const int m = (idx >> 2) % MT;
            const int ks = (idx >> 2) / MT;    // k-step within the sub-chunk
            const int64_t k = (int64_t)sub * kGroup + ks * 16 + q4 * 4;
            uint2 out = make_uint2(0u, 0u);
            if (m < M) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(xr + (int64_t)m * K + k);
                const __half2 lo = *reinterpret_cast<const __half2 *>(&raw.x);
                const __half2 hi = *reinterpret_cast<const __half2 *>(&raw.y);
                const __half2 f01 = __hmul2(lo, __floats2half2_rn(1.f, 0.25f));
                const __half2 f23 = __hmul2(hi, __floats2half2_rn(0.0625f, 0.015625f));
                out.x = *reinterpret_cast<const uint32_t *>(&f01);
                out.y = *reinterpret_cast<const uint32_t *>(&f23);
            }
            *reinterpret_cast<uint2 *>(xs + ((ks * MT + m) * 16 + q4 * 4)) = out;
        }
        // group sums of x' per token (FP32 sum of the FP16 values)
        for (int pair = warp; pair < MT * nsub; pair += kWarps) {
            const int m = pair % MT, gl = pair / MT;
            float v = 0.f;
            if (m < M) {
                float f[4];
                load_half4(xr + (int64_t)m * K + (int64_t)(sub + gl) * kGroup + 4 * lane, f);
                v = (f[0] + f[1]) + (f[2] + f[3]);
            }
            v = warp_sum(v);
            if (lane == 0) gsum[m * kSubGroups + gl] = v;
        }
        __syncthreads();

        for (int gl = 0; gl < nsub; gl++) {
            const int g = sub + gl;
            if (g + 1 < g_end) load_raw(g + 1, na, nb, ns0, ns1);  // next group in flight
            float d[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; nt++)
#pragma unroll
                for (int e = 0; e < 4; e++) d[nt][e] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint32_t p0 = __byte_perm(word_of(ca, i), 0u, sel);
                const uint32_t p1 = __byte_perm(word_of(cb, i), 0u, sel);
                const uint32_t a0 = p0 & 0x000C0003u, a1 = p1 & 0x000C0003u;
                const uint32_t a2 = p0 & 0x00C00030u, a3 = p1 & 0x00C00030u;
                const int ks = gl * 8 + i;
#pragma unroll
                for (int nt = 0; nt < NT; nt++) {
                    const uint2 b = *reinterpret_cast<const uint2 *>(xs + ((ks * MT + nt * 8 + gid) * 16 + tq * 4));
                    mma16816(d[nt], a0, a1, a2, a3, b.x, b.y);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const int m0 = nt * 8 + 2 * tq;
                const float gs0 = gsum[m0 * kSubGroups + gl], gs1 = gsum[(m0 + 1) * kSubGroups + gl];
                // d[0], d[1]: row r0, tokens m0, m0+1; d[2], d[3]: row r1
                acc[nt][0] = fmaf(cs0, fmaf(d[nt][0], 16777216.f, -gs0), acc[nt][0]);
                acc[nt][1] = fmaf(cs0, fmaf(d[nt][1], 16777216.f, -gs1), acc[nt][1]);
                acc[nt][2] = fmaf(cs1, fmaf(d[nt][2], 16777216.f, -gs0), acc[nt][2]);
                acc[nt][3] = fmaf(cs1, fmaf(d[nt][3], 16777216.f, -gs1), acc[nt][3]);
            }
            ca = na, cb = nb, cs0 = ns0, cs1 = ns1;
        }
    }

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

int smem_bytes(int NT) { return kSubGroups * 8 * NT * 8 * 32 + NT * 8 * kSubGroups * 4; }

// K chunks: enough CTAs for about two waves, unless split_k (> 0) says otherwise.
void choose_split(int64_t N, int64_t K, int split_k, const DeviceInfo &dev, int *S, int *gpc) {
    const int64_t G = K / kGroup;
    const int64_t rb = (N + kRowsPerCta - 1) / kRowsPerCta;
    int64_t s = split_k > 0 ? split_k : (2 * (int64_t)dev.sm_count + rb - 1) / rb;
    if (s < 1) s = 1;
    if (s > G) s = G;
    const int64_t per = (G + s - 1) / s;
    *gpc = (int)per;
    *S = (int)((G + per - 1) / per);
}

}  // namespace

bool skinny_supported(int64_t M, int64_t N, int64_t K, int fmt) {
    return fmt == 2 && M >= 1 && M <= 16 && K % kGroup == 0 && (N + 15) / 16 <= kMaxTiles &&
           K < ((int64_t)1 << 31);
}

size_t skinny_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev) {
    (void)fmt;
    int S, gpc;
    choose_split(N, K, split_k, dev, &S, &gpc);
    const size_t xbytes = ((size_t)M * (size_t)K * 2 + 255) / 256 * 256;
    return xbytes + (S > 1 ? (size_t)S * (size_t)M * (size_t)N * sizeof(float) : 0);
}

cudaError_t launch_skinny(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                          uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int split_k,
                          const Workspace &ws, cudaStream_t s, const DeviceInfo &dev) {
    (void)fmt;
    uint16_t *xr = reinterpret_cast<uint16_t *>(ws.data);
    cudaError_t err = launch_hadamard_f16(x, xr, M, K, s, dev);
    if (err != cudaSuccess) return err;
    int S, gpc;
    choose_split(N, K, split_k, dev, &S, &gpc);
    float *partials = reinterpret_cast<float *>(ws.data + ((size_t)M * (size_t)K * 2 + 255) / 256 * 256);
    const dim3 grid((unsigned)((N + kRowsPerCta - 1) / kRowsPerCta), (unsigned)S);
    if (M <= 8) {
        err = cudaFuncSetAttribute(skinny_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes(1));
        if (err != cudaSuccess) return err;
        skinny_kernel<1><<<grid, kThreads, smem_bytes(1), s>>>(xr, packed, scales, y, partials, ws.counters,
                                                               (int)M, N, K, S, gpc);
    } else {
        err = cudaFuncSetAttribute(skinny_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes(2));
        if (err != cudaSuccess) return err;
        skinny_kernel<2><<<grid, kThreads, smem_bytes(2), s>>>(xr, packed, scales, y, partials, ws.counters,
                                                               (int)M, N, K, S, gpc);
    }
    return cudaGetLastError();
}

}  // namespace bonsai
