// pack.cu -- PTQ1_0 / PQ2_0 packing and unpacking of trits.
//
// Formats: "27B 模型压到 5.95GB，推理能力还保住 98%" (allhereai.com), paragraph on
// the two file packings: PTQ1_0 stores trits compactly (five per byte as a
// base-3 number, 3^5 = 243 <= 256, per "Bonsai把 27B 大模型塞进手机..." (wmrh.cn),
// section 关键机制), PQ2_0 puts each trit in a 2-bit slot.  Byte layouts as
// stated in include/bonsai.h.  Packing runs offline, so these kernels favour
// plainness over speed: one thread per packed byte, grid-stride loops.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

__device__ __forceinline__ bool trit_ok(int t) { return t >= -1 && t <= 1; }

__global__ void pack_ptq1_kernel(const int8_t *__restrict__ trits, uint8_t *__restrict__ packed,
                                 int64_t total, int64_t K) {
    const int64_t G = K / kGroup;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t q = i / kPtq1GroupBytes;  // q = n * G + g
        const int b = (int)(i - q * kPtq1GroupBytes);
        const int64_t n = q / G, g = q - n * G;
        const int8_t *t = trits + n * K + g * kGroup + 5 * b;
        const int count = b < 25 ? 5 : 3;
        int value = 0, power = 1;
        bool ok = true;
        for (int j = 0; j < count; j++) {
            const int tj = t[j];
            ok = ok && trit_ok(tj);
            value += (tj + 1) * power;
            power *= 3;
        }
        packed[i] = ok ? (uint8_t)value : (uint8_t)0xFF;
    }
}

__global__ void pack_pq2_kernel(const int8_t *__restrict__ trits, uint8_t *__restrict__ packed,
                                int64_t total) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        // byte i of the plane holds weights 4i .. 4i+3 of the row-major N x K matrix
        const char4 t = *reinterpret_cast<const char4 *>(trits + 4 * i);
        const int tt[4] = {t.x, t.y, t.z, t.w};
        int value = 0;
        for (int j = 0; j < 4; j++) {
            const int code = trit_ok(tt[j]) ? tt[j] + 1 : 3;
            value |= code << (2 * j);
        }
        packed[i] = (uint8_t)value;
    }
}

__global__ void pack_q1_kernel(const int8_t *__restrict__ trits, uint8_t *__restrict__ packed,
                               int64_t total) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        // byte i of the plane holds weights 8i .. 8i+7, bit j = (weight 8i+j == +1)
        const int2 t8 = *reinterpret_cast<const int2 *>(trits + 8 * i);
        int value = 0;
        for (int j = 0; j < 8; j++) {
            const int t = (int8_t)(((j < 4 ? t8.x : t8.y) >> (8 * (j & 3))) & 0xFF);
            value |= (t == 1 ? 1 : 0) << j;
        }
        packed[i] = (uint8_t)value;
    }
}

__global__ void unpack_q1_kernel(const uint8_t *__restrict__ packed, int8_t *__restrict__ trits,
                                 int64_t total) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int v = packed[i];
        int8_t out[8];
        for (int j = 0; j < 8; j++) out[j] = ((v >> j) & 1) ? (int8_t)1 : (int8_t)-1;
        *reinterpret_cast<char4 *>(trits + 8 * i) = make_char4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<char4 *>(trits + 8 * i + 4) = make_char4(out[4], out[5], out[6], out[7]);
    }
}

__global__ void unpack_ptq1_kernel(const uint8_t *__restrict__ packed, int8_t *__restrict__ trits,
                                   int64_t total, int64_t K) {
    const int64_t G = K / kGroup;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t q = i / kPtq1GroupBytes;
        const int b = (int)(i - q * kPtq1GroupBytes);
        const int64_t n = q / G, g = q - n * G;
        int8_t *t = trits + n * K + g * kGroup + 5 * b;
        const int count = b < 25 ? 5 : 3;
        int v = packed[i];
        const bool ok = v < 243;
        for (int j = 0; j < count; j++) {
            t[j] = ok ? (int8_t)(v % 3 - 1) : (int8_t)-128;
            v /= 3;
        }
    }
}

__global__ void unpack_pq2_kernel(const uint8_t *__restrict__ packed, int8_t *__restrict__ trits,
                                  int64_t total) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int v = packed[i];
        int8_t out[4];
        for (int j = 0; j < 4; j++) {
            const int code = (v >> (2 * j)) & 3;
            out[j] = code == 3 ? (int8_t)-128 : (int8_t)(code - 1);
        }
        *reinterpret_cast<char4 *>(trits + 4 * i) = make_char4(out[0], out[1], out[2], out[3]);
    }
}

int grid_for(int64_t work, int threads, const DeviceInfo &dev) {
    const int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)dev.sm_count * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_pack_ptq1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                             cudaStream_t s, const DeviceInfo &dev) {
    const int64_t total = N * (K / kGroup) * kPtq1GroupBytes;
    if (total == 0) return cudaSuccess;
    pack_ptq1_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(trits, packed, total, K);
    return cudaGetLastError();
}

cudaError_t launch_pack_pq2(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                            cudaStream_t s, const DeviceInfo &dev) {
    const int64_t total = N * (K / 4);
    if (total == 0) return cudaSuccess;
    pack_pq2_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(trits, packed, total);
    return cudaGetLastError();
}

cudaError_t launch_pack_q1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo &dev) {
    const int64_t total = N * (K / 8);
    if (total == 0) return cudaSuccess;
    pack_q1_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(trits, packed, total);
    return cudaGetLastError();
}

cudaError_t launch_unpack(int fmt, const uint8_t *packed, int8_t *trits, int64_t N, int64_t K,
                          cudaStream_t s, const DeviceInfo &dev) {
    if (fmt == 3) {
        const int64_t total = N * (K / 8);
        if (total == 0) return cudaSuccess;
        unpack_q1_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(packed, trits, total);
    } else if (fmt == 1) {
        const int64_t total = N * (K / kGroup) * kPtq1GroupBytes;
        if (total == 0) return cudaSuccess;
        unpack_ptq1_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(packed, trits, total, K);
    } else {
        const int64_t total = N * (K / 4);
        if (total == 0) return cudaSuccess;
        unpack_pq2_kernel<<<grid_for(total, 256, dev), 256, 0, s>>>(packed, trits, total);
    }
    return cudaGetLastError();
}

}  // namespace bonsai
