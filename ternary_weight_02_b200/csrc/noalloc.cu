// noalloc.cu -- bonsai_ternary_linear_noalloc: the batch-1 ternary linear layer for
// callers that cannot allocate device memory (code running while a CUDA graph is being
// captured, allocators that must own every byte of the device, hosts that forbid
// allocation after start-up).
//
// The split-K GEMV needs scratch: one FP32 partial per (512-weight K slice, row), summed
// in slice order by its second kernel.  Here that scratch is a fixed array in the
// library's own device image instead of the per-device workspace, so the call never
// allocates.  Every GPU that loads the library holds the array (4 MiB) until the process
// exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bonsai.h"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kScratchPartials = 1 << 20;    // FP32 partials: (K / 512) * N <= 2^20
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_scratch[kScratchPartials];

std::mutex g_setup_mutex;
float *g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device

// Looks up the current device's copy of the array once (that device must be current).
int scratch_for_current_device(float **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return BONSAI_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return BONSAI_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<float *>(p);
    }
    *out = g_scratch_addr[dev];
    return BONSAI_OK;
}

}  // namespace
}  // namespace bonsai

using namespace bonsai;

extern "C" int bonsai_ternary_linear_noalloc(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                             uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt,
                                             void *stream) {
    if (fmt != BONSAI_FMT_PTQ1_0 && fmt != BONSAI_FMT_PQ2_0) return BONSAI_ERR_FMT;
    if (M < 0 || N < 0 || K <= 0 || K % 128 != 0) return BONSAI_ERR_SHAPE;
    if (M == 0 || N == 0) return BONSAI_OK;
    if (!x || !packed || !scales || !y) return BONSAI_ERR_NULL;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(packed) |
                          reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(y);
    if (mis & 15u) return BONSAI_ERR_ALIGN;
    if (M != 1 || K % 512 != 0 || gemv_split_partial_floats(N, K) > (size_t)kScratchPartials)
        return BONSAI_ERR_TOO_LARGE;

    DeviceInfo info;
    int rc = current_device_info(&info);
    if (rc != BONSAI_OK) return rc;
    float *partials = nullptr;
    rc = scratch_for_current_device(&partials);
    if (rc != BONSAI_OK) return rc;
    // Every partial the reduction reads is written by the same call first, so nothing in
    // the array needs clearing; the array keeps whatever the last call left.
    const cudaError_t e = launch_gemv_split_scratch(x, packed, scales, y, N, K, fmt, partials,
                                                    (size_t)kScratchPartials, static_cast<cudaStream_t>(stream), info);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return BONSAI_ERR_CUDA;
    }
    return BONSAI_OK;
}
