// bonsai_api.cu -- the extern "C" boundary of libbonsai (declared in include/bonsai.h).
//
// Every entry point validates its arguments on the host before touching the
// GPU, returns a bonsai_status code, and launches asynchronously on the
// caller's stream.  Per-device state (device properties, the workspace) is
// created on first use and kept until bonsai_shutdown().
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/bonsai.h"
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

constexpr int kMaxDevices = 64;
// Sizes are int64 in the interface; kernels index with int64 but grid and
// per-row arithmetic assumes a row of K activations and a plane of N rows fit
// comfortably below these bounds.
constexpr int64_t kMaxDim = int64_t(1) << 31;

struct DeviceState {
    bool probed = false;
    int status = BONSAI_OK;  // BONSAI_ERR_ARCH if the device cannot run sm_100a code
    DeviceInfo info;
    void *ws_base = nullptr;
    size_t ws_bytes = 0;  // total allocation (counters + data)
    void *zb_base = nullptr;
    size_t zb_bytes = 0;  // the zero-initialised region
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
bool g_force_wait_timeouts = false;  // test hook (bonsai_debug_force_timeouts)

int probe_current(int *dev_out, DeviceState **st_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return BONSAI_ERR_CUDA;
    }
    DeviceState &st = g_dev[dev];
    if (!st.probed) {
        DeviceInfo info;
        if (cudaDeviceGetAttribute(&info.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&info.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&info.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&info.l2_bytes, cudaDevAttrL2CacheSize, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&info.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
            cudaGetLastError();
            return BONSAI_ERR_CUDA;
        }
        st.info = info;
        // the library is built for sm_100a only
        st.status = (info.major == 10 && info.minor == 0) ? BONSAI_OK : BONSAI_ERR_ARCH;
        st.probed = true;
    }
    st.info.force_wait_timeouts = g_force_wait_timeouts;
    *dev_out = dev;
    *st_out = &st;
    return st.status;
}

// Makes sure the current device's workspace holds at least data_bytes after the
// counter block.  Grows by reallocating (after a device synchronisation, since
// work in flight may still use the old buffer).
int ensure_workspace(DeviceState &st, size_t data_bytes, size_t zeroed_bytes, Workspace *ws) {
    const size_t need = kCounterBytes + ((data_bytes + 255) / 256) * 256;
    // the zeroed region always holds at least the control words (the device status word)
    if (zeroed_bytes < kCtlRegionBytes) zeroed_bytes = kCtlRegionBytes;
    if (st.ws_bytes < need) {
        if (st.ws_base) {
            if (cudaDeviceSynchronize() != cudaSuccess) return BONSAI_ERR_CUDA;
            cudaFree(st.ws_base);
            st.ws_base = nullptr;
            st.ws_bytes = 0;
        }
        size_t grow = need < (size_t(64) << 20) ? (size_t(64) << 20) : need;  // at least 64 MiB
        void *p = nullptr;
        if (cudaMalloc(&p, grow) != cudaSuccess) {
            cudaGetLastError();
            return BONSAI_ERR_NOMEM;
        }
        // counters must start at zero; the kernels keep them at zero afterwards
        if (cudaMemset(p, 0, kCounterBytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
            cudaFree(p);
            return BONSAI_ERR_CUDA;
        }
        st.ws_base = p;
        st.ws_bytes = grow;
    }
    if (st.zb_bytes < zeroed_bytes) {
        if (st.zb_base) {
            if (cudaDeviceSynchronize() != cudaSuccess) return BONSAI_ERR_CUDA;
            cudaFree(st.zb_base);
            st.zb_base = nullptr;
            st.zb_bytes = 0;
        }
        const size_t grow = zeroed_bytes < (size_t(16) << 20) ? (size_t(16) << 20) : zeroed_bytes;
        void *p = nullptr;
        if (cudaMalloc(&p, grow) != cudaSuccess) {
            cudaGetLastError();
            return BONSAI_ERR_NOMEM;
        }
        if (cudaMemset(p, 0, grow) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
            cudaFree(p);
            return BONSAI_ERR_CUDA;
        }
        st.zb_base = p;
        st.zb_bytes = grow;
    }
    ws->zeroed = static_cast<uint8_t *>(st.zb_base);
    ws->zeroed_bytes = st.zb_bytes;
    ws->counters = static_cast<unsigned int *>(st.ws_base);
    ws->data = static_cast<uint8_t *>(st.ws_base) + kCounterBytes;
    ws->data_bytes = st.ws_bytes - kCounterBytes;
    return BONSAI_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K <= 0 || K % kGroup != 0) return BONSAI_ERR_SHAPE;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return BONSAI_ERR_SHAPE;
    return BONSAI_OK;
}

int check_fmt(int fmt) {
    return (fmt == BONSAI_FMT_PTQ1_0 || fmt == BONSAI_FMT_PQ2_0 || fmt == BONSAI_FMT_Q1_0 ||
            fmt == BONSAI_FMT_PQ2_0_G64)
               ? BONSAI_OK
               : BONSAI_ERR_FMT;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return BONSAI_OK;
    cudaGetLastError();
    return BONSAI_ERR_CUDA;
}

// Picks the kernel for AUTO, or checks an explicit choice.  Without the device (argument
// checks before the device is probed) AUTO assumes the integer GEMV's grid fits; callers
// resolve AUTO again with the device once it is known.
int resolve_algo(int algo, int64_t M, int64_t N, int64_t K, int fmt, const DeviceInfo *dev = nullptr) {
    if (algo == BONSAI_ALGO_AUTO) {
        if (M <= 3 && gemv_imma_supported(M, N, K, fmt) && (dev == nullptr || gemv_imma_grid_fits(N, K, *dev)))
            return BONSAI_ALGO_IMMA;
        if (M == 1 && gemv_supported(M, N, K, fmt)) return BONSAI_ALGO_GEMV;
        if (M <= 16 && skinny_supported(M, N, K, fmt)) return BONSAI_ALGO_SKINNY;
        if (gemm_supported(M, N, K, fmt)) return BONSAI_ALGO_GEMM;
        return BONSAI_ALGO_SIMPLE;
    }
    switch (algo) {
        case BONSAI_ALGO_SIMPLE: return algo;
        case BONSAI_ALGO_GEMV: return gemv_supported(M, N, K, fmt) ? algo : BONSAI_ERR_ALGO;
        case BONSAI_ALGO_SKINNY: return skinny_supported(M, N, K, fmt) ? algo : BONSAI_ERR_ALGO;
        case BONSAI_ALGO_GEMM: return gemm_supported(M, N, K, fmt) ? algo : BONSAI_ERR_ALGO;
        case BONSAI_ALGO_IMMA: return gemv_imma_supported(M, N, K, fmt) ? algo : BONSAI_ERR_ALGO;
        default: return BONSAI_ERR_ALGO;
    }
}

// Launches the chosen kernel (argument checks and the workspace are the caller's).
cudaError_t run_linear(int chosen, const uint16_t *x, const uint8_t *packed, const uint16_t *scales, uint16_t *y,
                       int64_t M, int64_t N, int64_t K, int fmt, int split_k, const Workspace &ws, cudaStream_t s,
                       const DeviceInfo &info) {
    switch (chosen) {
        case BONSAI_ALGO_GEMV: return launch_gemv(x, packed, scales, y, N, K, fmt, split_k, ws, s, info);
        case BONSAI_ALGO_SKINNY: return launch_skinny(x, packed, scales, y, M, N, K, fmt, split_k, ws, s, info);
        case BONSAI_ALGO_GEMM: return launch_gemm(x, packed, scales, y, M, N, K, fmt, split_k, ws, s, info);
        case BONSAI_ALGO_IMMA: return launch_gemv_imma(x, packed, scales, y, M, N, K, fmt, ws, s, info);
        default: return launch_linear_simple(x, packed, scales, y, M, N, K, fmt, ws, s, info);
    }
}

size_t workspace_for(int algo, int64_t M, int64_t N, int64_t K, int fmt, int split_k,
                     const DeviceInfo &info) {
    switch (algo) {
        case BONSAI_ALGO_GEMV: return gemv_workspace_bytes(N, K, fmt, split_k, info);
        case BONSAI_ALGO_SKINNY: return skinny_workspace_bytes(M, N, K, fmt, split_k, info);
        case BONSAI_ALGO_GEMM: return gemm_workspace_bytes(M, N, K, fmt, info);
        case BONSAI_ALGO_IMMA: return 0;
        default: return simple_workspace_bytes(M, N, K);
    }
}

}  // namespace

int current_device_info(DeviceInfo *out) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    const int rc = probe_current(&dev, &st);
    if (rc == BONSAI_OK) *out = st->info;
    return rc;
}

}  // namespace bonsai

using namespace bonsai;

extern "C" {

int bonsai_version(void) { return (0 << 16) | (1 << 8) | 0; }

const char *bonsai_status_string(int status) {
    switch (status) {
        case BONSAI_OK: return "ok";
        case BONSAI_ERR_NULL: return "a required pointer is NULL";
        case BONSAI_ERR_SHAPE: return "bad shape (negative size, K not a positive multiple of 128, or too large)";
        case BONSAI_ERR_FMT: return "unknown packing format";
        case BONSAI_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case BONSAI_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case BONSAI_ERR_ARCH: return "current device is not an sm_100 (B200-class) GPU";
        case BONSAI_ERR_NOMEM: return "could not allocate the device workspace";
        case BONSAI_ERR_ALGO: return "the requested kernel cannot run this shape";
        case BONSAI_ERR_TOO_LARGE: return "the problem needs more than the fixed device scratch of the no-allocation entry point";
        default: return "unknown status";
    }
}

int bonsai_check_device(void) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    return probe_current(&dev, &st);
}

int64_t bonsai_packed_bytes(int fmt, int64_t N, int64_t K) {
    if (check_fmt(fmt) != BONSAI_OK) return BONSAI_ERR_FMT;
    if (check_shape(0, N, K) != BONSAI_OK) return BONSAI_ERR_SHAPE;
    if (fmt == BONSAI_FMT_PTQ1_0) return N * (K / kGroup) * kPtq1GroupBytes;
    if (fmt == BONSAI_FMT_Q1_0) return N * (K / 8);
    return N * (K / 4);
}

static int pack_common(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream,
                       int fmt) {
    int rc = check_shape(0, N, K);
    if (rc != BONSAI_OK) return rc;
    if (N == 0) return BONSAI_OK;
    if (!trits || !packed) return BONSAI_ERR_NULL;
    if (!aligned16(trits) || !aligned16(packed)) return BONSAI_ERR_ALIGN;
    int dev;
    DeviceState *st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        rc = probe_current(&dev, &st);
    }
    if (rc != BONSAI_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fmt == BONSAI_FMT_PTQ1_0) return cuda_status(launch_pack_ptq1(trits, packed, N, K, s, st->info));
    if (fmt == BONSAI_FMT_Q1_0) return cuda_status(launch_pack_q1(trits, packed, N, K, s, st->info));
    return cuda_status(launch_pack_pq2(trits, packed, N, K, s, st->info));
}

int bonsai_pack_ptq1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream) {
    return pack_common(trits, packed, N, K, stream, BONSAI_FMT_PTQ1_0);
}

int bonsai_pack_pq2(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream) {
    return pack_common(trits, packed, N, K, stream, BONSAI_FMT_PQ2_0);
}

int bonsai_pack_q1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K, void *stream) {
    return pack_common(trits, packed, N, K, stream, BONSAI_FMT_Q1_0);
}

int bonsai_unpack(int fmt, const uint8_t *packed, int8_t *trits, int64_t N, int64_t K, void *stream) {
    int rc = check_fmt(fmt);
    if (rc != BONSAI_OK) return rc;
    rc = check_shape(0, N, K);
    if (rc != BONSAI_OK) return rc;
    if (N == 0) return BONSAI_OK;
    if (!trits || !packed) return BONSAI_ERR_NULL;
    if (!aligned16(trits) || !aligned16(packed)) return BONSAI_ERR_ALIGN;
    int dev;
    DeviceState *st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        rc = probe_current(&dev, &st);
    }
    if (rc != BONSAI_OK) return rc;
    return cuda_status(launch_unpack(fmt, packed, trits, N, K, static_cast<cudaStream_t>(stream), st->info));
}

int bonsai_hadamard128(const uint16_t *x, uint16_t *x_out, int64_t M, int64_t K, void *stream) {
    int rc = check_shape(M, 0, K);
    if (rc != BONSAI_OK) return rc;
    if (M == 0) return BONSAI_OK;
    if (!x || !x_out) return BONSAI_ERR_NULL;
    if (!aligned16(x) || !aligned16(x_out)) return BONSAI_ERR_ALIGN;
    int dev;
    DeviceState *st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        rc = probe_current(&dev, &st);
    }
    if (rc != BONSAI_OK) return rc;
    return cuda_status(launch_hadamard_f16(x, x_out, M, K, static_cast<cudaStream_t>(stream), st->info));
}

int bonsai_ternary_linear_algo(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                               uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int algo,
                               int split_k, void *stream) {
    int rc = check_fmt(fmt);
    if (rc != BONSAI_OK) return rc;
    rc = check_shape(M, N, K);
    if (rc != BONSAI_OK) return rc;
    if (split_k < 0) return BONSAI_ERR_SHAPE;
    if (M == 0 || N == 0) return BONSAI_OK;
    if (!x || !packed || !scales || !y) return BONSAI_ERR_NULL;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y))
        return BONSAI_ERR_ALIGN;
    int chosen = resolve_algo(algo, M, N, K, fmt);
    if (chosen < 0) return chosen;

    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    if (algo == BONSAI_ALGO_AUTO) chosen = resolve_algo(algo, M, N, K, fmt, &st->info);
    // the integer GEMV's hand-over between CTAs needs its whole grid on the GPU at once
    if (chosen == BONSAI_ALGO_IMMA && !gemv_imma_grid_fits(N, K, st->info)) return BONSAI_ERR_ALGO;
    Workspace ws;
    rc = ensure_workspace(*st, workspace_for(chosen, M, N, K, fmt, split_k, st->info),
                          chosen == BONSAI_ALGO_IMMA ? gemv_imma_zeroed_bytes(M, N, K) : 0, &ws);
    if (rc != BONSAI_OK) return rc;
    return cuda_status(run_linear(chosen, x, packed, scales, y, M, N, K, fmt, split_k, ws,
                                  static_cast<cudaStream_t>(stream), st->info));
}

int bonsai_ternary_linear(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                          uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, void *stream) {
    return bonsai_ternary_linear_algo(x, packed, scales, y, M, N, K, fmt, BONSAI_ALGO_AUTO, 0,
                                      stream);
}

int bonsai_swiglu(const uint16_t *y, uint16_t *h, int64_t M, int64_t F, void *stream) {
    if (M < 0 || F < 0 || M > kMaxDim || F > kMaxDim) return BONSAI_ERR_SHAPE;
    if (M == 0 || F == 0) return BONSAI_OK;
    if (!y || !h) return BONSAI_ERR_NULL;
    if (!aligned16(y) || !aligned16(h)) return BONSAI_ERR_ALIGN;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    const int rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    return cuda_status(launch_swiglu(y, h, M, F, static_cast<cudaStream_t>(stream), st->info));
}

int bonsai_ternary_linear_swiglu(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                 uint16_t *h, int64_t M, int64_t F, int64_t K, int fmt, void *stream) {
    int rc = check_fmt(fmt);
    if (rc != BONSAI_OK) return rc;
    if (F < 0 || F > kMaxDim / 2) return BONSAI_ERR_SHAPE;
    const int64_t N = 2 * F;
    rc = check_shape(M, N, K);
    if (rc != BONSAI_OK) return rc;
    if (M == 0 || F == 0) return BONSAI_OK;
    if (!x || !packed || !scales || !h) return BONSAI_ERR_NULL;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(h))
        return BONSAI_ERR_ALIGN;
    int chosen = resolve_algo(BONSAI_ALGO_AUTO, M, N, K, fmt);
    if (chosen < 0) return chosen;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    chosen = resolve_algo(BONSAI_ALGO_AUTO, M, N, K, fmt, &st->info);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Workspace ws;
    if (chosen == BONSAI_ALGO_IMMA) {  // fused into the GEMV's epilogue
        rc = ensure_workspace(*st, 0, gemv_imma_zeroed_bytes(M, N, K), &ws);
        if (rc != BONSAI_OK) return rc;
        return cuda_status(launch_gemv_imma(x, packed, scales, h, M, N, K, fmt, ws, s, st->info, F));
    }
    if (chosen == BONSAI_ALGO_GEMM) {  // fused into the GEMM's epilogue
        rc = ensure_workspace(*st, workspace_for(chosen, M, N, K, fmt, 0, st->info), 0, &ws);
        if (rc != BONSAI_OK) return rc;
        return cuda_status(launch_gemm(x, packed, scales, h, M, N, K, fmt, 0, ws, s, st->info, F));
    }
    // otherwise: the linear layer into the tail of the workspace, then the SwiGLU kernel
    const size_t need = (workspace_for(chosen, M, N, K, fmt, 0, st->info) + 255) / 256 * 256;
    rc = ensure_workspace(*st, need + (size_t)M * (size_t)N * 2,
                          chosen == BONSAI_ALGO_IMMA ? gemv_imma_zeroed_bytes(M, N, K) : 0, &ws);
    if (rc != BONSAI_OK) return rc;
    uint16_t *y = reinterpret_cast<uint16_t *>(ws.data + need);
    Workspace inner = ws;
    inner.data_bytes = need;
    cudaError_t e = run_linear(chosen, x, packed, scales, y, M, N, K, fmt, 0, inner, s, st->info);
    if (e == cudaSuccess) e = launch_swiglu(y, h, M, F, s, st->info);
    return cuda_status(e);
}

int bonsai_launch_count(int64_t M, int64_t N, int64_t K, int fmt, int algo, int split_k) {
    int rc = check_fmt(fmt);
    if (rc != BONSAI_OK) return rc;
    rc = check_shape(M, N, K);
    if (rc != BONSAI_OK) return rc;
    if (M == 0 || N == 0) return 0;
    int chosen = resolve_algo(algo, M, N, K, fmt);
    if (chosen < 0) return chosen;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    if (algo == BONSAI_ALGO_AUTO) chosen = resolve_algo(algo, M, N, K, fmt, &st->info);
    if (chosen == BONSAI_ALGO_IMMA && !gemv_imma_grid_fits(N, K, st->info)) return BONSAI_ERR_ALGO;
    switch (chosen) {
        case BONSAI_ALGO_GEMV: return gemv_launches(N, K, fmt, split_k, st->info);
        case BONSAI_ALGO_IMMA: return 1;  // the rotation and quantisation of x are fused
        case BONSAI_ALGO_GEMM: return 1;  // the rotation is the kernel's first phase
        case BONSAI_ALGO_SKINNY: {  // fused when its grid is resident at once
            const int n = skinny_launches(M, N, K, fmt, split_k, st->info);
            return n < 0 ? BONSAI_ERR_CUDA : n;
        }
        default: return 2;  // the rotation pass, then the kernel
    }
}

int bonsai_reserve(int64_t M, int64_t N, int64_t K) {
    int rc = check_shape(M, N, K);
    if (rc != BONSAI_OK) return rc;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    size_t need = simple_workspace_bytes(M, N, K), zneed = 0;
    for (int fmt = BONSAI_FMT_PTQ1_0; fmt <= BONSAI_FMT_PQ2_0_G64; fmt++) {
        size_t v;
        if (M <= 1 && gemv_supported(1, N, K, fmt)) {
            v = gemv_workspace_bytes(N, K, fmt, 0, st->info);
            need = v > need ? v : need;
        }
        for (int64_t m = 1; m <= 3 && m <= (M > 1 ? M : 1); m++)
            if (gemv_imma_supported(m, N, K, fmt)) {
                v = gemv_imma_zeroed_bytes(m, N, K);
                zneed = v > zneed ? v : zneed;
            }
        if (skinny_supported(M < 16 ? M : 16, N, K, fmt)) {
            v = skinny_workspace_bytes(M < 16 ? M : 16, N, K, fmt, 0, st->info);
            need = v > need ? v : need;
        }
        if (gemm_supported(M, N, K, fmt)) {
            v = gemm_workspace_bytes(M, N, K, fmt, st->info);
            need = v > need ? v : need;
        }
    }
    Workspace ws;
    // + the tail in which a non-fused bonsai_ternary_linear_swiglu keeps its M x N output
    need = (need + 255) / 256 * 256 + (size_t)M * (size_t)N * 2;
    return ensure_workspace(*st, need, zneed, &ws);
}

int bonsai_device_status(void *stream, uint32_t *bits, int clear) {
    if (!bits) return BONSAI_ERR_NULL;
    *bits = 0;
    std::lock_guard<std::mutex> lock(g_mutex);
    int dev;
    DeviceState *st;
    int rc = probe_current(&dev, &st);
    if (rc != BONSAI_OK) return rc;
    if (!st->zb_base) return BONSAI_OK;  // no call has run on this device: nothing to report
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int *word = static_cast<unsigned int *>(st->zb_base) + kCtlStatus;
    unsigned int host = 0;
    if (cudaMemcpyAsync(&host, word, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        (clear && cudaMemsetAsync(word, 0, sizeof(unsigned int), s) != cudaSuccess) ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return BONSAI_ERR_CUDA;
    }
    *bits = host;
    return BONSAI_OK;
}

int bonsai_debug_force_timeouts(int enable) {
    std::lock_guard<std::mutex> lock(g_mutex);
    g_force_wait_timeouts = enable != 0;
    return BONSAI_OK;
}

void bonsai_shutdown(void) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int current = -1;
    cudaGetDevice(&current);
    for (int d = 0; d < kMaxDevices; d++) {
        if (g_dev[d].ws_base) {
            cudaSetDevice(d);
            cudaDeviceSynchronize();
            cudaFree(g_dev[d].ws_base);
            g_dev[d].ws_base = nullptr;
            g_dev[d].ws_bytes = 0;
        }
        if (g_dev[d].zb_base) {
            cudaSetDevice(d);
            cudaDeviceSynchronize();
            cudaFree(g_dev[d].zb_base);
            g_dev[d].zb_base = nullptr;
            g_dev[d].zb_bytes = 0;
        }
    }
    if (current >= 0) cudaSetDevice(current);
    cudaGetLastError();
}

}  // extern "C"
