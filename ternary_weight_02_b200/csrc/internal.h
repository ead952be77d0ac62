// internal.h -- launchers shared between the C-ABI layer (bonsai_api.cu) and the
// kernel files.  Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bonsai {

struct DeviceInfo {
    int sm_count = 0;
    int major = 0, minor = 0;
    int smem_optin = 0;  // max dynamic shared memory per block (opt-in), bytes
    int l2_bytes = 0;
    int smem_reserved = 0;  // shared memory the system reserves per block, bytes
    // test hook (bonsai_debug_force_timeouts): cross-CTA waits look for a value nobody
    // writes and give up after kForcedWaitPolls polls
    bool force_wait_timeouts = false;
};
constexpr uint32_t kForcedWaitPolls = 64;

// Split-K bookkeeping lives at the start of the workspace: kMaxTiles arrival
// counters, zero when the workspace is created and returned to zero by the
// last CTA of each tile, so consecutive calls need no memset.
constexpr int kMaxTiles = 65536;
constexpr size_t kCounterBytes = kMaxTiles * sizeof(unsigned int);

struct Workspace {
    unsigned int *counters = nullptr;  // kMaxTiles entries
    uint8_t *data = nullptr;           // the rest, 256-byte aligned
    size_t data_bytes = 0;
    // a separate region that is zero when created and that its one user (the integer
    // GEMV's split row tiles) returns to zero after every call
    uint8_t *zeroed = nullptr;
    size_t zeroed_bytes = 0;
};

// ---- pack.cu
cudaError_t launch_pack_ptq1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                             cudaStream_t s, const DeviceInfo &dev);
cudaError_t launch_pack_pq2(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                            cudaStream_t s, const DeviceInfo &dev);
cudaError_t launch_pack_q1(const int8_t *trits, uint8_t *packed, int64_t N, int64_t K,
                           cudaStream_t s, const DeviceInfo &dev);
cudaError_t launch_unpack(int fmt, const uint8_t *packed, int8_t *trits, int64_t N, int64_t K,
                          cudaStream_t s, const DeviceInfo &dev);

// ---- hadamard.cu
cudaError_t launch_hadamard_f16(const uint16_t *x, uint16_t *out, int64_t M, int64_t K,
                                cudaStream_t s, const DeviceInfo &dev);
cudaError_t launch_hadamard_f32(const uint16_t *x, float *out, int64_t M, int64_t K,
                                cudaStream_t s, const DeviceInfo &dev);

// ---- linear_simple.cu: x' (FP32, M x K) in the workspace, then one warp per row
size_t simple_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_linear_simple(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                 uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt,
                                 const Workspace &ws, cudaStream_t s, const DeviceInfo &dev);

// ---- gemv_lut.cu: M == 1
bool gemv_supported(int64_t M, int64_t N, int64_t K, int fmt);
size_t gemv_workspace_bytes(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev);
int gemv_launches(int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev);
cudaError_t launch_gemv(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t N, int64_t K, int fmt, int split_k,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev);

// split-mode GEMV on caller-provided scratch for its FP32 partials (no-allocation entry point)
size_t gemv_split_partial_floats(int64_t N, int64_t K);
cudaError_t launch_gemv_split_scratch(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                                      uint16_t *y, int64_t N, int64_t K, int fmt, float *partials,
                                      size_t partial_floats, cudaStream_t s, const DeviceInfo &dev);
// current device's properties (the same probe the other entry points use)
int current_device_info(DeviceInfo *out);

// The zero-initialised workspace region starts with control words that kernels keep across
// calls, as 32-bit words: [kCtlCalls, +1] a 64-bit call counter (low half: CTAs of the
// running call that have read it; high half: calls counted so far, the epoch of the
// cross-CTA hand-over data being one more), [kCtlStatus] sticky device status bits.
// [kCtlGemmFlags, + kCtlGemmMaxCtas): the prefill GEMM's hand-over flags, one per CTA.
constexpr int kCtlCalls = 0, kCtlStatus = 2, kCtlGemmFlags = 64;
constexpr int kCtlGemmMaxCtas = 960;
constexpr size_t kCtlRegionBytes = 4096;
// device status bits (kCtlStatus); the same values are public in bonsai.h
constexpr unsigned int kDevStatusGemvCopyTimeout = 1u;   // integer GEMV: a weight copy never landed
constexpr unsigned int kDevStatusGemvPieceTimeout = 2u;  // integer GEMV: a split tile's later piece never came
constexpr unsigned int kDevStatusGemmTimeout = 4u;       // prefill GEMM: a barrier or hand-over wait gave up
constexpr unsigned int kDevStatusSkinnyTimeout = 8u;     // skinny kernel: the wait for the rotated x, or a TMA copy, gave up

// ---- gemv_imma.cu: M <= 3 (g64: 2), PQ2_0 and g64, integer tensor cores
bool gemv_imma_supported(int64_t M, int64_t N, int64_t K, int fmt);
size_t gemv_imma_zeroed_bytes(int64_t M, int64_t N, int64_t K);  // of Workspace::zeroed
bool gemv_imma_grid_fits(int64_t N, int64_t K, const DeviceInfo &dev);
// swiglu_f > 0: fused gate/up rows, write silu(gate) * up (M x swiglu_f).
cudaError_t launch_gemv_imma(const uint16_t *x, const uint8_t *packed, const uint16_t *scales, uint16_t *y,
                             int64_t M, int64_t N, int64_t K, int fmt, const Workspace &ws, cudaStream_t s,
                             const DeviceInfo &dev, int64_t swiglu_f = 0);

// ---- skinny_mma.cu: 1 <= M <= 16 (one launch when its grid is resident at once: the
// rotation, a barrier on the call counter in Workspace::zeroed, the kernel; else two)
bool skinny_supported(int64_t M, int64_t N, int64_t K, int fmt);
size_t skinny_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int split_k,
                              const DeviceInfo &dev);
int skinny_launches(int64_t M, int64_t N, int64_t K, int fmt, int split_k, const DeviceInfo &dev);
cudaError_t launch_skinny(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                          uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int split_k,
                          const Workspace &ws, cudaStream_t s, const DeviceInfo &dev);

// ---- swiglu.cu: h = silu(y[:, :F]) * y[:, F:] for an M x 2F FP16 y
cudaError_t launch_swiglu(const uint16_t *y, uint16_t *h, int64_t M, int64_t F, cudaStream_t s,
                          const DeviceInfo &dev);

// ---- gemm_tcgen05.cu: prefill
bool gemm_supported(int64_t M, int64_t N, int64_t K, int fmt);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, const DeviceInfo &dev);
// tile_hint: 0 automatic, 1 one 128-row accumulator per CTA, 2 two (256 rows).  One launch:
// the rotation of x into the workspace, a grid barrier, the tiles; hand-over flags and the
// barrier live in the control words of Workspace::zeroed.
// swiglu_f > 0: the N = 2 swiglu_f rows are gate then up rows and y
// gets silu(gate) * up, M x swiglu_f.
cudaError_t launch_gemm(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                        uint16_t *y, int64_t M, int64_t N, int64_t K, int fmt, int tile_hint,
                        const Workspace &ws, cudaStream_t s, const DeviceInfo &dev, int64_t swiglu_f = 0);

}  // namespace bonsai
