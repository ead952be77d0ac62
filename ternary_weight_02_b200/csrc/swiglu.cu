// swiglu.cu -- the SwiGLU step after a fused gate/up projection, as its own kernel.
//
// h[m][f] = silu(y[m][f]) * y[m][F + f], silu(z) = z / (1 + e^-z), for y the M x 2F FP16
// output of one linear layer whose rows 0 .. F-1 are the gate projection and F .. 2F-1 the
// up projection (the 27B-class MLP: F = 17408, fused gate/up N = 34816).  FP32 arithmetic,
// FP16 (nearest even) output.  The batch-1 integer GEMV applies the same step in its
// epilogue (bonsai_ternary_linear_swiglu); this kernel serves every other path, and is
// also exported alone.
//
// Elementwise and HBM-bound: 6 bytes per output.  Launched with programmatic dependent
// launch: it lets the next kernel start and waits for the previous one before reading y.
#include "common.cuh"
#include "internal.h"

namespace bonsai {
namespace {

__global__ void __launch_bounds__(256) swiglu_kernel(const uint16_t *__restrict__ y, uint16_t *__restrict__ h,
                                                     int64_t M, int64_t F) {
    pdl_launch_dependents();
    pdl_wait();  // y may belong to the previous kernel
    const int64_t total = M * F;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / F, f = i - m * F;
        const float g = half_bits_to_float(y[m * 2 * F + f]);
        const float u = half_bits_to_float(y[m * 2 * F + F + f]);
        h[i] = float_to_half_bits(g / (1.f + expf(-g)) * u);
    }
}

}  // namespace

cudaError_t launch_swiglu(const uint16_t *y, uint16_t *h, int64_t M, int64_t F, cudaStream_t s,
                          const DeviceInfo &dev) {
    const int64_t total = M * F;
    if (total == 0) return cudaSuccess;
    const int64_t want = (total + 255) / 256;
    const int64_t cap = (int64_t)dev.sm_count * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, swiglu_kernel, y, h, M, F);
}

}  // namespace bonsai
