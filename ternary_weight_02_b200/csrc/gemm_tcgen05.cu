// gemm_tcgen05.cu -- prefill GEMM (placeholder until the kernel lands).
#include "internal.h"
namespace bonsai {
bool gemm_supported(int64_t, int64_t, int64_t, int) { return false; }
size_t gemm_workspace_bytes(int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemm(const uint16_t *, const uint8_t *, const uint16_t *, uint16_t *, int64_t,
                        int64_t, int64_t, int, const Workspace &, cudaStream_t, const DeviceInfo &) {
    return cudaErrorNotSupported;
}
}  // namespace bonsai
