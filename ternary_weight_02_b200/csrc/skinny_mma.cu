// skinny_mma.cu -- skinny ternary kernel (placeholder until the kernel lands).
#include "internal.h"
namespace bonsai {
bool skinny_supported(int64_t, int64_t, int64_t, int) { return false; }
size_t skinny_workspace_bytes(int64_t, int64_t, int64_t, int, int, const DeviceInfo &) { return 0; }
cudaError_t launch_skinny(const uint16_t *, const uint8_t *, const uint16_t *, uint16_t *, int64_t,
                          int64_t, int64_t, int, int, const Workspace &, cudaStream_t,
                          const DeviceInfo &) {
    return cudaErrorNotSupported;
}
}  // namespace bonsai
