// tc.cu -- tcgen05 / TMA tensor-core kernels (bf16 storage).  Placeholder until written.
#include "internal.h"

namespace dynconv {
bool tc_supported(const Prob&) { return false; }
size_t tc_workspace_bytes(const Prob&) { return 0; }
cudaError_t tc_forward(const Prob&, const void*, const void*, const void*, const void*, void*, void*, void*,
                       cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_backward(const Prob&, const void*, const void*, const void*, const void*, const void*,
                        const void*, void*, void*, float*, float*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace dynconv
