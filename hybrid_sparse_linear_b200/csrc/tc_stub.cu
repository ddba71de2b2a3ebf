// Placeholder dispatch for the tensor-core kernels until they land: reports "unsupported" so
// the CUDA-core kernels run.
#include "kernels.h"

namespace sala {
bool linear_prefill_tc_supported(int) { return false; }
bool sparse_prefill_tc_supported(int, int, int) { return false; }
cudaError_t launch_linear_prefill_tc(const void*, const void*, const void*, const float*, void*,
                                     const float*, float*, int, int, int, int, cudaStream_t,
                                     DevCtx) {
    return cudaErrorNotSupported;
}
cudaError_t launch_sparse_prefill_tc(const void*, const void*, const void*, const int32_t*, void*,
                                     int, int, int, int, int, int, float, cudaStream_t, DevCtx) {
    return cudaErrorNotSupported;
}
}  // namespace sala
