// Diagnostics kept in the product library: the bounded-wait self-test behind
// sala_selftest_wait_timeout.  One block waits on a shared-memory mbarrier that nothing ever
// arrives on; the wait gives up after the configured limit, records the timeout in the status
// word and the kernel returns normally, leaving the context usable.
#include "kernels.h"
#include "ptx.cuh"

namespace sala {
namespace {

__global__ void selftest_wait_kernel(DevCtx ctx) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)ptx::mbar_wait(&bar, 0, ctx);  // no arrival ever comes
    __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(cudaStream_t st, DevCtx ctx) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(ctx);
    return cudaGetLastError();
}

}  // namespace sala
