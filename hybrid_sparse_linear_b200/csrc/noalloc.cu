// sala_sparse_decode_noalloc: the sparse decode step for callers that cannot allocate device
// memory.
//
// Some hosts of this library forbid device allocations once they are running -- a serving loop
// that sizes every buffer at start-up so that no allocation can stall or fail in the middle of a
// request, or a plug-in inside an application that owns the whole device memory pool and hands
// out no allocator.  Such a caller can still pass its inputs and outputs, but it has no way to
// provide the scratch space sala_sparse_decode asks for.  This entry point brings that scratch
// with it: a fixed area compiled into the library (a file-scope __device__ array), so the call
// itself allocates nothing, directly or through any library.
//
// The area is kNoallocScratchBytes (4 MiB) per GPU and exists on every GPU that loads the library
// until the process exits.  All calls on a GPU share it, so two calls that may run at the same
// time on that GPU (different streams, no ordering between them) race on it and must not be made.
// The area keeps whatever the previous call left there.  Its first 256 bytes are the counters of
// the one-launch path's grid barrier, which must read zero when a call starts.  A call that gave
// up on a wait (SALA_ERR_TIMEOUT) can leave them nonzero, and no caller can reach the area to
// clear them, so every call, once its arguments have passed validation, first zeroes those 256 bytes on its
// own stream (cudaMemsetAsync, which allocates nothing): each call starts from clean counters
// whatever the previous call did.  Every
// other byte a call reads it has written earlier in the same call.
#include <mutex>

#include "../../include/sala.h"
#include "kernels.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch area on the current device.  The host-side name of a __device__
// array is only a stand-in; the address a kernel can use comes from cudaGetSymbolAddress, looked
// up once per device (with that device current) and cached.
sala_status scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        sala::set_last_error("sala_sparse_decode_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
        return SALA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        sala::set_last_error("sala_sparse_decode_noalloc: device index %d is not supported", dev);
        return SALA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            sala::set_last_error("sala_sparse_decode_noalloc: cudaGetSymbolAddress failed: %s",
                                 cudaGetErrorString(e));
            return SALA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SALA_OK;
}

}  // namespace

extern "C" sala_status sala_sparse_decode_noalloc(const void* q, const void* kcache,
                                                  const void* vcache, const void* kbar,
                                                  const int32_t* idx_in, int32_t* idx_out,
                                                  void* o, int B, int H, int Hkv, int pos,
                                                  int Tmax, int nb_cap, int d, int block,
                                                  int topk, int n_init, int n_local, float scale,
                                                  sala_dtype dt, sala_stream stream) {
    const size_t need =
        sala_sparse_decode_workspace(B, H, Hkv, pos, block, topk, n_init, n_local, d);
    if (need > kNoallocScratchBytes) {
        sala::set_last_error(
            "sala_sparse_decode_noalloc: this problem needs %zu bytes of scratch but the built-in "
            "area holds %zu; use sala_sparse_decode with a caller-provided workspace",
            need, kNoallocScratchBytes);
        return SALA_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    sala_status s = scratch_on_current_device(&scratch);
    if (s != SALA_OK) return s;
    return sala::sparse_decode_impl(q, kcache, vcache, kbar, idx_in, idx_out, o, B, H, Hkv, pos,
                                    Tmax, nb_cap, d, block, topk, n_init, n_local, scale, scratch,
                                    kNoallocScratchBytes, dt, stream, /*zero_barrier=*/true,
                                    /*pdl=*/false);
}
