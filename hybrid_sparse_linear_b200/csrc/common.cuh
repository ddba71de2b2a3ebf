// Internal helpers shared by the CUDA kernels of libsala (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace sala {

// Bits of the per-device status word (read and cleared by sala_check_status).
enum : unsigned { kStatusTimeout = 1u, kStatusBounds = 2u };

// Passed by value to every kernel: where to record device-side faults, and how long a bounded
// wait may spin before it gives up.
struct DevCtx {
    unsigned* status;
    unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void flag(const DevCtx& c, unsigned bits) { atomicOr(c.status, bits); }

// Index checks of the debug build (compiled with -DSALA_DEBUG_BOUNDS into libsala_debug.so):
// in_bounds(c, ok) records kStatusBounds when ok is false and returns ok, so the caller skips the
// access instead of making it; the release build folds it to true and emits nothing.
#ifdef SALA_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool in_bounds(const DevCtx& c, bool ok) {
    if constexpr (kDebugBounds) {
        if (!ok) flag(c, kStatusBounds);
        return ok;
    } else {
        (void)c;
        (void)ok;
        return true;
    }
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Correct rounding of an fp64 value to the element type: fp32 directly (round to nearest
// even); bf16 through round-to-odd at fp32 followed by round-to-nearest-even at bf16, which is
// exact-once rounding because fp32 carries more than two extra bits (Boldo & Melquiond,
// "Emulation of FMA and correctly rounded sums: proved algorithms using rounding to odd").
template <typename T> __device__ __forceinline__ T round_from_double(double x);
template <> __device__ __forceinline__ float round_from_double<float>(double x) {
    return __double2float_rn(x);
}
template <> __device__ __forceinline__ __nv_bfloat16 round_from_double<__nv_bfloat16>(double x) {
    float f = __double2float_rz(x);
    if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __float2bfloat16_rn(f);
}

// Monotone map of fp32 to uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t orderable(float s) {
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Selection key: higher score first, then lower block index.  Key 0 means "empty".
__device__ __forceinline__ uint64_t sel_key(float score, int blk) {
    return ((uint64_t)orderable(score) << 32) | (uint32_t)(~(uint32_t)blk);
}
__device__ __forceinline__ int key_block(uint64_t key) { return (int)(~(uint32_t)(key & 0xffffffffu)); }

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The current device's SM count, read once per device (any host thread may call it; a failed
// query counts as a B200's 148).
inline int device_sm_count() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> cache[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Raises a kernel's dynamic shared memory limit once per device, so later launches (including
// ones recorded into a CUDA graph) only enqueue work.
template <auto Kern>
cudaError_t ensure_smem(int bytes) {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

}  // namespace sala
