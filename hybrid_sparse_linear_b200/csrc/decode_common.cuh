// Device helpers shared by the sparse decode kernels: a bounded grid-wide barrier on one word of
// global memory, a warp sort of 64 ints, and the warp-level bf16 tensor-core tile (m16n8k16) with
// its shared-memory fragment loaders.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace sala {
namespace dec {

// Grid-wide barrier for a cooperative launch on one 32-bit word: arrivals of the current barrier
// in the low 16 bits (zero between barriers), a generation count above.  The arrival's atomic
// returns the generation it belongs to; the last arrival clears the count and bumps the generation
// in one atomic.  Returns false after a timeout.  Ordering: the block barrier orders every thread's
// writes before thread 0's arrival, an acquire-release atomic (the arrivals form one release
// sequence), so the last arrival's release of the bump carries all CTAs' writes to each waiter's
// acquire load; no full fence is needed on either side.
__device__ __forceinline__ bool grid_barrier(unsigned* word, unsigned nblocks, const DevCtx& ctx, int* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        unsigned old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(word) : "memory");
        if ((old & 0xFFFFu) == nblocks - 1) {
            asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(word), "r"(0x10000u - nblocks)
                         : "memory");
        } else {
            const unsigned g0 = old >> 16;
            const uint64_t t0 = globaltimer_ns();
            while (true) {
                unsigned v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(word) : "memory");
                if ((v >> 16) != g0) break;
                if (globaltimer_ns() - t0 > ctx.wait_limit_ns) {
                    flag(ctx, kStatusTimeout);
                    ok = 0;
                    break;
                }
            }
        }
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Ascending bitonic sort of 64 ints held two per lane (position 2*lane + j).
__device__ __forceinline__ void warp_sort64(int& x0, int& x1, int lane) {
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int s = k >> 1; s > 0; s >>= 1) {
            if (s == 1) {
                const bool asc = ((2 * lane) & k) == 0;
                const int lo = min(x0, x1), hi = max(x0, x1);
                x0 = asc ? lo : hi;
                x1 = asc ? hi : lo;
            } else {
                const int lm = s >> 1;
                const int y0 = __shfl_xor_sync(0xffffffffu, x0, lm);
                const int y1 = __shfl_xor_sync(0xffffffffu, x1, lm);
                const int p0 = 2 * lane, p1 = 2 * lane + 1;
                const bool asc0 = (p0 & k) == 0, low0 = (p0 & s) == 0;
                const bool asc1 = (p1 & k) == 0, low1 = (p1 & s) == 0;
                x0 = (low0 == asc0) ? min(x0, y0) : max(x0, y0);
                x1 = (low1 == asc1) ? min(x1, y1) : max(x1, y1);
            }
        }
    }
}

// Warp-level bf16 tensor-core tile (m16n8k16, fp32 accumulate) and its shared-memory loaders.
// Decode's products are 16 heads x 64 keys x d: far too small for the CTA-wide tensor-core path,
// but on CUDA cores they cost thousands of shared-memory loads per thread.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(a));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// 16-byte raw loads, converted later: issuing every load of a phase before the first conversion
// keeps them all in flight (converting each load as it arrives would serialize the round trips).
__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
}  // namespace dec
}  // namespace sala
