// QK normalisation: every head row of q and of k divided by its root mean square,
//   y_c = x_c / sqrt((1/d) sum_e x_e^2 + eps),
// with no learned scale (MiniCPM-SALA summaries, DE section 2 "additional improvements": queries
// and keys are normalised to keep the activations stable).  The layer applies it before RoPE,
// block compression and selection.
//
// HBM-bound: each row is read once and written once (4 d bytes per bf16 row).  Each lane moves
// 16 bytes per access, a row spans d * sizeof(T) / 16 lanes (16 for bf16 d = 128), so one warp
// instruction covers two to four whole rows and each lane keeps four such loads in flight
// (2 KB per warp) to cover the DRAM latency.  The squares are summed in fp32 (per lane, then a
// butterfly over the row's lanes).  q and k go through
// one launch, rows [0, nq) from q and [nq, nq + nk) from k, so a decode step pays one launch.
// Output may alias input exactly (in place): each element is read and written by the same lane.
//
// The same pass can also rotate q and k by position (RoPE, the linear layers' half of HyPE), so
// a linear layer's prologue costs one read and one write of q and k: rows are [B, heads, N, d]
// flattened, row r at position pos0 + r % N; the rotate-half partner of a lane's elements sits
// in the lane kL/2 away within the row's lanes (one shuffle per 32-bit word).  The norm comes
// first (a rotation keeps every pair's length, so the two commute up to rounding).  Angles are
// reduced in turns in double (rope.cuh) before the fp32 sine and cosine.
#include <algorithm>

#include "kernels.h"
#include "rope.cuh"

namespace sala {
namespace {

constexpr int kThreads = 256;
constexpr int kU = 4;  // 16-byte loads in flight per lane

struct alignas(16) Vec16 {
    uint4 u;
};

template <typename T>
__device__ __forceinline__ void unpack(const uint4& u, float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void unpack<float>(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
template <>
__device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack(const float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ uint4 pack<float>(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
template <>
__device__ __forceinline__ uint4 pack<__nv_bfloat16>(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Lane layout: a row is d * sizeof(T) / 16 lanes of 16 bytes (8 bf16 or 4 fp32 elements), so
// one warp instruction covers 32 / that many consecutive rows; kU such instructions per lane are
// in flight before the first reduction.  The squares' sum is a butterfly inside the row's lanes.
template <typename T, int D, bool kNorm, bool kRope>
__global__ void __launch_bounds__(kThreads, kRope ? 2 : 4)
qk_norm_kernel(const T* xq, T* yq, int64_t nq, const T* xk, T* yk, int64_t nk, float eps, int N,
               int64_t pos0, double base) {
    constexpr int kE = 16 / (int)sizeof(T);  // elements per lane
    constexpr int kL = D / kE;               // lanes per row
    constexpr int kRPI = 32 / kL;            // rows per warp instruction
    constexpr int kRPW = kRPI * kU;          // rows per warp iteration
    const int lane = threadIdx.x & 31;
    const int sub = lane / kL, col = (lane % kL) * kE;
    // RoPE: this lane's frequencies (turns per position) and the side of its pairs
    double turn[kRope ? kE : 1];
    const bool upper = col >= D / 2;
    if constexpr (kRope) {
#pragma unroll
        for (int e = 0; e < kE; ++e) turn[e] = rope_turn(base, (col + e) % (D / 2), D);
    }
    const int64_t warp = (blockIdx.x * (int64_t)kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t total = nq + nk;
    for (int64_t r0 = warp * kRPW; r0 < total; r0 += n_warps * kRPW) {
        uint4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t r = r0 + u * kRPI + sub;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < total) {
                const T* src = r < nq ? xq + r * D : xk + (r - nq) * D;
                v[u] = reinterpret_cast<const Vec16*>(src + col)->u;
            }
        }
        float ss[kU];
        if constexpr (kNorm) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                float f[kE];
                unpack<T>(v[u], f);
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < kE; ++e) s = fmaf(f[e], f[e], s);
                ss[u] = s;
            }
#pragma unroll
            for (int off = kL / 2; off > 0; off >>= 1)
#pragma unroll
                for (int u = 0; u < kU; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t r = r0 + u * kRPI + sub;
            float f[kE];
            unpack<T>(v[u], f);
            if constexpr (kNorm) {
                const float inv = rsqrtf(ss[u] * (1.f / D) + eps);
#pragma unroll
                for (int e = 0; e < kE; ++e) f[e] *= inv;
            }
            if constexpr (kRope) {
                // partner values from the lane kL/2 away (all lanes take part in the shuffle)
                float g[kE];
#pragma unroll
                for (int e = 0; e < kE; ++e) g[e] = __shfl_xor_sync(0xffffffffu, f[e], kL / 2);
                const int64_t p = pos0 + (r < nq ? r : r - nq) % N;
#pragma unroll
                for (int e = 0; e < kE; ++e) {
                    float c, sn;
                    rope_cs(turn[e], p, c, sn);
                    // lower half: x c - x_hi s;  upper half: x c + x_lo s
                    f[e] = upper ? fmaf(g[e], sn, f[e] * c) : fmaf(-g[e], sn, f[e] * c);
                }
            }
            if (r < total) {
                T* dst = r < nq ? yq + r * D : yk + (r - nq) * D;
                reinterpret_cast<Vec16*>(dst + col)->u = pack<T>(f);
            }
        }
    }
}

// RoPE variants: a lane holds both halves of its pairs -- a 16-byte chunk of elements
// [c, c + kE) and the chunk [c + d/2, c + d/2 + kE) -- so each pair's sine and cosine is formed
// once and no lane exchange is needed; a row spans d/2 * sizeof(T) / 16 lanes (8 for bf16,
// d = 128).
template <typename T, int D, bool kNorm>
__global__ void __launch_bounds__(kThreads, 3)
qk_rope_kernel(const T* xq, T* yq, int64_t nq, const T* xk, T* yk, int64_t nk, float eps, int N,
               int64_t pos0, double base) {
    constexpr int kE = 16 / (int)sizeof(T);  // elements per chunk
    constexpr int kL = (D / 2) / kE;         // lanes per row
    constexpr int kRPI = 32 / kL;            // rows per warp instruction
    constexpr int kV = 2;                    // row groups in flight per lane
    constexpr int kRPW = kRPI * kV;
    const int lane = threadIdx.x & 31;
    const int sub = lane / kL, col = (lane % kL) * kE;
    double turn[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) turn[e] = rope_turn(base, col + e, D);
    const int64_t warp = (blockIdx.x * (int64_t)kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t total = nq + nk;
    for (int64_t r0 = warp * kRPW; r0 < total; r0 += n_warps * kRPW) {
        uint4 lo[kV], hi[kV];
#pragma unroll
        for (int u = 0; u < kV; ++u) {
            const int64_t r = r0 + u * kRPI + sub;
            lo[u] = hi[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < total) {
                const T* src = r < nq ? xq + r * D : xk + (r - nq) * D;
                lo[u] = reinterpret_cast<const Vec16*>(src + col)->u;
                hi[u] = reinterpret_cast<const Vec16*>(src + col + D / 2)->u;
            }
        }
#pragma unroll
        for (int u = 0; u < kV; ++u) {
            const int64_t r = r0 + u * kRPI + sub;
            float a[kE], b[kE];
            unpack<T>(lo[u], a);
            unpack<T>(hi[u], b);
            if constexpr (kNorm) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < kE; ++e) ss = fmaf(b[e], b[e], fmaf(a[e], a[e], ss));
#pragma unroll
                for (int off = kL / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = rsqrtf(ss * (1.f / D) + eps);
#pragma unroll
                for (int e = 0; e < kE; ++e) {
                    a[e] *= inv;
                    b[e] *= inv;
                }
            }
            const int64_t p = pos0 + (r < nq ? r : r - nq) % N;
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                float c, sn;
                rope_cs(turn[e], p, c, sn);
                rope_rot(a[e], b[e], c, sn);
            }
            if (r < total) {
                T* dst = r < nq ? yq + r * D : yk + (r - nq) * D;
                reinterpret_cast<Vec16*>(dst + col)->u = pack<T>(a);
                reinterpret_cast<Vec16*>(dst + col + D / 2)->u = pack<T>(b);
            }
        }
    }
}

template <typename T, int D, bool kNorm, bool kRope>
cudaError_t launch_qn(const void* q, void* qo, int64_t nq, const void* k, void* ko, int64_t nk,
                      float eps, int N, int64_t pos0, double base, cudaStream_t st) {
    const int64_t total = nq + nk;
    if (total == 0) return cudaSuccess;
    constexpr int64_t kRowsPerBlock = (kThreads / 32) * (32 / (D * (int)sizeof(T) / 16)) * kU;
    // one wave: the SMs times the blocks resident per SM, the rows striding over it
    // (any positive count is correct: it only sizes the grid)
    static std::atomic<int> wave_cache{0};
    int wave = wave_cache.load(std::memory_order_relaxed);
    if (!wave) {
        const int n_sm = device_sm_count();
        int per_sm = 0;
        if constexpr (kRope)
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qk_rope_kernel<T, D, kNorm>,
                                                          kThreads, 0);
        else
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qk_norm_kernel<T, D, kNorm, false>,
                                                          kThreads, 0);
        wave = std::max(1, n_sm * std::max(1, per_sm));
        wave_cache.store(wave, std::memory_order_relaxed);
    }
    const int64_t blocks = std::min<int64_t>((total + kRowsPerBlock - 1) / kRowsPerBlock, wave);
    if constexpr (kRope)
        qk_rope_kernel<T, D, kNorm><<<(unsigned)blocks, kThreads, 0, st>>>(
            static_cast<const T*>(q), static_cast<T*>(qo), nq, static_cast<const T*>(k),
            static_cast<T*>(ko), nk, eps, N, pos0, base);
    else
        qk_norm_kernel<T, D, kNorm, false><<<(unsigned)blocks, kThreads, 0, st>>>(
            static_cast<const T*>(q), static_cast<T*>(qo), nq, static_cast<const T*>(k),
            static_cast<T*>(ko), nk, eps, N, pos0, base);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_pick(const void* q, void* qo, int64_t nq, const void* k, void* ko, int64_t nk,
                        float eps, int N, int64_t pos0, double base, cudaStream_t st) {
    const bool norm = eps > 0.f, rope = base > 0.0;
    if (norm && rope) return launch_qn<T, D, true, true>(q, qo, nq, k, ko, nk, eps, N, pos0, base, st);
    if (norm) return launch_qn<T, D, true, false>(q, qo, nq, k, ko, nk, eps, N, pos0, base, st);
    if (rope) return launch_qn<T, D, false, true>(q, qo, nq, k, ko, nk, eps, N, pos0, base, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_qk_prologue(DType dt, const void* q, void* q_out, int64_t q_rows, const void* k,
                               void* k_out, int64_t k_rows, int d, float eps, int N, int64_t pos0,
                               double rope_base, cudaStream_t st) {
    if (dt == DType::F32)
        return d == 64 ? launch_pick<float, 64>(q, q_out, q_rows, k, k_out, k_rows, eps, N, pos0, rope_base, st)
                       : launch_pick<float, 128>(q, q_out, q_rows, k, k_out, k_rows, eps, N, pos0, rope_base, st);
    return d == 64 ? launch_pick<__nv_bfloat16, 64>(q, q_out, q_rows, k, k_out, k_rows, eps, N, pos0, rope_base, st)
                   : launch_pick<__nv_bfloat16, 128>(q, q_out, q_rows, k, k_out, k_rows, eps, N, pos0, rope_base, st);
}

cudaError_t launch_qk_norm(DType dt, const void* q, void* q_out, int64_t q_rows, const void* k,
                           void* k_out, int64_t k_rows, int d, float eps, cudaStream_t st) {
    return launch_qk_prologue(dt, q, q_out, q_rows, k, k_out, k_rows, d, eps, 1, 0, 0.0, st);
}

}  // namespace sala
