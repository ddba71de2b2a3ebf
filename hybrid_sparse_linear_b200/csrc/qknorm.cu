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
#include <algorithm>

#include "kernels.h"

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
template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 4)
qk_norm_kernel(const T* xq, T* yq, int64_t nq, const T* xk, T* yk, int64_t nk, float eps) {
    constexpr int kE = 16 / (int)sizeof(T);  // elements per lane
    constexpr int kL = D / kE;               // lanes per row
    constexpr int kRPI = 32 / kL;            // rows per warp instruction
    constexpr int kRPW = kRPI * kU;          // rows per warp iteration
    const int lane = threadIdx.x & 31;
    const int sub = lane / kL, col = (lane % kL) * kE;
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
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t r = r0 + u * kRPI + sub;
            if (r < total) {
                const float inv = rsqrtf(ss[u] * (1.f / D) + eps);
                float f[kE];
                unpack<T>(v[u], f);
#pragma unroll
                for (int e = 0; e < kE; ++e) f[e] *= inv;
                T* dst = r < nq ? yq + r * D : yk + (r - nq) * D;
                reinterpret_cast<Vec16*>(dst + col)->u = pack<T>(f);
            }
        }
    }
}

template <typename T, int D>
cudaError_t launch_qn(const void* q, void* qo, int64_t nq, const void* k, void* ko, int64_t nk,
                      float eps, cudaStream_t st) {
    const int64_t total = nq + nk;
    if (total == 0) return cudaSuccess;
    constexpr int64_t kRowsPerBlock = (kThreads / 32) * (32 / (D * (int)sizeof(T) / 16)) * kU;
    // one wave: the SMs times the blocks resident per SM, the rows striding over it
    static int wave = 0;
    if (!wave) {
        int dev = 0, n_sm = 0, per_sm = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qk_norm_kernel<T, D>, kThreads, 0);
        wave = std::max(1, n_sm * std::max(1, per_sm));
    }
    const int64_t blocks = std::min<int64_t>((total + kRowsPerBlock - 1) / kRowsPerBlock, wave);
    qk_norm_kernel<T, D><<<(unsigned)blocks, kThreads, 0, st>>>(
        static_cast<const T*>(q), static_cast<T*>(qo), nq, static_cast<const T*>(k),
        static_cast<T*>(ko), nk, eps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_norm(DType dt, const void* q, void* q_out, int64_t q_rows, const void* k,
                           void* k_out, int64_t k_rows, int d, float eps, cudaStream_t st) {
    if (dt == DType::F32)
        return d == 64 ? launch_qn<float, 64>(q, q_out, q_rows, k, k_out, k_rows, eps, st)
                       : launch_qn<float, 128>(q, q_out, q_rows, k, k_out, k_rows, eps, st);
    return d == 64 ? launch_qn<__nv_bfloat16, 64>(q, q_out, q_rows, k, k_out, k_rows, eps, st)
                   : launch_qn<__nv_bfloat16, 128>(q, q_out, q_rows, k, k_out, k_rows, eps, st);
}

}  // namespace sala
