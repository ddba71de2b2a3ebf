// CUDA-core pieces of the sparse attention backward (the tensor-core passes are in
// sparse_bwd_tc.cu).  With the selection held fixed, o_i = sum_j P_ij v_j over the visible keys,
// P_ij = exp(scale q_i.k_j - lse_i), and for the upstream gradient do:
//   dP_ij = do_i . v_j,   D_i = sum_j P_ij dP_ij (= do_i . o_i),   dS_ij = P_ij (dP_ij - D_i)
//   dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij do_i
// where i runs over the query rows of the KV group's G heads.
//
//   * the transposed selection (CSR): for every (batch, KV group, key block j) the query tokens
//     whose selection holds j, so the dk / dv pass can walk key blocks and gather their rows;
//   * finish: dk = scale * dk_acc and dv = dv_acc rounded to bf16 (the dk / dv pass adds fp32
//     partial sums into dk_acc, dv_acc).
#include <algorithm>

#include "kernels.h"

namespace sala {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------------- CSR
// Entry e of the traversal is (slot s, row) with rows consecutive within a warp, so the forced
// blocks (the same for neighbouring tokens) aggregate into one atomic per warp.  An entry is
// listed when it is a block id (>= 0) that is not in the future of its token, below nb, and not a
// repeat of the previous slot (rows are ascending); anything else but padding is flagged.
__device__ __forceinline__ int csr_key(const int32_t* __restrict__ idx, int64_t row, int s, int N,
                                       int slots, int nb, const DevCtx& ctx) {
    const int32_t* r = idx + row * slots;
    const int v = __ldg(r + s);
    if (v < 0) return -1;
    const int i = (int)(row % N);
    if (v >= nb || v > i / 64 || (s > 0 && __ldg(r + s - 1) >= v)) {
        flag(ctx, kStatusBounds);
        return -1;
    }
    return (int)((row / N) * nb + v);
}

__global__ void __launch_bounds__(kThreads)
csr_count_kernel(const int32_t* __restrict__ idx, int* __restrict__ cnt, int64_t rows, int N,
                 int slots, int nb, DevCtx ctx) {
    const int64_t total = rows * slots;
    for (int64_t e = blockIdx.x * (int64_t)kThreads + threadIdx.x; e - threadIdx.x % 32 < total;
         e += (int64_t)gridDim.x * kThreads) {
        const bool in = e < total;
        const int key = in ? csr_key(idx, e % rows, (int)(e / rows), N, slots, nb, ctx) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(cnt + key, __popc(peers));
    }
}

__global__ void __launch_bounds__(kThreads)
csr_fill_kernel(const int32_t* __restrict__ idx, const int* __restrict__ off, int* __restrict__ cur,
                int* __restrict__ list, int64_t rows, int N, int slots, int nb, DevCtx ctx) {
    const int64_t total = rows * slots;
    const int lane = threadIdx.x & 31;
    for (int64_t e = blockIdx.x * (int64_t)kThreads + threadIdx.x; e - lane < total;
         e += (int64_t)gridDim.x * kThreads) {
        const bool in = e < total;
        const int64_t row = in ? e % rows : 0;
        const int key = in ? csr_key(idx, row, (int)(e / rows), N, slots, nb, ctx) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const int leader = __ffs(peers) - 1;
        int base = 0;
        if (key >= 0 && lane == leader) base = atomicAdd(cur + key, __popc(peers));
        base = __shfl_sync(peers, base, leader);
        if (key >= 0) list[off[key] + base + __popc(peers & ((1u << lane) - 1u))] = (int)(row % N);
    }
}

// Exclusive prefix sum of cnt[0, n) into off[0, n], one CTA (n is a few thousand keys).
__global__ void __launch_bounds__(1024) csr_scan_kernel(const int* __restrict__ cnt,
                                                        int* __restrict__ off, int n) {
    __shared__ int part[1024];
    const int t = threadIdx.x;
    const int per = (n + 1023) / 1024;
    const int a = min(n, t * per), b = min(n, a + per);
    int s = 0;
    for (int k = a; k < b; ++k) s += cnt[k];
    part[t] = s;
    __syncthreads();
    for (int w = 1; w < 1024; w <<= 1) {
        const int x = t >= w ? part[t - w] : 0;
        __syncthreads();
        part[t] += x;
        __syncthreads();
    }
    int run = t > 0 ? part[t - 1] : 0;
    for (int k = a; k < b; ++k) {
        off[k] = run;
        run += cnt[k];
    }
    if (t == 1023) off[n] = part[1023];
}

// ---------------------------------------------------------------------------------- finish
__global__ void __launch_bounds__(kThreads)
finish_kernel(const float4* __restrict__ dk_acc, const float4* __restrict__ dv_acc,
              uint2* __restrict__ dk, uint2* __restrict__ dv, int64_t n4, float scale) {
    for (int64_t e = blockIdx.x * (int64_t)kThreads + threadIdx.x; e < n4;
         e += (int64_t)gridDim.x * kThreads) {
        const float4 a = __ldcs(dk_acc + e), b = __ldcs(dv_acc + e);
        dk[e] = make_uint2(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale));
        dv[e] = make_uint2(pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
    }
}

}  // namespace

SparseBwdCsr sparse_bwd_csr_layout(void* ws, int B, int Hkv, int N, int slots) {
    const int nb = (N + 63) / 64;
    const int64_t n_keys = (int64_t)B * Hkv * nb;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t o_cur = up(n_keys * 4), o_off = o_cur + up(n_keys * 4);
    const size_t o_list = o_off + up((n_keys + 1) * 4);
    const uintptr_t base = reinterpret_cast<uintptr_t>(ws);
    SparseBwdCsr c;
    c.nb = nb;
    c.n_keys = (int)n_keys;
    c.cnt = reinterpret_cast<int*>(base);
    c.cur = reinterpret_cast<int*>(base + o_cur);
    c.off = reinterpret_cast<int*>(base + o_off);
    c.list = reinterpret_cast<int*>(base + o_list);
    c.bytes = o_list + up((size_t)B * Hkv * N * slots * 4);
    return c;
}

cudaError_t launch_sparse_bwd_csr(const int32_t* idx, int B, int Hkv, int N, int slots,
                                  const SparseBwdCsr& c, cudaStream_t st, DevCtx ctx) {
    cudaError_t e = cudaMemsetAsync(c.cnt, 0, (size_t)c.n_keys * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(c.cur, 0, (size_t)c.n_keys * 4, st);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * Hkv * N;
    const int64_t blocks = std::min<int64_t>((rows * slots + kThreads - 1) / kThreads, 148 * 16);
    csr_count_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(idx, c.cnt, rows, N, slots, c.nb, ctx);
    csr_scan_kernel<<<1, 1024, 0, st>>>(c.cnt, c.off, c.n_keys);
    csr_fill_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(idx, c.off, c.cur, c.list, rows, N,
                                                          slots, c.nb, ctx);
    return cudaGetLastError();
}

cudaError_t launch_sparse_bwd_finish(const float* dk_acc, const float* dv_acc, void* dk, void* dv,
                                     int64_t n, float scale, cudaStream_t st) {
    const int64_t n4 = n / 4;
    if (n4 == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n4 + kThreads - 1) / kThreads, 148 * 8);
    finish_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(
        reinterpret_cast<const float4*>(dk_acc), reinterpret_cast<const float4*>(dv_acc),
        static_cast<uint2*>(dk), static_cast<uint2*>(dv), n4, scale);
    return cudaGetLastError();
}

}  // namespace sala
