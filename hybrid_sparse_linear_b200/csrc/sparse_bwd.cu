// CUDA-core pieces of the sparse attention backward (the tensor-core passes are in
// sparse_bwd_tc.cu).  With the selection held fixed, o_i = sum_j P_ij v_j over the visible keys,
// P_ij = exp(scale q_i.k_j - lse_i), and for the upstream gradient do:
//   dP_ij = do_i . v_j,   D_i = sum_j P_ij dP_ij = do_i . o_i,   dS_ij = P_ij (dP_ij - D_i)
//   dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij do_i
// where i runs over the query rows of the KV group's G heads.
//
//   * delta: D_i = do_i . (o_i + o_lo_i) per query row (fp32).  D_i enters every dS_ij through
//     dP_ij - D_i, which cancels on peaked softmaxes, so it needs o far beyond bf16: the training
//     forward returns o's bf16 rounding residual o_lo (o + o_lo carries it to ~2^-16, its P V
//     having taken P as bf16 hi + lo);
//   * the transposed selection (CSR): for every (batch, KV group, chunk of kChunkTok query
//     tokens, key block j) the chunk's tokens whose selection holds j, so the dk / dv pass can
//     walk key blocks and gather their rows.  Keyed chunk-major, the lists laid end to end visit
//     one chunk's tokens at a time: the key side, whose CTAs take items of kItem list positions
//     in turn, then re-reads only that chunk's Q and dO rows (64 MiB for 16 heads), from L2;
//     each item's first key is recorded for it;
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

// ---------------------------------------------------------------------------------- delta
// Rows of 128 bf16: 16 lanes of 16 bytes per row, two rows per warp instruction, four such
// loads in flight per lane per tensor.  o + o_lo is exact in fp32 (at most 17 significant bits).
__global__ void __launch_bounds__(kThreads)
delta_kernel(const uint4* __restrict__ o, const uint4* __restrict__ o_lo,
             const uint4* __restrict__ dout, float* __restrict__ delta, int64_t rows) {
    constexpr int kU = 4;
    const int lane = threadIdx.x & 31, sub = lane >> 4, col = lane & 15;
    const int64_t warp = (blockIdx.x * (int64_t)kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t r0 = warp * 2 * kU; r0 < rows; r0 += n_warps * 2 * kU) {
        uint4 a[kU], b[kU], c[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t r = r0 + 2 * u + sub;
            a[u] = b[u] = c[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows) {
                a[u] = __ldcs(o + r * 16 + col);
                b[u] = __ldcs(dout + r * 16 + col);
                if (o_lo != nullptr) c[u] = __ldcs(o_lo + r * 16 + col);
            }
        }
        float s[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const uint32_t x[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
            const uint32_t y[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
            const uint32_t z[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float o0 = __uint_as_float(x[e] << 16) + __uint_as_float(z[e] << 16);
                const float o1 = __uint_as_float(x[e] & 0xffff0000u) + __uint_as_float(z[e] & 0xffff0000u);
                acc = fmaf(o0, __uint_as_float(y[e] << 16), acc);
                acc = fmaf(o1, __uint_as_float(y[e] & 0xffff0000u), acc);
            }
            s[u] = acc;
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1)
#pragma unroll
            for (int u = 0; u < kU; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], off);
        if (col == 0) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int64_t r = r0 + 2 * u + sub;
                if (r < rows) delta[r] = s[u];
            }
        }
    }
}

// ---------------------------------------------------------------------------------- CSR
// Entry e of the traversal is (slot s, row) with rows consecutive within a warp, so the forced
// blocks (the same for neighbouring tokens) aggregate into one atomic per warp.  An entry is
// listed when it is a block id (>= 0) that is not in the future of its token, below nb, and not a
// repeat of the previous slot (rows are ascending); anything else but padding is flagged.
__device__ __forceinline__ int csr_key(const int32_t* __restrict__ idx, int64_t row, int s, int N,
                                       int slots, int nb, int n_chunks, const DevCtx& ctx) {
    const int32_t* r = idx + row * slots;
    const int v = __ldg(r + s);
    if (v < 0) return -1;
    const int i = (int)(row % N);
    if (v >= nb || v > i / 64 || (s > 0 && __ldg(r + s - 1) >= v)) {
        flag(ctx, kStatusBounds);
        return -1;
    }
    return (int)(((row / N) * n_chunks + i / kChunkTok) * nb + v);
}

__global__ void __launch_bounds__(kThreads)
csr_count_kernel(const int32_t* __restrict__ idx, int* __restrict__ cnt, int64_t rows, int N,
                 int slots, int nb, int n_chunks, DevCtx ctx) {
    const int64_t total = rows * slots;
    for (int64_t e = blockIdx.x * (int64_t)kThreads + threadIdx.x; e - threadIdx.x % 32 < total;
         e += (int64_t)gridDim.x * kThreads) {
        const bool in = e < total;
        const int key = in ? csr_key(idx, e % rows, (int)(e / rows), N, slots, nb, n_chunks, ctx) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(cnt + key, __popc(peers));
    }
}

__global__ void __launch_bounds__(kThreads)
csr_fill_kernel(const int32_t* __restrict__ idx, const int* __restrict__ off, int* __restrict__ cur,
                int* __restrict__ list, int64_t rows, int N, int slots, int nb, int n_chunks,
                DevCtx ctx) {
    const int64_t total = rows * slots;
    const int lane = threadIdx.x & 31;
    for (int64_t e = blockIdx.x * (int64_t)kThreads + threadIdx.x; e - lane < total;
         e += (int64_t)gridDim.x * kThreads) {
        const bool in = e < total;
        const int64_t row = in ? e % rows : 0;
        const int key = in ? csr_key(idx, row, (int)(e / rows), N, slots, nb, n_chunks, ctx) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const int leader = __ffs(peers) - 1;
        int base = 0;
        if (key >= 0 && lane == leader) base = atomicAdd(cur + key, __popc(peers));
        base = __shfl_sync(peers, base, leader);
        if (key >= 0) list[off[key] + base + __popc(peers & ((1u << lane) - 1u))] = (int)(row % N);
    }
}

// Exclusive prefix sum of cnt[0, n) into off[0, n]: blocks of 4096 keys scanned locally (their
// totals to bsum), the totals scanned by one CTA, then added back.
constexpr int kScanBlock = 4096;

__device__ __forceinline__ int block_excl_scan(int v, int* sh) {  // 1024 threads
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[w] = x;
    __syncthreads();
    if (w == 0) {
        int z = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        sh[lane] = z;
    }
    __syncthreads();
    const int r = (w > 0 ? sh[w - 1] : 0) + x - v;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(1024) scan_blocks_kernel(const int* __restrict__ cnt,
                                                           int* __restrict__ off,
                                                           int* __restrict__ bsum, int n) {
    __shared__ int sh[32];
    const int base = blockIdx.x * kScanBlock + threadIdx.x * 4;
    int v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = base + u < n ? cnt[base + u] : 0;
    const int tot = v[0] + v[1] + v[2] + v[3];
    int run = block_excl_scan(tot, sh);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (base + u < n) off[base + u] = run;
        run += v[u];
    }
    if (threadIdx.x == 1023) bsum[blockIdx.x] = run;
}

__global__ void __launch_bounds__(1024) scan_top_kernel(int* __restrict__ bsum, int nblk,
                                                        int* __restrict__ total) {
    __shared__ int sh[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int b0 = 0; b0 < nblk; b0 += 1024) {
        const int i = b0 + threadIdx.x;
        const int v = i < nblk ? bsum[i] : 0;
        const int e = block_excl_scan(v, sh) + carry;
        if (i < nblk) bsum[i] = e;
        __syncthreads();
        if (threadIdx.x == 1023) carry = e + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) *total = carry;
}

__global__ void __launch_bounds__(256) scan_add_kernel(int* __restrict__ off,
                                                       const int* __restrict__ bsum, int n) {
    for (int k = blockIdx.x * 256 + threadIdx.x; k < n; k += gridDim.x * 256)
        off[k] += bsum[k / kScanBlock];
}

// item_key[it] = the list holding position it * kItem: the last key with off[key] <= position
// (a non-empty list, as off[key + 1] > position then).  Items past the total are not read.
__global__ void __launch_bounds__(256) csr_items_kernel(const int* __restrict__ off, int n_keys,
                                                        int* __restrict__ item_key, int n_items) {
    const int64_t T = off[n_keys];
    for (int it = blockIdx.x * 256 + threadIdx.x; it < n_items; it += gridDim.x * 256) {
        const int64_t t0 = (int64_t)it * kItem;
        if (t0 >= T) break;
        int lo = 0, hi = n_keys - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= t0) lo = mid;
            else hi = mid - 1;
        }
        item_key[it] = lo;
    }
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
    const int n_chunks = (N + kChunkTok - 1) / kChunkTok;
    const int64_t n_keys = (int64_t)B * Hkv * n_chunks * nb;
    const int64_t n_entries = (int64_t)B * Hkv * N * slots;
    const int64_t n_items = (n_entries + kItem - 1) / kItem;
    const int64_t n_blk = (n_keys + kScanBlock - 1) / kScanBlock;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t o_cur = up(n_keys * 4), o_off = o_cur + up(n_keys * 4);
    const size_t o_list = o_off + up((n_keys + 1) * 4);
    const size_t o_items = o_list + up((size_t)n_entries * 4);
    const size_t o_bsum = o_items + up((size_t)n_items * 4);
    const uintptr_t base = reinterpret_cast<uintptr_t>(ws);
    SparseBwdCsr c;
    c.nb = nb;
    c.n_chunks = n_chunks;
    c.n_keys = (int)n_keys;
    c.n_items = (int)n_items;
    c.cnt = reinterpret_cast<int*>(base);
    c.cur = reinterpret_cast<int*>(base + o_cur);
    c.off = reinterpret_cast<int*>(base + o_off);
    c.list = reinterpret_cast<int*>(base + o_list);
    c.item_key = reinterpret_cast<int*>(base + o_items);
    c.bsum = reinterpret_cast<int*>(base + o_bsum);
    c.bytes = o_bsum + up((size_t)n_blk * 4);
    return c;
}

cudaError_t launch_sparse_bwd_delta(const void* o, const void* o_lo, const void* dout,
                                    float* delta, int64_t rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    // one wave of resident blocks, the rows striding over it (any positive count is correct)
    static std::atomic<int> wave_cache{0};
    int wave = wave_cache.load(std::memory_order_relaxed);
    if (!wave) {
        int per_sm = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, delta_kernel, kThreads, 0);
        wave = std::max(1, device_sm_count() * std::max(1, per_sm));
        wave_cache.store(wave, std::memory_order_relaxed);
    }
    const int64_t blocks = std::min<int64_t>((rows + 63) / 64, wave);
    delta_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(static_cast<const uint4*>(o),
                                                        static_cast<const uint4*>(o_lo),
                                                        static_cast<const uint4*>(dout), delta, rows);
    return cudaGetLastError();
}

cudaError_t launch_sparse_bwd_csr(const int32_t* idx, int B, int Hkv, int N, int slots,
                                  const SparseBwdCsr& c, cudaStream_t st, DevCtx ctx) {
    cudaError_t e = cudaMemsetAsync(c.cnt, 0, (size_t)c.n_keys * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(c.cur, 0, (size_t)c.n_keys * 4, st);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)B * Hkv * N;
    const int64_t blocks = std::min<int64_t>((rows * slots + kThreads - 1) / kThreads, 148 * 16);
    csr_count_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(idx, c.cnt, rows, N, slots, c.nb,
                                                           c.n_chunks, ctx);
    const int n_blk = (c.n_keys + kScanBlock - 1) / kScanBlock;
    scan_blocks_kernel<<<n_blk, 1024, 0, st>>>(c.cnt, c.off, c.bsum, c.n_keys);
    scan_top_kernel<<<1, 1024, 0, st>>>(c.bsum, n_blk, c.off + c.n_keys);
    scan_add_kernel<<<std::min(n_blk * 16, 148 * 8), 256, 0, st>>>(c.off, c.bsum, c.n_keys);
    csr_fill_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(idx, c.off, c.cur, c.list, rows, N,
                                                          slots, c.nb, c.n_chunks, ctx);
    csr_items_kernel<<<std::min((c.n_items + 255) / 256, 148 * 4), 256, 0, st>>>(
        c.off, c.n_keys, c.item_key, c.n_items);
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
