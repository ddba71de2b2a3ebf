// Block selection: group-summed query . block key scores, then a per-row top-k.
//
// For query row r at position p (block c = p / 64) of KV group g:
//   forced     = {0 .. n_init-1} U {c-n_local+1 .. c}
//   candidates = {n_init .. c-n_local}, score = (sum_{h in g} q_h) . kbar_j
//   selection  = forced U top_k(candidates), ties to the lower block index.
// When a row has at most k candidates the selection is every block 0 .. c.  Otherwise the
// forced blocks lie strictly below (init) and above (local) every candidate, so the ascending
// output is init ids, the sorted top-k ids, local ids, then -1 padding -- no merge needed.
//
// Top-k state: one warp per row keeps the best 64 keys sorted descending, two per lane
// (position 2*lane + j).  A key packs (orderable score, ~block) so that one unsigned compare
// orders by score and then by lower block index; key 0 is "empty".  Candidates are streamed;
// only those above the current k-th key are inserted (rank by two ballots, shift by one shuffle).
#include "kernels.h"

namespace sala {
namespace {

constexpr int kBlk = 64;
constexpr int kCap = 64;  // largest k the warp list holds

__device__ __forceinline__ uint64_t shfl64(uint64_t x, int src) {
    return __shfl_sync(0xffffffffu, x, src);
}

// Key at list position K-1 (the current k-th best), broadcast to the warp.
__device__ __forceinline__ uint64_t kth_key(uint64_t l0, uint64_t l1, int K) {
    const int src = (K - 1) >> 1;
    return shfl64(((K - 1) & 1) ? l1 : l0, src);
}

// Offer one key per lane to the warp's sorted list (capacity 64, keeps the best K).
__device__ __forceinline__ void warp_offer(uint64_t& l0, uint64_t& l1, uint64_t key, int K,
                                           int lane) {
    if (K <= 0) return;
    uint64_t thr = kth_key(l0, l1, K);
    bool take = key > thr;
    unsigned m = __ballot_sync(0xffffffffu, take);
    while (m) {
        const int src = __ffs(m) - 1;
        const uint64_t kn = shfl64(key, src);
        const int p = __popc(__ballot_sync(0xffffffffu, l0 > kn)) +
                      __popc(__ballot_sync(0xffffffffu, l1 > kn));
        const uint64_t prev1 = __shfl_up_sync(0xffffffffu, l1, 1);
        const int q0 = 2 * lane, q1 = 2 * lane + 1;
        const uint64_t n0 = q0 < p ? l0 : (q0 == p ? kn : prev1);
        const uint64_t n1 = q1 < p ? l1 : (q1 == p ? kn : l0);
        l0 = n0;
        l1 = n1;
        if (lane == src) take = false;
        thr = kth_key(l0, l1, K);
        m = __ballot_sync(0xffffffffu, take && key > thr);
    }
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

// Writes one row's selection (see the file comment).  ncand = number of candidates.
__device__ __forceinline__ void write_row(int32_t* out, int slots, int c, int ncand, int topk,
                                          int n_init, int n_local, uint64_t l0, uint64_t l1,
                                          int lane) {
    if (ncand <= topk) {
        for (int s = lane; s < slots; s += 32) out[s] = s <= c ? s : -1;
        return;
    }
    const int K = topk;
    int x0 = (2 * lane < K && l0) ? key_block(l0) : 0x7fffffff;
    int x1 = (2 * lane + 1 < K && l1) ? key_block(l1) : 0x7fffffff;
    warp_sort64(x0, x1, lane);
    for (int s = lane; s < n_init; s += 32) out[s] = s;
    if (2 * lane < K) out[n_init + 2 * lane] = x0;
    if (2 * lane + 1 < K) out[n_init + 2 * lane + 1] = x1;
    for (int t = lane; t < n_local; t += 32) out[n_init + K + t] = c - n_local + 1 + t;
    for (int s = n_init + K + n_local + lane; s < slots; s += 32) out[s] = -1;
}

// ---------------------------------------------------------------------------------------------
// Tiled path: one CTA = 64 query rows of one (batch, KV group), 8 warps x 8 rows.  Scores for a
// 64 x 64 (rows x candidates) tile come from an fp32 register-blocked product out of shared
// memory (transposed q-bar and kbar tiles), then each warp streams its rows' scores into the
// rows' top-k lists.
constexpr int kRT = 64, kCT = 64, kTThreads = 256;

template <int D>
struct TopkSmem {
    static constexpr int kQ = D * (kRT + 4), kK = D * (kCT + 4), kS = kRT * (kCT + 1);
    static constexpr size_t bytes = sizeof(float) * (kQ + kK + kS);
};

template <typename T, int D>
__global__ void __launch_bounds__(kTThreads)
topk_tiled_kernel(const T* __restrict__ q, const T* __restrict__ kbar, int32_t* __restrict__ idx,
                  int H, int Hkv, int Hs, int Nq, int q_pos0, int nb, int topk, int n_init,
                  int n_local, int slots) {
    extern __shared__ __align__(16) float smt[];
    float* QBt = smt;                          // [D][RT+4]  group-summed queries, transposed
    float* KBt = QBt + TopkSmem<D>::kQ;        // [D][CT+4]  block keys, transposed
    float* SC = KBt + TopkSmem<D>::kK;         // [RT][CT+1] scores
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Selection group bg = (b, g) of Hs per batch: the G = H / Hs query heads g*G .. g*G+G-1 are
    // summed and scored against the kbar of their KV head (Hs = Hkv: the KV group; Hs = H: one
    // head); idx rows are [B, Hs, Nq, slots].
    const int G = H / Hs;
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hs;
    const int g = (int)(bg % Hs);
    const int64_t kv_plane = b * Hkv + g / (Hs / Hkv);
    const int r0 = blockIdx.x * kRT;
    const int rend = min(Nq, r0 + kRT);

    for (int e = tid; e < kRT * D; e += kTThreads) {
        const int r = e / D, a = e % D;
        float s = 0.f;
        if (r0 + r < Nq)
            for (int hh = 0; hh < G; ++hh)
                s += to_f(q[((b * H + (int64_t)g * G + hh) * Nq + r0 + r) * D + a]);
        QBt[a * (kRT + 4) + r] = s;
    }

    const int c_last = (q_pos0 + rend - 1) / kBlk;
    const int cand_lo = n_init;
    int cand_hi = c_last - n_local;  // inclusive candidate range of the tile
    if (cand_hi - cand_lo + 1 <= topk) cand_hi = cand_lo - 1;  // every row takes all: no ranking

    uint64_t L0[8], L1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) L0[i] = L1[i] = 0ull;
    int lim[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + warp * 8 + i;
        lim[i] = r < Nq ? (q_pos0 + r) / kBlk - n_local : -1;
    }
    const int K = min(topk, kCap);

    const T* kb = kbar + kv_plane * (int64_t)nb * D;
    for (int j0 = cand_lo; j0 <= cand_hi; j0 += kCT) {
        __syncthreads();
        for (int e = tid; e < kCT * D; e += kTThreads) {
            const int c = e / D, a = e % D;
            KBt[a * (kCT + 4) + c] = (j0 + c <= cand_hi) ? to_f(kb[(int64_t)(j0 + c) * D + a]) : 0.f;
        }
        __syncthreads();
        {
            const int rr = (tid >> 4) * 4, cc = (tid & 15) * 4;
            float acc[4][4] = {};
#pragma unroll 4
            for (int a = 0; a < D; ++a) {
                const float4 qa = *reinterpret_cast<const float4*>(QBt + a * (kRT + 4) + rr);
                const float4 ka = *reinterpret_cast<const float4*>(KBt + a * (kCT + 4) + cc);
                const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
                const float kv[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) SC[(rr + i) * (kCT + 1) + cc + j] = acc[i][j];
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int rl = warp * 8 + i;
            if (lim[i] - n_init + 1 <= topk) continue;  // every candidate taken: no ranking
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int cidx = half * 32 + lane;
                const int blk = j0 + cidx;
                const uint64_t key = (blk <= lim[i]) ? sel_key(SC[rl * (kCT + 1) + cidx], blk) : 0ull;
                warp_offer(L0[i], L1[i], key, K, lane);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + warp * 8 + i;
        if (r >= Nq) continue;
        const int c = (q_pos0 + r) / kBlk;
        write_row(idx + (bg * Nq + r) * (int64_t)slots, slots, c, lim[i] - n_init + 1, topk,
                  n_init, n_local, L0[i], L1[i], lane);
    }
}

template <typename T, int D>
cudaError_t tiled(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv, int Hs,
                  int Nq, int q_pos0, int nb, int topk, int n_init, int n_local, cudaStream_t st) {
    auto kern = topk_tiled_kernel<T, D>;
    const size_t smem = TopkSmem<D>::bytes;
    cudaError_t e = ensure_smem<topk_tiled_kernel<T, D>>((int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(Nq, kRT), (unsigned)(B * Hs));
    kern<<<grid, kTThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(kbar), idx,
                                        H, Hkv, Hs, Nq, q_pos0, nb, topk, n_init, n_local,
                                        n_init + n_local + topk);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Row-wise path (few rows, many blocks -- decode): candidates split into spans of 256 across
// CTAs; each CTA scores its span (one warp per candidate group, coalesced d-wide reads of kbar)
// and keeps a partial top-64; a second kernel merges the partial lists of a row.
constexpr int kSpan = 256;

int rowwise_splits(int q_pos0, int Nq) {
    const int max_c = (q_pos0 + Nq - 1) / kBlk;
    return ceil_div(max_c + 1, kSpan);
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
topk_rowwise_score_kernel(const T* __restrict__ q, const T* __restrict__ kbar,
                          uint64_t* __restrict__ part, int H, int Hkv, int Nq, int q_pos0, int nb,
                          int topk, int n_init, int n_local, int nsplit) {
    constexpr int kPer = D / 32;
    __shared__ float qs[D];
    __shared__ float sc[kSpan];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, r = blockIdx.y;
    const int64_t bg = blockIdx.z;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int c = (q_pos0 + r) / kBlk;
    const int lo = n_init, hi = c - n_local;
    const int j0 = lo + split * kSpan;
    for (int a = tid; a < D; a += 256) {
        float s = 0.f;
        for (int hh = 0; hh < G; ++hh) s += to_f(q[((b * H + (int64_t)g * G + hh) * Nq + r) * D + a]);
        qs[a] = s;
    }
    __syncthreads();
    float qv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) qv[j] = qs[lane * kPer + j];
    const T* kb = kbar + bg * (int64_t)nb * D;
    for (int t = warp; t < kSpan; t += 8) {
        const int blk = j0 + t;
        float s = 0.f;
        if (blk <= hi) {
            const T* row = kb + (int64_t)blk * D + lane * kPer;
#pragma unroll
            for (int j = 0; j < kPer; ++j) s = fmaf(qv[j], to_f(row[j]), s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) sc[t] = s;
    }
    __syncthreads();
    if (warp != 0) return;
    uint64_t l0 = 0, l1 = 0;
    const int K = min(topk, kCap);
    for (int t0 = 0; t0 < kSpan; t0 += 32) {
        const int blk = j0 + t0 + lane;
        const uint64_t key = (blk <= hi) ? sel_key(sc[t0 + lane], blk) : 0ull;
        warp_offer(l0, l1, key, K, lane);
    }
    uint64_t* dst = part + ((bg * Nq + r) * nsplit + split) * kCap;
    dst[2 * lane] = l0;
    dst[2 * lane + 1] = l1;
}

__global__ void __launch_bounds__(32)
topk_rowwise_merge_kernel(const uint64_t* __restrict__ part, int32_t* __restrict__ idx, int Hkv,
                          int Nq, int q_pos0, int topk, int n_init, int n_local, int nsplit,
                          int slots) {
    const int lane = threadIdx.x;
    const int r = blockIdx.x;
    const int64_t bg = blockIdx.y;
    const int c = (q_pos0 + r) / kBlk;
    const int ncand = c - n_local - n_init + 1;
    uint64_t l0 = 0, l1 = 0;
    const int K = min(topk, kCap);
    if (ncand > topk) {
        const uint64_t* src = part + (bg * Nq + r) * (int64_t)nsplit * kCap;
        const int used = min(nsplit, ceil_div(ncand, kSpan));
        for (int e = lane; e < used * kCap; e += 32) warp_offer(l0, l1, src[e], K, lane);
    }
    write_row(idx + (bg * Nq + r) * (int64_t)slots, slots, c, ncand, topk, n_init, n_local, l0, l1,
              lane);
}

template <typename T, int D>
cudaError_t rowwise(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv, int Nq,
                    int q_pos0, int nb, int topk, int n_init, int n_local, void* ws,
                    cudaStream_t st) {
    const int nsplit = rowwise_splits(q_pos0, Nq);
    uint64_t* part = static_cast<uint64_t*>(ws);
    dim3 g1(nsplit, Nq, (unsigned)(B * Hkv));
    topk_rowwise_score_kernel<T, D><<<g1, 256, 0, st>>>(static_cast<const T*>(q),
                                                        static_cast<const T*>(kbar), part, H, Hkv,
                                                        Nq, q_pos0, nb, topk, n_init, n_local,
                                                        nsplit);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2(Nq, (unsigned)(B * Hkv));
    topk_rowwise_merge_kernel<<<g2, 32, 0, st>>>(part, idx, Hkv, Nq, q_pos0, topk, n_init, n_local,
                                                 nsplit, n_init + n_local + topk);
    return cudaGetLastError();
}

}  // namespace

size_t rowwise_topk_workspace(int B, int Hkv, int Nq, int q_pos0, int topk) {
    (void)topk;
    if (B <= 0 || Hkv <= 0 || Nq <= 0) return 0;
    return (size_t)B * Hkv * Nq * rowwise_splits(q_pos0, Nq) * kCap * sizeof(uint64_t);
}

cudaError_t launch_block_topk_tiled(DType dt, const void* q, const void* kbar, int32_t* idx, int B,
                                    int H, int Hkv, int Hs, int Nq, int q_pos0, int nb, int d,
                                    int topk, int n_init, int n_local, cudaStream_t st, DevCtx) {
    if (dt == DType::F32)
        return d == 64 ? tiled<float, 64>(q, kbar, idx, B, H, Hkv, Hs, Nq, q_pos0, nb, topk, n_init, n_local, st)
                       : tiled<float, 128>(q, kbar, idx, B, H, Hkv, Hs, Nq, q_pos0, nb, topk, n_init, n_local, st);
    return d == 64 ? tiled<__nv_bfloat16, 64>(q, kbar, idx, B, H, Hkv, Hs, Nq, q_pos0, nb, topk, n_init, n_local, st)
                   : tiled<__nv_bfloat16, 128>(q, kbar, idx, B, H, Hkv, Hs, Nq, q_pos0, nb, topk, n_init, n_local, st);
}

cudaError_t launch_block_topk_rowwise(DType dt, const void* q, const void* kbar, int32_t* idx,
                                      int B, int H, int Hkv, int Nq, int q_pos0, int nb, int d,
                                      int topk, int n_init, int n_local, void* ws, cudaStream_t st,
                                      DevCtx) {
    if (dt == DType::F32)
        return d == 64 ? rowwise<float, 64>(q, kbar, idx, B, H, Hkv, Nq, q_pos0, nb, topk, n_init, n_local, ws, st)
                       : rowwise<float, 128>(q, kbar, idx, B, H, Hkv, Nq, q_pos0, nb, topk, n_init, n_local, ws, st);
    return d == 64 ? rowwise<__nv_bfloat16, 64>(q, kbar, idx, B, H, Hkv, Nq, q_pos0, nb, topk, n_init, n_local, ws, st)
                   : rowwise<__nv_bfloat16, 128>(q, kbar, idx, B, H, Hkv, Nq, q_pos0, nb, topk, n_init, n_local, ws, st);
}

}  // namespace sala
