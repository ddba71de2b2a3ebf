// Query-block-granular block selection (the variant of the selection step in which the tokens of
// one query block share one selection): per (batch, KV group, query block c of 64 tokens) the
// score vector is the sum of q over the group's G heads and the block's tokens, the candidates are
// the blocks n_init .. c - n_local, the best k by (score, lower block first) join the forced init
// and local blocks, and the resulting ascending row is written to every token row of the block,
// in the layout of the per-token selection (so the sparse prefill takes it unchanged).
//
// One CTA per (batch, group, query block), 256 threads, on the CUDA cores (the scoring is a
// matrix-vector product per block, ~0.5 % of the per-token selection's work):
//   1. the summed query in fp32: thread = (4 columns, a stride of the G * 64 rows), partials
//      reduced through shared memory;
//   2. scores: one warp per candidate row of kbar (coalesced), four rows in flight per warp;
//   3. the exact best k: chunks of kChunk candidates plus the best k so far, radix select
//      (blocksel.cuh), winners carried to the next chunk;
//   4. the winners sorted ascending by one warp, the slot row written to the block's token rows.
#include <type_traits>

#include "blocksel.cuh"
#include "kernels.h"

namespace sala {
namespace {

constexpr int kThreads = 256;
constexpr int kQB = 64;                    // tokens per query block (= key block)
constexpr int kCapK = 64;                  // largest k that ranks
constexpr int kE = 16;                     // keys per thread in one radix select
constexpr int kChunk = kE * kThreads;      // keys per select: new candidates + carried winners
constexpr int kNew = kChunk - kCapK;

template <int D>
struct QbSmem {
    float part[kThreads / (D / 4)][D];     // partial sums of the query block
    float qs[D];                           // the summed query
    uint64_t keys[kChunk];                 // one chunk's keys, then the carried winners
    uint64_t carry[kCapK];
    int win[kCapK];
    int n_win;
    RadixSelSmem rs;
};

// Ascending bitonic sort of 64 ints held two per lane (position 2 * lane + j).
__device__ __forceinline__ void sort64_asc(int& x0, int& x1, int lane) {
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

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&f)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&f)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[4]) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
}

// Partial dot product of a kbar row with the summed query: lane covers D / 32 elements.
template <typename T, int D>
__device__ __forceinline__ float dot_lane(const T* row, const float* qs, int lane) {
    if constexpr (D == 128) {
        float f[4];
        load4<T>(row + 4 * lane, f);
        return f[0] * qs[4 * lane] + f[1] * qs[4 * lane + 1] + f[2] * qs[4 * lane + 2] +
               f[3] * qs[4 * lane + 3];
    } else {
        return to_f(row[2 * lane]) * qs[2 * lane] + to_f(row[2 * lane + 1]) * qs[2 * lane + 1];
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
topk_qblock_kernel(const T* __restrict__ q, const T* __restrict__ kbar, int32_t* __restrict__ idx,
                   int H, int Hkv, int Nq, int nb, int topk, int n_init, int n_local, int slots) {
    extern __shared__ __align__(16) unsigned char smraw[];
    QbSmem<D>& sm = *reinterpret_cast<QbSmem<D>*>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nqb = (Nq + kQB - 1) / kQB;
    const int64_t bg = blockIdx.x / nqb;
    const int c = (int)(blockIdx.x % nqb);
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int r0 = c * kQB, nr = min(Nq, r0 + kQB) - r0;
    const int lo = n_init, hi = c - n_local;
    const int ncand = hi - lo + 1;
    int32_t* out = idx + (bg * Nq + r0) * (int64_t)slots;  // the block's first token row
    if (ncand <= topk) {  // every candidate taken: blocks 0 .. c
        for (int e = tid; e < nr * slots; e += kThreads) out[e] = (e % slots) <= c ? e % slots : -1;
        return;
    }
    const int K = min(topk, kCapK);  // a ranking k is at most 64 (validated by the caller)

    // 1. the summed query (fp32)
    {
        constexpr int kCG = D / 4, kRL = kThreads / kCG;
        const int cg = tid % kCG, rl = tid / kCG;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int nrows = G * nr;
#pragma unroll 4
        for (int e = rl; e < nrows; e += kRL) {
            const int h = e / nr, r = r0 + e % nr;
            float f[4];
            load4<T>(q + ((b * H + (int64_t)g * G + h) * Nq + r) * D + 4 * cg, f);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] += f[i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) sm.part[rl][4 * cg + i] = acc[i];
        if (tid < kCapK) sm.carry[tid] = 0ull;
        __syncthreads();
        if (tid < D) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kRL; ++w) s += sm.part[w][tid];
            sm.qs[tid] = s;
        }
        __syncthreads();
    }

    // 2.-3. scores chunk by chunk, the best K carried through a radix select per chunk
    const T* kb = kbar + bg * (int64_t)nb * D;
    auto sync = [] { __syncthreads(); };
    for (int cb = 0; cb < ncand; cb += kNew) {
        const int nc = min(kNew, ncand - cb);
        for (int i0 = warp * 4; i0 < nc; i0 += (kThreads / 32) * 4) {
            float dv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                dv[u] = i0 + u < nc ? dot_lane<T, D>(kb + (int64_t)(lo + cb + i0 + u) * D, sm.qs, lane) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dv[u] += __shfl_xor_sync(0xffffffffu, dv[u], off);
            if (lane < 4 && i0 + lane < nc) {
                const float d = lane == 0 ? dv[0] : lane == 1 ? dv[1] : lane == 2 ? dv[2] : dv[3];
                sm.keys[i0 + lane] = sel_key(d, lo + cb + i0 + lane);
            }
        }
        for (int i = nc + tid; i < kNew; i += kThreads) sm.keys[i] = 0ull;
        if (tid < kCapK) sm.keys[kNew + tid] = sm.carry[tid];
        __syncthreads();
        uint64_t key[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) key[e] = sm.keys[e * kThreads + tid];
        if (tid == 0) sm.n_win = 0;
        uint64_t prefix, mask;
        radix_kth<kE>(key, K, sm.rs, prefix, mask, tid, sync);
#pragma unroll
        for (int e = 0; e < kE; ++e)
            if (key[e] && (key[e] & mask) >= prefix) sm.carry[atomicAdd(&sm.n_win, 1)] = key[e];
        __syncthreads();
    }

    // 4. winners ascending, then the slot row for every token of the block
    if (warp == 0) {
        int x0 = 2 * lane < K ? key_block(sm.carry[2 * lane]) : 0x7fffffff;
        int x1 = 2 * lane + 1 < K ? key_block(sm.carry[2 * lane + 1]) : 0x7fffffff;
        sort64_asc(x0, x1, lane);
        sm.win[2 * lane] = x0;
        sm.win[2 * lane + 1] = x1;
    }
    __syncthreads();
    for (int e = tid; e < nr * slots; e += kThreads) {
        const int s = e % slots;
        int v;
        if (s < n_init) v = s;
        else if (s < n_init + K) v = sm.win[s - n_init];
        else if (s < n_init + K + n_local) v = c - n_local + 1 + (s - n_init - K);
        else v = -1;
        out[e] = v;
    }
}

// ---------------------------------------------------------------------------------------------
// Softmax-probability group aggregation (same granularity and output): head h of the group scores
// candidate j with the logit scale * (u_h . kbar_j), u_h the mean of the block's queries of head
// h; each head's logits go through a softmax over the candidates, and a block's score is the sum
// over the heads of its probabilities.
//   1. u_h for the G <= 16 heads (fp32, scaled by scale * log2 e: logits in log2 units);
//   2. pass 1: lane pair (h, half) holds u_h's half in registers and dots it with each
//      candidate's k-bar half (every lane of a half reads the same row: one load per address),
//      the pair combines, and keeps a running max and sum of 2^logit; the warps' partial
//      (max, sum) pairs are merged per head;
//   3. pass 2: the same dots, 2^(logit - M_h) / S_h summed over the heads, then the chunked exact
//      top k of the plain query-block kernel.
constexpr int kGmax = 16;

template <int D>
struct QsSmem {
    float u[kGmax][D];
    float m[kThreads / 32][kGmax], s[kThreads / 32][kGmax];
    float M[kGmax], S[kGmax];
    uint64_t keys[kChunk];
    uint64_t carry[kCapK];
    int win[kCapK];
    int n_win;
    RadixSelSmem rs;
};

// Dot of the lane's half of u_h (registers) with the same half of a k-bar row, both halves
// summed (lane pairs 2h, 2h + 1).
template <typename T, int D>
__device__ __forceinline__ float pair_dot(const T* row, const float (&uh)[D / 2], int half) {
    float acc = 0.f;
    const T* p = row + half * (D / 2);
#pragma unroll
    for (int e = 0; e < D / 2; e += 4) {
        float f[4];
        load4<T>(p + e, f);
        acc = fmaf(f[0], uh[e], acc);
        acc = fmaf(f[1], uh[e + 1], acc);
        acc = fmaf(f[2], uh[e + 2], acc);
        acc = fmaf(f[3], uh[e + 3], acc);
    }
    return acc + __shfl_xor_sync(0xffffffffu, acc, 1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
topk_qblock_softmax_kernel(const T* __restrict__ q, const T* __restrict__ kbar,
                           int32_t* __restrict__ idx, int H, int Hkv, int Nq, int nb, int topk,
                           int n_init, int n_local, int slots, float sl2) {
    extern __shared__ __align__(16) unsigned char smraw[];
    QsSmem<D>& sm = *reinterpret_cast<QsSmem<D>*>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kThreads / 32;
    const int nqb = (Nq + kQB - 1) / kQB;
    const int64_t bg = blockIdx.x / nqb;
    const int c = (int)(blockIdx.x % nqb);
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int r0 = c * kQB, nr = min(Nq, r0 + kQB) - r0;
    const int lo = n_init, hi = c - n_local;
    const int ncand = hi - lo + 1;
    int32_t* out = idx + (bg * Nq + r0) * (int64_t)slots;
    if (ncand <= topk) {  // every candidate taken: blocks 0 .. c
        for (int e = tid; e < nr * slots; e += kThreads) out[e] = (e % slots) <= c ? e % slots : -1;
        return;
    }
    const int K = min(topk, kCapK);

    // 1. scaled mean queries
    for (int e = tid; e < kGmax * (D / 4); e += kThreads) {
        const int h = e / (D / 4), c4 = e % (D / 4);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (h < G) {
            const T* qh = q + ((b * H + (int64_t)g * G + h) * Nq + r0) * D + 4 * c4;
            for (int r = 0; r < nr; ++r) {
                float f[4];
                load4<T>(qh + (int64_t)r * D, f);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] += f[i];
            }
        }
        const float w = sl2 / (float)nr;
#pragma unroll
        for (int i = 0; i < 4; ++i) sm.u[h][4 * c4 + i] = acc[i] * w;
    }
    if (tid < kCapK) sm.carry[tid] = 0ull;
    __syncthreads();
    const int h = lane >> 1, half = lane & 1;
    const bool live = h < G;
    float uh[D / 2];
#pragma unroll
    for (int e = 0; e < D / 2; ++e) uh[e] = sm.u[h][half * (D / 2) + e];
    const T* kb = kbar + bg * (int64_t)nb * D;

    // 2. per-head max and sum of 2^logit over the candidates
    float m = -INFINITY, sum = 0.f;
    for (int i = warp; i < ncand; i += kWarps) {
        const float l = pair_dot<T, D>(kb + (int64_t)(lo + i) * D, uh, half);
        if (l > m) {
            sum = sum * exp2f(m - l) + 1.f;
            m = l;
        } else {
            sum += exp2f(l - m);
        }
    }
    if (half == 0 && live) {
        sm.m[warp][h] = m;
        sm.s[warp][h] = sum;
    }
    __syncthreads();
    if (tid < G) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.m[w][tid]);
        float S = 0.f;
        for (int w = 0; w < kWarps; ++w)
            if (sm.m[w][tid] != -INFINITY) S += sm.s[w][tid] * exp2f(sm.m[w][tid] - M);
        sm.M[tid] = M;
        sm.S[tid] = S;
    }
    __syncthreads();
    const float Mh = live ? sm.M[h] : 0.f, invS = live ? 1.f / sm.S[h] : 0.f;

    // 3. scores chunk by chunk, the best K carried through a radix select per chunk
    auto sync = [] { __syncthreads(); };
    for (int cb = 0; cb < ncand; cb += kNew) {
        const int nc = min(kNew, ncand - cb);
        for (int i = warp; i < nc; i += kWarps) {
            const float l = pair_dot<T, D>(kb + (int64_t)(lo + cb + i) * D, uh, half);
            float p = (live && half == 0) ? exp2f(l - Mh) * invS : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
            if (lane == 0) sm.keys[i] = sel_key(p, lo + cb + i);
        }
        for (int i = nc + tid; i < kNew; i += kThreads) sm.keys[i] = 0ull;
        if (tid < kCapK) sm.keys[kNew + tid] = sm.carry[tid];
        __syncthreads();
        uint64_t key[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) key[e] = sm.keys[e * kThreads + tid];
        if (tid == 0) sm.n_win = 0;
        uint64_t prefix, mask;
        radix_kth<kE>(key, K, sm.rs, prefix, mask, tid, sync);
#pragma unroll
        for (int e = 0; e < kE; ++e)
            if (key[e] && (key[e] & mask) >= prefix) sm.carry[atomicAdd(&sm.n_win, 1)] = key[e];
        __syncthreads();
    }

    // 4. winners ascending, then the slot row for every token of the block
    if (warp == 0) {
        int x0 = 2 * lane < K ? key_block(sm.carry[2 * lane]) : 0x7fffffff;
        int x1 = 2 * lane + 1 < K ? key_block(sm.carry[2 * lane + 1]) : 0x7fffffff;
        sort64_asc(x0, x1, lane);
        sm.win[2 * lane] = x0;
        sm.win[2 * lane + 1] = x1;
    }
    __syncthreads();
    for (int e = tid; e < nr * slots; e += kThreads) {
        const int s = e % slots;
        int v;
        if (s < n_init) v = s;
        else if (s < n_init + K) v = sm.win[s - n_init];
        else if (s < n_init + K + n_local) v = c - n_local + 1 + (s - n_init - K);
        else v = -1;
        out[e] = v;
    }
}

// bf16 inputs: the same two passes with the scoring on the tensor cores.  Per warp and group of
// 8 candidates, m16n8k16 MMAs give the 16 heads' logits (rows: heads, columns: candidates) from
// the mean queries split into bf16 hi + lo (two MMAs per K step, so a logit carries ~2^-17
// relative error, like the fp32 dot products) and the candidates' k-bar rows, loaded straight
// into the B fragments.  Lane (g = lane / 4, t = lane % 4) holds heads g and g + 8 of candidates
// 2t and 2t + 1.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(kThreads)
topk_qblock_softmax_mma_kernel(const __nv_bfloat16* __restrict__ q,
                               const __nv_bfloat16* __restrict__ kbar, int32_t* __restrict__ idx,
                               int H, int Hkv, int Nq, int nb, int topk, int n_init, int n_local,
                               int slots, float sl2) {
    constexpr int kKS = D / 16;  // K steps
    extern __shared__ __align__(16) unsigned char smraw[];
    QsSmem<D>& sm = *reinterpret_cast<QsSmem<D>*>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kThreads / 32;
    const int nqb = (Nq + kQB - 1) / kQB;
    const int64_t bg = blockIdx.x / nqb;
    const int c = (int)(blockIdx.x % nqb);
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int G = H / Hkv;
    const int r0 = c * kQB, nr = min(Nq, r0 + kQB) - r0;
    const int lo = n_init, hi = c - n_local;
    const int ncand = hi - lo + 1;
    int32_t* out = idx + (bg * Nq + r0) * (int64_t)slots;
    if (ncand <= topk) {
        for (int e = tid; e < nr * slots; e += kThreads) out[e] = (e % slots) <= c ? e % slots : -1;
        return;
    }
    const int K = min(topk, kCapK);

    // 1. scaled mean queries (fp32, heads past G zero)
    for (int e = tid; e < kGmax * (D / 4); e += kThreads) {
        const int h = e / (D / 4), c4 = e % (D / 4);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (h < G) {
            const __nv_bfloat16* qh = q + ((b * H + (int64_t)g * G + h) * Nq + r0) * D + 4 * c4;
            for (int r = 0; r < nr; ++r) {
                float f[4];
                load4<__nv_bfloat16>(qh + (int64_t)r * D, f);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] += f[i];
            }
        }
        const float w = sl2 / (float)nr;
#pragma unroll
        for (int i = 0; i < 4; ++i) sm.u[h][4 * c4 + i] = acc[i] * w;
    }
    if (tid < kCapK) sm.carry[tid] = 0ull;
    __syncthreads();
    const int gi = lane >> 2, ti = lane & 3;
    // A fragments of u (hi and lo terms) for every K step
    uint32_t ah[kKS][4], al[kKS][4];
#pragma unroll
    for (int ks = 0; ks < kKS; ++ks) {
        const int k0 = 16 * ks + 2 * ti;
        const float x[4][2] = {{sm.u[gi][k0], sm.u[gi][k0 + 1]},
                               {sm.u[gi + 8][k0], sm.u[gi + 8][k0 + 1]},
                               {sm.u[gi][k0 + 8], sm.u[gi][k0 + 9]},
                               {sm.u[gi + 8][k0 + 8], sm.u[gi + 8][k0 + 9]}};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            ah[ks][r] = pack_bf2(x[r][0], x[r][1]);
            al[ks][r] = pack_bf2(x[r][0] - __uint_as_float(ah[ks][r] << 16),
                                 x[r][1] - __uint_as_float(ah[ks][r] & 0xffff0000u));
        }
    }
    const __nv_bfloat16* kb = kbar + bg * (int64_t)nb * D;
    // logits of candidates j0 .. j0+7 (rows past the last candidate read a valid row, unused)
    auto logits = [&](int j0, float (&acc)[4]) {
        const int j = min(j0 + gi, hi);
        const uint32_t* row = reinterpret_cast<const uint32_t*>(kb + (int64_t)j * D);
        uint32_t bf[kKS][2];
#pragma unroll
        for (int ks = 0; ks < kKS; ++ks) {
            bf[ks][0] = __ldg(row + 8 * ks + ti);
            bf[ks][1] = __ldg(row + 8 * ks + ti + 4);
        }
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < kKS; ++ks) {
            mma_bf16_16816(acc, ah[ks], bf[ks][0], bf[ks][1]);
            mma_bf16_16816(acc, al[ks], bf[ks][0], bf[ks][1]);
        }
    };
    const bool live0 = gi < G, live1 = gi + 8 < G;

    // 2. per-head max and sum of 2^logit over the candidates (heads g and g + 8 of this lane)
    float m0 = -INFINITY, s0 = 0.f, m1 = -INFINITY, s1 = 0.f;
    auto fold = [](float& m, float& s, float l) {
        if (l > m) {
            s = s * exp2f(m - l) + 1.f;
            m = l;
        } else {
            s += exp2f(l - m);
        }
    };
    for (int j0 = lo + 8 * warp; j0 <= hi; j0 += 8 * kWarps) {
        float acc[4];
        logits(j0, acc);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (j0 + 2 * ti + e > hi) continue;
            fold(m0, s0, acc[e]);
            fold(m1, s1, acc[2 + e]);
        }
    }
    // merge the four lanes of a head (t = 0..3), then the warps
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        const float om0 = __shfl_xor_sync(0xffffffffu, m0, off), os0 = __shfl_xor_sync(0xffffffffu, s0, off);
        const float om1 = __shfl_xor_sync(0xffffffffu, m1, off), os1 = __shfl_xor_sync(0xffffffffu, s1, off);
        const float n0 = fmaxf(m0, om0), n1 = fmaxf(m1, om1);
        s0 = (m0 == -INFINITY ? 0.f : s0 * exp2f(m0 - n0)) + (om0 == -INFINITY ? 0.f : os0 * exp2f(om0 - n0));
        s1 = (m1 == -INFINITY ? 0.f : s1 * exp2f(m1 - n1)) + (om1 == -INFINITY ? 0.f : os1 * exp2f(om1 - n1));
        m0 = n0;
        m1 = n1;
    }
    if (ti == 0) {
        sm.m[warp][gi] = m0;
        sm.s[warp][gi] = s0;
        sm.m[warp][gi + 8] = m1;
        sm.s[warp][gi + 8] = s1;
    }
    __syncthreads();
    if (tid < kGmax) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.m[w][tid]);
        float S = 0.f;
        for (int w = 0; w < kWarps; ++w)
            if (sm.m[w][tid] != -INFINITY) S += sm.s[w][tid] * exp2f(sm.m[w][tid] - M);
        sm.M[tid] = M;
        sm.S[tid] = S;
    }
    __syncthreads();
    const float M0 = sm.M[gi], M1 = sm.M[gi + 8];
    const float iS0 = live0 ? 1.f / sm.S[gi] : 0.f, iS1 = live1 ? 1.f / sm.S[gi + 8] : 0.f;

    // 3. scores chunk by chunk (8 candidates per warp step), the best K carried through a radix
    //    select per chunk
    auto sync = [] { __syncthreads(); };
    for (int cb = 0; cb < ncand; cb += kNew) {
        const int nc = min(kNew, ncand - cb);
        for (int i0 = 8 * warp; i0 < nc; i0 += 8 * kWarps) {
            float acc[4];
            logits(lo + cb + i0, acc);
            float p[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
                p[e] = (live0 ? exp2f(acc[e] - M0) * iS0 : 0.f) + (live1 ? exp2f(acc[2 + e] - M1) * iS1 : 0.f);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                p[0] += __shfl_xor_sync(0xffffffffu, p[0], off);
                p[1] += __shfl_xor_sync(0xffffffffu, p[1], off);
            }
            if (gi == 0) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int i = i0 + 2 * ti + e;
                    if (i < nc) sm.keys[i] = sel_key(p[e], lo + cb + i);
                }
            }
        }
        for (int i = nc + tid; i < kNew; i += kThreads) sm.keys[i] = 0ull;
        if (tid < kCapK) sm.keys[kNew + tid] = sm.carry[tid];
        __syncthreads();
        uint64_t key[kE];
#pragma unroll
        for (int e = 0; e < kE; ++e) key[e] = sm.keys[e * kThreads + tid];
        if (tid == 0) sm.n_win = 0;
        uint64_t prefix, mask;
        radix_kth<kE>(key, K, sm.rs, prefix, mask, tid, sync);
#pragma unroll
        for (int e = 0; e < kE; ++e)
            if (key[e] && (key[e] & mask) >= prefix) sm.carry[atomicAdd(&sm.n_win, 1)] = key[e];
        __syncthreads();
    }

    // 4. winners ascending, then the slot row for every token of the block
    if (warp == 0) {
        int x0 = 2 * lane < K ? key_block(sm.carry[2 * lane]) : 0x7fffffff;
        int x1 = 2 * lane + 1 < K ? key_block(sm.carry[2 * lane + 1]) : 0x7fffffff;
        sort64_asc(x0, x1, lane);
        sm.win[2 * lane] = x0;
        sm.win[2 * lane + 1] = x1;
    }
    __syncthreads();
    for (int e = tid; e < nr * slots; e += kThreads) {
        const int s = e % slots;
        int v;
        if (s < n_init) v = s;
        else if (s < n_init + K) v = sm.win[s - n_init];
        else if (s < n_init + K + n_local) v = c - n_local + 1 + (s - n_init - K);
        else v = -1;
        out[e] = v;
    }
}

template <typename T, int D>
cudaError_t launch_qbs(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv, int Nq,
                       int nb, int topk, int n_init, int n_local, float scale, cudaStream_t st) {
    const int nqb = (Nq + kQB - 1) / kQB;
    const int64_t grid = (int64_t)B * Hkv * nqb;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff || H / Hkv > kGmax) return cudaErrorNotSupported;
    const int smem = (int)sizeof(QsSmem<D>);
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        cudaError_t e = ensure_smem<topk_qblock_softmax_mma_kernel<D>>(smem);
        if (e != cudaSuccess) return e;
        topk_qblock_softmax_mma_kernel<D><<<(unsigned)grid, kThreads, smem, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(kbar), idx, H, Hkv, Nq, nb, topk,
            n_init, n_local, n_init + n_local + topk, scale * 1.4426950408889634f);
    } else {
        cudaError_t e = ensure_smem<topk_qblock_softmax_kernel<T, D>>(smem);
        if (e != cudaSuccess) return e;
        topk_qblock_softmax_kernel<T, D><<<(unsigned)grid, kThreads, smem, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(kbar), idx, H, Hkv, Nq, nb, topk,
            n_init, n_local, n_init + n_local + topk, scale * 1.4426950408889634f);
    }
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_qb(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv, int Nq,
                      int nb, int topk, int n_init, int n_local, cudaStream_t st) {
    const int nqb = (Nq + kQB - 1) / kQB;
    const int64_t grid = (int64_t)B * Hkv * nqb;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorNotSupported;
    const int smem = (int)sizeof(QbSmem<D>);
    cudaError_t e = ensure_smem<topk_qblock_kernel<T, D>>(smem);
    if (e != cudaSuccess) return e;
    topk_qblock_kernel<T, D><<<(unsigned)grid, kThreads, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(kbar), idx, H, Hkv, Nq, nb, topk, n_init,
        n_local, n_init + n_local + topk);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_topk_qblock(DType dt, const void* q, const void* kbar, int32_t* idx, int B,
                                     int H, int Hkv, int Nq, int nb, int d, int topk, int n_init,
                                     int n_local, cudaStream_t st, DevCtx) {
    if (dt == DType::F32)
        return d == 64 ? launch_qb<float, 64>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, st)
                       : launch_qb<float, 128>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, st);
    return d == 64 ? launch_qb<__nv_bfloat16, 64>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, st)
                   : launch_qb<__nv_bfloat16, 128>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, st);
}

cudaError_t launch_block_topk_qblock_softmax(DType dt, const void* q, const void* kbar, int32_t* idx,
                                             int B, int H, int Hkv, int Nq, int nb, int d, int topk,
                                             int n_init, int n_local, float scale, cudaStream_t st,
                                             DevCtx) {
    if (dt == DType::F32)
        return d == 64 ? launch_qbs<float, 64>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, scale, st)
                       : launch_qbs<float, 128>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, scale, st);
    return d == 64 ? launch_qbs<__nv_bfloat16, 64>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, scale, st)
                   : launch_qbs<__nv_bfloat16, 128>(q, kbar, idx, B, H, Hkv, Nq, nb, topk, n_init, n_local, scale, st);
}

}  // namespace sala
