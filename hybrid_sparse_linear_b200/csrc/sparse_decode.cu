// Sparse decode in one launch: block scoring, top-k selection and attention for one query token
// per (batch, KV group), at any context length the workspace covers.
//
// One query row per KV group meets a context of up to millions of keys, so every phase is a
// memory stream with little arithmetic: the scores read the whole block-key table k_bar (8 MiB at
// 2^20 tokens and 2 KV heads), the attention reads the ~67 selected K/V blocks (4 MiB).  Spread
// over the GPU, each phase is one round of loads.  The kernel runs all of them in one cooperative
// launch (all CTAs resident, so a grid-wide barrier is safe), with `cpg` CTAs per (batch, group):
//   A  CTA j scores candidate span j (256 blocks, 256 bytes of k_bar each, read coalesced) and
//      publishes the span's top-k keys sorted largest first (a bitonic sort of the 256 keys).
//   -- grid barrier --
//   B  every CTA of the group finds the group's top-k from the spans' first 8 keys (a radix
//      select on 64-bit keys; exact unless some span's 8th key is itself a winner, in which case
//      the spans' whole lists are merged), the same deterministic result in each CTA, so no
//      second exchange is needed, and forms the ascending slot list: init blocks, top-k, local
//      blocks, -1 padding.
//   C  CTA j attends slot j (and j + cpg, ...): K and V of the block staged in shared memory,
//      G heads' logits and p v (bf16: warp-level tensor-core tiles; fp32: CUDA cores), a per-head
//      softmax partial (max, sum, sum of p v) written to workspace.
//   -- grid barrier --
//   D  CTA j combines the partials of one (head, 32-column) piece of the output.
// Selection keys pack (orderable score << 32 | ~block): one unsigned compare orders by score,
// then by lower block index, so the k-th largest key is unique and ties go to the lower block.
//
// The grid barrier counts arrivals in the low half of the workspace's first word, which must be
// zero before the first call; the last CTA to arrive puts it back to zero, so every call that
// completes leaves it as it found it.  Waits are bounded (the device status word records a
// timeout).
#include <mutex>
#include <type_traits>

#include "blocksel.cuh"
#include "decode_common.cuh"
#include "kernels.h"

namespace sala {
namespace {

using namespace dec;

constexpr int kBlk = 64;
constexpr int kSpan = 256;
constexpr int kThreads = 256;
constexpr int kCap = 64;       // largest k
constexpr int kMaxSlots = 80;  // n_init + n_local + k
constexpr int kMaxG = 16;
constexpr int kMergeE = 32;    // keys per thread in phase B: spans * k <= 8192

__device__ __forceinline__ uint64_t sel_key_u(float score, int blk) { return sel_key(score, blk); }

// Block-wide bitonic sort, largest first, of the E keys each thread holds (element E*tid + i).
// Partners within a thread swap in registers, within a warp by shuffle, else through buf (one
// slot per element, E * blockDim.x keys).
template <int E>
__device__ __forceinline__ void block_sort_desc(uint64_t (&x)[E], uint64_t* buf) {
    const int tid = threadIdx.x;
#pragma unroll
    for (int kk = 2; kk <= E * kThreads; kk <<= 1) {
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            uint64_t y[E];
            if (jj < E) {
#pragma unroll
                for (int i = 0; i < E; ++i) y[i] = x[i ^ jj];
            } else if (jj < 32 * E) {
#pragma unroll
                for (int i = 0; i < E; ++i) y[i] = __shfl_xor_sync(0xffffffffu, x[i], jj / E);
            } else {
#pragma unroll
                for (int i = 0; i < E; ++i) buf[E * tid + i] = x[i];
                __syncthreads();
#pragma unroll
                for (int i = 0; i < E; ++i) y[i] = buf[(E * tid + i) ^ jj];
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const int e = E * tid + i;
                const bool dsc = (e & kk) == 0, lower = (e & jj) == 0;
                x[i] = (lower == dsc) ? (x[i] > y[i] ? x[i] : y[i]) : (x[i] < y[i] ? x[i] : y[i]);
            }
        }
    }
}

template <int D>
struct DecSmem {
    union {
        struct {                  // fp32 inputs: the slot's block and the queries as fp32
            float K[kBlk][D + 4];  // rows padded: aligned and conflict-free
            float V[kBlk][D];
            float Q[kMaxG][D];
        };
        struct {                  // bf16 inputs: tensor-core operands (rows padded by 16 bytes)
            __nv_bfloat16 Kb[kBlk][D + 8];
            __nv_bfloat16 Vb[kBlk][D + 8];
            __nv_bfloat16 Qb[kMaxG][D + 8];
            __nv_bfloat16 Pb[kMaxG][kBlk + 8];
        };
    };
    float P[kMaxG][kBlk];   // logits, then probabilities
    float m[kMaxG], l[kMaxG];
    float qbar[D];
    float sc[kSpan];
    int sel[kMaxSlots];
    int sel_top[kCap];
    uint64_t cand[2 * kThreads];
    RadixSelSmem ss;
    int sel_n;
    int ok, overflow;
    float cm[8][32], cl[8][32], co[8][32];  // phase D per-warp partials
};

template <typename T>
__device__ __forceinline__ void cvt16(const uint4& u, float* f);  // sizeof(T) * ... elements
template <>
__device__ __forceinline__ void cvt16<__nv_bfloat16>(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
template <>
__device__ __forceinline__ void cvt16<float>(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
sparse_decode_fused_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                           const T* __restrict__ vc, const T* __restrict__ kbar,
                           const int32_t* __restrict__ idx_in, int32_t* __restrict__ idx_out,
                           T* __restrict__ o, int H, int Hkv, int pos, int Tmax, int nb_cap,
                           int topk, int n_init, int n_local, int slots, float scale, int cpg,
                           int span_stride, const int32_t* __restrict__ pos_b,
                           const int32_t* __restrict__ pages, int max_pages, int n_pages,
                           unsigned* bar, uint64_t* part, float* rec, DevCtx ctx) {
    extern __shared__ __align__(16) unsigned char dsm_raw[];
    DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>(dsm_raw);
    // A kernel launched after this one as its programmatic dependent (sala_linear_decode_pdl)
    // may start now: it reads only its own state until this grid has completed.  (This kernel is
    // not itself a programmatic dependent, so everything launched before it has completed.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / Hkv;
    const int bg = blockIdx.x / cpg, j = blockIdx.x % cpg;
    const int64_t b = bg / Hkv;
    const int g = bg % Hkv;
    // This sequence's query position: the launch's pos for all, or its own (pos_b[b], at most pos;
    // one out of range is flagged and clamped, so every CTA still reaches both grid barriers).
    int pos_s = pos;
    if (pos_b) {
        pos_s = __ldg(pos_b + b);
        if (pos_s < 0 || pos_s > pos) {
            if (tid == 0) flag(ctx, kStatusBounds);
            pos_s = pos_s < 0 ? 0 : pos;
        }
    }
    const int c = pos_s / kBlk;
    const int lo = n_init, hi = c - n_local;
    const int ncand = hi - lo + 1;
    const int K = topk;
    const bool do_sel = idx_in == nullptr && ncand > K;
    const int nspan = ncand > K ? (ncand + kSpan - 1) / kSpan : 0;  // this sequence's spans
    const T* qg = q + (b * H + (int64_t)g * G) * D;  // the group's G query rows

    // ---------------------------------------------------------------- A: span scores + top-k
    // Rows of k_bar are read coalesced: kLPR lanes per row, 16 elements per lane.  Each span
    // publishes its top-k keys sorted, largest first.
    constexpr int kLPR = D / 16, kRPS = 32 / kLPR, kSteps = (kSpan / 8) / kRPS;
    if (do_sel && K > 0) {
        const T* kb = kbar + (int64_t)bg * nb_cap * D;
        const int part16 = (lane % kLPR) * 16;
        constexpr int kU = 16 * sizeof(T) / 16;   // 16-byte pieces per lane and row
        constexpr int kEl = 16 / sizeof(T);        // elements per piece
        uint4 raw[kSteps][kU];
        auto load_span = [&](int span) {  // every load of the span in flight at once
            const int base = lo + span * kSpan;
#pragma unroll
            for (int st = 0; st < kSteps; ++st) {
                const int blk = base + warp * (kSpan / 8) + st * kRPS + lane / kLPR;
                const T* row = kb + (int64_t)blk * D + part16;
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    raw[st][u] = blk <= hi ? ld16(row + u * kEl) : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        // The first span's k_bar rows are requested before the query rows they are scored
        // against, so the two memory round trips overlap.
        if (j < nspan) load_span(j);
        if (tid < D) {  // all G loads in flight at once (a runtime-G loop would issue them one by one)
            float qv[kMaxG];
#pragma unroll
            for (int hh = 0; hh < kMaxG; ++hh) qv[hh] = hh < G ? to_f(qg[hh * D + tid]) : 0.f;
            float s = 0.f;
#pragma unroll
            for (int hh = 0; hh < kMaxG; ++hh) s += qv[hh];
            sm.qbar[tid] = s;
        }
        __syncthreads();
        for (int span = j; span < nspan; span += cpg) {
            const int base = lo + span * kSpan;
            if (span != j) load_span(span);
#pragma unroll
            for (int st = 0; st < kSteps; ++st) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    float f[kEl];
                    cvt16<T>(raw[st][u], f);
#pragma unroll
                    for (int i = 0; i < kEl; i += 2) {
                        a0 = fmaf(sm.qbar[part16 + u * kEl + i], f[i], a0);
                        a1 = fmaf(sm.qbar[part16 + u * kEl + i + 1], f[i + 1], a1);
                    }
                }
                float d = a0 + a1;
#pragma unroll
                for (int off = 1; off < kLPR; off <<= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                if (lane % kLPR == 0) sm.sc[warp * (kSpan / 8) + st * kRPS + lane / kLPR] = d;
            }
            __syncthreads();
            // The span's keys sorted largest first (block-wide bitonic network, one key per
            // thread; strides below 32 within the warp), then its first k written out.
            const int blk = base + tid;
            uint64_t x[1] = {blk <= hi ? sel_key_u(sm.sc[tid], blk) : 0ull};
            block_sort_desc<1>(x, sm.cand);
            if (tid < kCap) part[((int64_t)bg * span_stride + span) * kCap + tid] = tid < K ? x[0] : 0ull;
        }
    }
    if (!grid_barrier(bar, gridDim.x, ctx, &sm.ok)) return;

    // ---------------------------------------------------------------- B: the group's slot list
    if (idx_in) {
        for (int s = tid; s < slots; s += kThreads) {
            int blk = idx_in[(int64_t)bg * slots + s];
            if (blk > c) {
                flag(ctx, kStatusBounds);
                blk = -1;
            }
            sm.sel[s] = blk;
        }
    } else if (!do_sel) {
        for (int s = tid; s < slots; s += kThreads) sm.sel[s] = s <= c ? s : -1;
    } else {
        if (K > 0) {
            // The group's top-k from the spans' first kPre keys: if no span has all kPre of its
            // loaded keys among the winners, no span can hide a winner further down its list, so
            // the k-th largest loaded key is the group's k-th key.  Otherwise (rare) merge the
            // spans' whole lists.
            constexpr int kPre = 8, kPreE = kMergeE * kPre / kCap;  // prefix keys per thread (spans <= 128)
            const unsigned long long* src =
                reinterpret_cast<const unsigned long long*>(part) + (int64_t)bg * span_stride * kCap;
            if (tid == 0) {
                sm.sel_n = 0;
                sm.overflow = 0;
            }
            if (nspan * kPre <= 2 * kThreads) {
                // up to 64 spans: sort the prefixes (two keys per thread); winners are the first k
                uint64_t x[2], k8[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int e = 2 * tid + i, span = e / kPre;
                    x[i] = span < nspan ? __ldcg(src + span * kCap + e % kPre) : 0ull;
                    k8[i] = e % kPre == kPre - 1 ? x[i] : 0ull;  // a span's last loaded key
                }
                block_sort_desc<2>(x, sm.cand);
                if (tid == (K - 1) / 2) sm.cand[0] = ((K - 1) & 1) ? x[1] : x[0];  // buf is free again
                __syncthreads();
                const uint64_t kth = sm.cand[0];  // the K-th best loaded key
                if (kth == 0ull || (k8[0] && k8[0] >= kth) || (k8[1] && k8[1] >= kth)) sm.overflow = 1;
                __syncthreads();
                if (!sm.overflow) {
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        if (2 * tid + i < K) sm.sel_top[2 * tid + i] = key_block(x[i]);
                }
            } else {
                uint64_t pk[kPreE];
#pragma unroll
                for (int e = 0; e < kPreE; ++e) {
                    const int i = e * kThreads + tid, span = i / kPre;
                    pk[e] = span < nspan ? __ldcg(src + span * kCap + i % kPre) : 0ull;
                }
                uint64_t prefix, mask;
                radix_kth<kPreE>(pk, K, sm.ss, prefix, mask, tid, [] { __syncthreads(); });
                if (tid == 0) sm.sel_n = 0;
                __syncthreads();
#pragma unroll
                for (int e = 0; e < kPreE; ++e) {
                    const int i = e * kThreads + tid;
                    if (pk[e] && (pk[e] & mask) >= prefix && i % kPre == kPre - 1) sm.overflow = 1;
                }
                __syncthreads();
                if (!sm.overflow) {
#pragma unroll
                    for (int e = 0; e < kPreE; ++e)
                        if (pk[e] && (pk[e] & mask) >= prefix) sm.sel_top[atomicAdd(&sm.sel_n, 1)] = key_block(pk[e]);
                }
            }
            if (sm.overflow) {
                uint64_t prefix, mask;
                uint64_t key[kMergeE];
                const int nk = nspan * kCap;
#pragma unroll
                for (int e = 0; e < kMergeE; ++e) {
                    const int i = e * kThreads + tid;
                    key[e] = i < nk ? __ldcg(src + i) : 0ull;
                }
                radix_kth<kMergeE>(key, K, sm.ss, prefix, mask, tid, [] { __syncthreads(); });
                if (tid == 0) sm.sel_n = 0;
                __syncthreads();
#pragma unroll
                for (int e = 0; e < kMergeE; ++e)
                    if (key[e] && (key[e] & mask) >= prefix) sm.sel_top[atomicAdd(&sm.sel_n, 1)] = key_block(key[e]);
            }
            __syncthreads();
        }
        if (warp == 0) {
            int x0 = 2 * lane < K ? sm.sel_top[2 * lane] : 0x7fffffff;
            int x1 = 2 * lane + 1 < K ? sm.sel_top[2 * lane + 1] : 0x7fffffff;
            warp_sort64(x0, x1, lane);
            for (int s = lane; s < n_init; s += 32) sm.sel[s] = s;
            if (2 * lane < K) sm.sel[n_init + 2 * lane] = x0;
            if (2 * lane + 1 < K) sm.sel[n_init + 2 * lane + 1] = x1;
            for (int t = lane; t < n_local; t += 32) sm.sel[n_init + K + t] = c - n_local + 1 + t;
            for (int s = n_init + K + n_local + lane; s < slots; s += 32) sm.sel[s] = -1;
        }
    }
    __syncthreads();
    if (idx_out && j == 0)
        for (int s = tid; s < slots; s += kThreads) idx_out[(int64_t)bg * slots + s] = sm.sel[s];

    // ---------------------------------------------------------------- C: per-slot partials
    // bf16: the two products on the tensor cores (warp-level m16n8k16, heads padded to 16 rows);
    // fp32: on CUDA cores in fp32.
    constexpr bool kTC = std::is_same<T, __nv_bfloat16>::value;
    if constexpr (kTC) {
        for (int e = tid; e < kMaxG * (D / 8); e += kThreads) {
            const int h = e / (D / 8), c8 = (e % (D / 8)) * 8;
            *reinterpret_cast<uint4*>(&sm.Qb[h][c8]) = h < G ? ld16(qg + h * D + c8) : make_uint4(0u, 0u, 0u, 0u);
        }
    } else {
        constexpr int kQIt = kMaxG * D / kThreads;
        float qv[kQIt];
#pragma unroll
        for (int u = 0; u < kQIt; ++u) {
            const int e = u * kThreads + tid;
            qv[u] = e < G * D ? to_f(qg[e]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kQIt; ++u) {
            const int e = u * kThreads + tid;
            if (e < G * D) sm.Q[e / D][e % D] = qv[u];
        }
    }
    constexpr int kStage = kBlk * (D / 8) / kThreads;  // 8-element pieces of K (and V) per thread
    for (int s = j; s < slots; s += cpg) {
        int blk = sm.sel[s];
        float* r = rec + ((int64_t)bg * slots + s) * G * (D + 2);
        // the block's 64 K and V rows: in the dense cache [B * Hkv][Tmax][D], or in the page the
        // sequence's table names for it ([n_pages][Hkv][64][D]); a bad page id is flagged and the
        // slot left empty
        const T* kblk = nullptr;
        const T* vblk = nullptr;
        if (blk >= 0) {
            if (pages) {
                const int pg = blk < max_pages ? __ldg(pages + b * max_pages + blk) : -1;
                if (pg < 0 || pg >= n_pages) {
                    if (tid == 0) flag(ctx, kStatusBounds);
                    blk = -1;
                } else {
                    kblk = kc + ((int64_t)pg * Hkv + g) * kBlk * D;
                    vblk = vc + ((int64_t)pg * Hkv + g) * kBlk * D;
                }
            } else {
                kblk = kc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
                vblk = vc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
            }
        }
        if (blk < 0) {
            for (int hh = tid; hh < G; hh += kThreads) {
                r[hh * (D + 2)] = -INFINITY;
                r[hh * (D + 2) + 1] = 0.f;
            }
            continue;
        }
        const int lim = min(kBlk - 1, pos_s - blk * kBlk);  // last visible key of the block
        constexpr int kU = 8 * sizeof(T) / 16;  // 16-byte pieces per 8 elements
        constexpr int kEl = 16 / sizeof(T);
        uint4 rk[kStage][kU], rv[kStage][kU];
#pragma unroll
        for (int u = 0; u < kStage; ++u) {  // every load issued before the first use
            const int e = u * kThreads + tid;
            const int row = e / (D / 8), c8 = (e % (D / 8)) * 8;
            const bool ok = row <= lim;
            const T* pk = kblk + (int64_t)row * D + c8;
            const T* pv = vblk + (int64_t)row * D + c8;
#pragma unroll
            for (int w = 0; w < kU; ++w) {
                rk[u][w] = ok ? ld16(pk + w * kEl) : make_uint4(0u, 0u, 0u, 0u);
                rv[u][w] = ok ? ld16(pv + w * kEl) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        __syncthreads();  // the previous slot's readers are done with K, V, P
#pragma unroll
        for (int u = 0; u < kStage; ++u) {
            const int e = u * kThreads + tid;
            const int row = e / (D / 8), c8 = (e % (D / 8)) * 8;
            if constexpr (kTC) {
                *reinterpret_cast<uint4*>(&sm.Kb[row][c8]) = rk[u][0];
                *reinterpret_cast<uint4*>(&sm.Vb[row][c8]) = rv[u][0];
            } else {
                float fk[8], fv[8];
#pragma unroll
                for (int w = 0; w < kU; ++w) {
                    cvt16<T>(rk[u][w], fk + w * kEl);
                    cvt16<T>(rv[u][w], fv + w * kEl);
                }
                *reinterpret_cast<float4*>(&sm.K[row][c8]) = make_float4(fk[0], fk[1], fk[2], fk[3]);
                *reinterpret_cast<float4*>(&sm.K[row][c8 + 4]) = make_float4(fk[4], fk[5], fk[6], fk[7]);
                *reinterpret_cast<float4*>(&sm.V[row][c8]) = make_float4(fv[0], fv[1], fv[2], fv[3]);
                *reinterpret_cast<float4*>(&sm.V[row][c8 + 4]) = make_float4(fv[4], fv[5], fv[6], fv[7]);
            }
        }
        __syncthreads();
        if constexpr (kTC) {
            // logits: warp w owns keys 8w .. 8w+7; A = Q (16 heads x 16 d), B = K rows (keys x d)
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const int n0 = 8 * warp;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t af[4], bf[2];
                ldsm_x4(af, &sm.Qb[lane & 15][16 * ks + (lane >> 4) * 8]);
                ldsm_x2(bf, &sm.Kb[n0 + (lane & 7)][16 * ks + ((lane >> 3) & 1) * 8]);
                mma16816(acc, af, bf);
            }
            const int hr = lane >> 2, key = n0 + 2 * (lane & 3);
            sm.P[hr][key] = key <= lim ? acc[0] * scale : -INFINITY;
            sm.P[hr][key + 1] = key + 1 <= lim ? acc[1] * scale : -INFINITY;
            sm.P[hr + 8][key] = key <= lim ? acc[2] * scale : -INFINITY;
            sm.P[hr + 8][key + 1] = key + 1 <= lim ? acc[3] * scale : -INFINITY;
        } else {
            // logits: thread = one key x four heads (K row read once for four heads)
            const int key = tid % kBlk, h0 = (tid / kBlk) * 4;
            if (h0 < G) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int dd = 0; dd < D; dd += 4) {
                    const float4 k4 = *reinterpret_cast<const float4*>(&sm.K[key][dd]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (h0 + i < G) {
                            const float4 q4 = *reinterpret_cast<const float4*>(&sm.Q[h0 + i][dd]);
                            acc[i] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, fmaf(q4.w, k4.w, acc[i]))));
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (h0 + i < G) sm.P[h0 + i][key] = key <= lim ? acc[i] * scale : -INFINITY;
            }
        }
        __syncthreads();
        for (int hh = warp; hh < G; hh += kThreads / 32) {
            const float s0 = sm.P[hh][lane], s1 = sm.P[hh][lane + 32];
            float m = fmaxf(s0, s1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            const float p0 = expf(s0 - m), p1 = expf(s1 - m);  // lim >= 0, so m is finite
            float l = p0 + p1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
            sm.P[hh][lane] = p0;
            sm.P[hh][lane + 32] = p1;
            if constexpr (kTC) {
                sm.Pb[hh][lane] = __float2bfloat16_rn(p0);
                sm.Pb[hh][lane + 32] = __float2bfloat16_rn(p1);
            }
            if (lane == 0) {
                sm.m[hh] = m;
                sm.l[hh] = l;
            }
        }
        if constexpr (kTC) {  // padding heads: zero probabilities (their rows are never written)
            for (int e = tid; e < (kMaxG - G) * kBlk; e += kThreads)
                sm.Pb[G + e / kBlk][e % kBlk] = __float2bfloat16_rn(0.f);
        }
        __syncthreads();
        if constexpr (kTC) {
            // p v: warp w owns columns 16w .. 16w+15 of d (two n-tiles; D = 64 uses warps 0-3);
            // A = P (16 heads x 16 keys), B = V (16 keys x 8 columns, transposed on load)
            constexpr int kNT = D / 8 / (kThreads / 32);  // n-tiles per warp
            if (warp * kNT * 8 < D) {
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int ks = 0; ks < kBlk / 16; ++ks) {
                    uint32_t af[4];
                    ldsm_x4(af, &sm.Pb[lane & 15][16 * ks + (lane >> 4) * 8]);
#pragma unroll
                    for (int t = 0; t < (kNT > 0 ? kNT : 1); ++t) {
                        uint32_t bf[2];
                        ldsm_x2_t(bf, &sm.Vb[16 * ks + (lane & 15)][(warp * kNT + t) * 8]);
                        mma16816(acc[t], af, bf);
                    }
                }
                const int hr = lane >> 2;
#pragma unroll
                for (int t = 0; t < (kNT > 0 ? kNT : 1); ++t) {
                    const int col = (warp * kNT + t) * 8 + 2 * (lane & 3);
                    if (hr < G) {
                        r[hr * (D + 2) + 2 + col] = acc[t][0];
                        r[hr * (D + 2) + 3 + col] = acc[t][1];
                    }
                    if (hr + 8 < G) {
                        r[(hr + 8) * (D + 2) + 2 + col] = acc[t][2];
                        r[(hr + 8) * (D + 2) + 3 + col] = acc[t][3];
                    }
                }
            }
            if (tid < G) {
                r[tid * (D + 2)] = sm.m[tid];
                r[tid * (D + 2) + 1] = sm.l[tid];
            }
        } else {
            // p v: thread = four columns x the heads hp, hp + ngrp, ... (V read once for them)
            constexpr int kQuads = D / 4, kGroups = kThreads / kQuads;
            const int dq = tid % kQuads, hp = tid / kQuads;
            for (int h0 = hp; h0 < G; h0 += 2 * kGroups) {
                const int h1 = h0 + kGroups;
                float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 8
                for (int key = 0; key < kBlk; ++key) {
                    const float4 v4 = *reinterpret_cast<const float4*>(&sm.V[key][4 * dq]);
                    const float p0 = sm.P[h0][key];
                    a0.x = fmaf(p0, v4.x, a0.x); a0.y = fmaf(p0, v4.y, a0.y);
                    a0.z = fmaf(p0, v4.z, a0.z); a0.w = fmaf(p0, v4.w, a0.w);
                    if (h1 < G) {
                        const float p1 = sm.P[h1][key];
                        a1.x = fmaf(p1, v4.x, a1.x); a1.y = fmaf(p1, v4.y, a1.y);
                        a1.z = fmaf(p1, v4.z, a1.z); a1.w = fmaf(p1, v4.w, a1.w);
                    }
                }
                float* r0 = r + h0 * (D + 2);
                r0[2 + 4 * dq] = a0.x; r0[3 + 4 * dq] = a0.y; r0[4 + 4 * dq] = a0.z; r0[5 + 4 * dq] = a0.w;
                if (dq == 0) { r0[0] = sm.m[h0]; r0[1] = sm.l[h0]; }
                if (h1 < G) {
                    float* r1 = r + h1 * (D + 2);
                    r1[2 + 4 * dq] = a1.x; r1[3 + 4 * dq] = a1.y; r1[4 + 4 * dq] = a1.z; r1[5 + 4 * dq] = a1.w;
                    if (dq == 0) { r1[0] = sm.m[h1]; r1[1] = sm.l[h1]; }
                }
            }
        }
    }
    if (!grid_barrier(bar, gridDim.x, ctx, &sm.ok)) return;

    // ---------------------------------------------------------------- D: combine
    // Warp w folds slots w, w + 8, ...; all of its records are loaded before the first use.
    constexpr int kPerWarp = (kMaxSlots + 7) / 8;
    for (int item = j; item < G * (D / 32); item += cpg) {
        const int hh = item / (D / 32), d0 = (item % (D / 32)) * 32;
        float ms[kPerWarp], ls[kPerWarp], os[kPerWarp];
#pragma unroll
        for (int i = 0; i < kPerWarp; ++i) {
            const int s = warp + 8 * i;
            if (s < slots) {
                const float* r = rec + (((int64_t)bg * slots + s) * G + hh) * (D + 2);
                ms[i] = __ldcg(r);
                ls[i] = __ldcg(r + 1);
                os[i] = __ldcg(r + 2 + d0 + lane);
            } else {
                ms[i] = -INFINITY;
                ls[i] = os[i] = 0.f;
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < kPerWarp; ++i) M = fmaxf(M, ms[i]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int i = 0; i < kPerWarp; ++i) {
                if (ms[i] == -INFINITY) continue;
                const float w8 = expf(ms[i] - M);
                L = fmaf(ls[i], w8, L);
                acc = fmaf(os[i], w8, acc);
            }
        }
        sm.cm[warp][lane] = M;
        sm.cl[warp][lane] = L;
        sm.co[warp][lane] = acc;
        __syncthreads();
        if (warp == 0) {
            float Mt = -INFINITY;
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) Mt = fmaxf(Mt, sm.cm[w][lane]);
            float Lt = 0.f, At = 0.f;
            if (Mt != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kThreads / 32; ++w) {
                    if (sm.cm[w][lane] == -INFINITY) continue;
                    const float a = expf(sm.cm[w][lane] - Mt);
                    Lt += a * sm.cl[w][lane];
                    At += a * sm.co[w][lane];
                }
            }
            o[(b * H + (int64_t)g * G + hh) * D + d0 + lane] = from_f<T>(Lt > 0.f ? At / Lt : 0.f);
        }
        __syncthreads();
    }
}

// Workspace of the one-launch path: [0, 256) barrier word ([256, 512) belongs to the prefetching
// path's epoch), then per (batch, group, span) the span's top-k keys, then the per-slot partial
// records.
struct FusedLayout {
    size_t part, rec, total;
};
FusedLayout fused_layout(int B, int H, int Hkv, int nspan, int slots, int d) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    FusedLayout L;
    L.part = 512;
    L.rec = L.part + up((size_t)B * Hkv * nspan * kCap * sizeof(uint64_t));
    L.total = L.rec + (size_t)B * Hkv * slots * (H / Hkv) * (d + 2) * sizeof(float);
    return L;
}

template <typename T, int D>
cudaError_t fused(const void* q, const void* kc, const void* vc, const void* kbar,
                  const int32_t* idx_in, int32_t* idx_out, void* o, int B, int H, int Hkv, int pos,
                  int Tmax, int nb_cap, int topk, int n_init, int n_local, float scale, void* ws,
                  size_t ws_bytes, DecodePaging pg, cudaStream_t st, DevCtx ctx) {
    const int slots = n_init + n_local + topk;
    const int G = H / Hkv;
    const int c = pos / kBlk;
    const int ncand = c - n_local - n_init + 1;
    const int nspan = ncand > topk ? (ncand + kSpan - 1) / kSpan : 0;
    if (topk > kCap || slots > kMaxSlots || G > kMaxG || nspan * kCap > kMergeE * kThreads)
        return cudaErrorNotSupported;
    auto kern = sparse_decode_fused_kernel<T, D>;
    const int smem = (int)sizeof(DecSmem<D>);
    // resident CTAs per SM and SM count, per device (a process may drive several GPUs from
    // several threads); read into locals under the lock
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static int occ_of[kMaxDev] = {}, nsm_of[kMaxDev] = {};
    int occ = 0, nsm = 0;
    {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDev) return cudaErrorNotSupported;
        std::lock_guard<std::mutex> lk(mu);
        if (occ_of[dev] == 0) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            int o = 0, n = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kThreads, smem);
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            if (o < 1) return cudaErrorNotSupported;
            occ_of[dev] = o;
            nsm_of[dev] = n;
        }
        occ = occ_of[dev];
        nsm = nsm_of[dev];
    }
    const int groups = B * Hkv;
    const int cap = occ * nsm / groups;
    const int want = max(max(nspan, slots), G * (D / 32));
    const int cpg = min(cap, want);
    if (cpg < 1) return cudaErrorNotSupported;
    const FusedLayout lay = fused_layout(B, H, Hkv, nspan, slots, D);
    if (lay.total > ws_bytes) return cudaErrorNotSupported;
    unsigned char* w = static_cast<unsigned char*>(ws);
    uint64_t* part = reinterpret_cast<uint64_t*>(w + lay.part);
    float* rec = reinterpret_cast<float*>(w + lay.rec);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(groups * cpg));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(kc),
                              static_cast<const T*>(vc), static_cast<const T*>(kbar), idx_in, idx_out,
                              static_cast<T*>(o), H, Hkv, pos, Tmax, nb_cap, topk, n_init, n_local,
                              slots, scale, cpg, nspan, pg.pos_b, pg.pages, pg.max_pages, pg.n_pages,
                              reinterpret_cast<unsigned*>(w), part, rec, ctx);
}

}  // namespace

size_t sparse_decode_fused_workspace(int B, int H, int Hkv, int pos, int topk, int n_init,
                                     int n_local, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || pos < 0) return 0;
    const int slots = n_init + n_local + topk;
    const int ncand = pos / kBlk - n_local - n_init + 1;
    const int nspan = ncand > topk ? (ncand + kSpan - 1) / kSpan : 0;
    return fused_layout(B, H, Hkv, nspan, slots, d).total;
}

cudaError_t launch_sparse_decode_fused(DType dt, const void* q, const void* kc, const void* vc,
                                       const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                       void* o, int B, int H, int Hkv, int pos, int Tmax,
                                       int nb_cap, int d, int topk, int n_init, int n_local,
                                       float scale, void* ws, size_t ws_bytes, DecodePaging pg,
                                       cudaStream_t st, DevCtx ctx) {
    if (dt == DType::F32)
        return d == 64 ? fused<float, 64>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init, n_local, scale, ws, ws_bytes, pg, st, ctx)
                       : fused<float, 128>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init, n_local, scale, ws, ws_bytes, pg, st, ctx);
    return d == 64 ? fused<__nv_bfloat16, 64>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init, n_local, scale, ws, ws_bytes, pg, st, ctx)
                   : fused<__nv_bfloat16, 128>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init, n_local, scale, ws, ws_bytes, pg, st, ctx);
}

}  // namespace sala
