// Sparse decode with the block-key table prefetched: block scoring, top-k selection and attention
// for one query token per (batch, KV group) in one launch, bf16, d = 64 or 128.
//
// The step reads two things: the whole block-key table k_bar of the group (8 MiB at 2^20 tokens
// and 2 KV heads) to score the candidates, and the ~67 selected K/V blocks (4 MiB) to attend.  The
// k_bar table does not depend on the query, so each CTA starts copying its share of it into shared
// memory (16-byte asynchronous copies from every thread) as soon as it runs -- before
// griddepcontrol.wait when the call is launched as a programmatic dependent, i.e. while the
// previous layer's kernel is still running.  Rows are dealt to the group's `cpg` CTAs in 4-row
// chunks, round robin, so blocks that are chosen together (recent context, a run of related
// blocks) land in different CTAs.
//
//   A  every CTA scores its rows on the tensor cores (the group-summed query split into bf16
//      hi + lo rows of an m16n8k16 tile against 8 k_bar rows at a time), keeps its best kPub + 1
//      selection keys (orderable score above the inverted block index: distinct, larger = better,
//      ties to the lower block) by counting ranks, and publishes them.
//   B  every CTA reads the group's published lists U (kPub keys per CTA) and ranks its own kPub
//      keys within U: a key of rank r < k is the group's (r+1)-th best block.  This is exact unless
//      some CTA has more than kPub winners: with X = the largest (kPub+1)-th key of any CTA, no
//      unpublished key can beat X, so when fewer than k keys of U exceed X (X would win), the lists
//      may hide winners and all CTAs of the group (they see the same U) take the fallback: all keys
//      published, an exact radix select over them.  Otherwise every published key of rank < k is a
//      winner and every other key is not.
//   C  each CTA attends the blocks it owns -- its own winners (record slot = rank) and, in the
//      last CTAs, the init and local blocks (slots k ..) -- or, on the list paths (given
//      selection, at most k candidates, k = 0, fallback), slots j, j + cpg, ...: the K and V of
//      every owned block requested at once (16-byte asynchronous copies into stages that reuse the
//      k_bar rows' shared memory), the G heads' logits and p v on warp-level tensor-core tiles, a
//      per-head softmax partial (max, sum, sum of p v) per slot.
//   D  the group's CTAs combine the partials, one (head, 32-column) piece each, in slot order;
//      CTA 0 writes idx_out (blocks ascending).
//
// The exchanges between A and B and between C and D need no barrier: every word another CTA
// reads is a tagged 8-byte word (32 bits of data above a 32-bit tag, written and read as one
// single-copy-atomic access), and a reader spins, bounded, until every word it needs carries this
// call's tag.  The tag is a signalling-NaN bit pattern (0x7F800001 + epoch mod 2^22 - 1); the epoch
// is a word at a fixed place in the workspace that every CTA reads after griddepcontrol.wait and
// CTA 0 advances once it has seen every CTA's tagged word (each CTA tags one word right after
// reading the epoch), so the next call on the workspace uses a new tag; a CTA that gives up on a
// wait advances it too.  A stale word therefore never carries the current tag, whatever layout the
// call that wrote it had (within 2^22 - 1 calls), and no value the other decode paths store in the
// same bytes (fp32 results, which arithmetic never makes signalling NaNs, block indices, counts)
// looks like a tag, so this path's region may overlap theirs.
#include <mutex>

#include "blocksel.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sala {
namespace {

using namespace dec;

constexpr int kBlk = 64;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCap = 64;         // largest k
constexpr int kMaxSlots = 80;    // n_init + n_local + k
constexpr int kMaxG = 16;
constexpr int kPub = 8;          // keys per CTA ranked on the fast path
constexpr int kPubWords = 32;    // tagged words per CTA's list: 2 per key (kPub + 1 keys), padding
constexpr int kPubCopies = 8;    // copies of every list, so that no line is read by every CTA
constexpr int kMaxCpg = 160;     // CTAs per group (a B200 has 148 SMs)
constexpr int kMaxGroups = 64;
constexpr int kChunk = 4;        // rows per round-robin chunk
constexpr int kMaxStages = 5;    // K|V stages of phase C

constexpr int kRowsMax = kThreads;  // k_bar rows a CTA scores: 32 per warp (four 8-row tiles)
template <int D>
constexpr int row_elems() { return D + 8; }  // padded rows: conflict-free ldmatrix
template <int D>
constexpr size_t stage_bytes() { return (size_t)2 * kBlk * row_elems<D>() * 2; }

template <int D>
struct PfSmem {
    __nv_bfloat16 Qb[kMaxG][D + 8];
    __nv_bfloat16 QS[16][D + 8];  // scoring A tile: row 0 bf16(qbar), row 1 the bf16 residual, others 0
    uint64_t wtop[kWarps][kPub + 1];  // per-warp best keys, largest first (0: none)
    uint64_t own[kPub + 1];           // this CTA's best keys, largest first
    uint64_t query[kPub + 1];         // keys ranked in phase B (own[0 .. kPub-1], X)
    int rpart[kWarps][kPub + 1];
    int rank[kPub + 1];
    uint64_t xmax[kWarps];
    int work_slot[kMaxSlots], work_blk[kMaxSlots];
    int nwork;
    int sel[kMaxSlots];
    uint64_t wkeys[kCap];
    int nwin;
    RadixSelSmem ss;
    int bad;
    float cm[8][32], cl[8][32], co[8][32];
};
// After the fixed part: the CTA's keys (kRowsMax of them), then one region holding first its
// k_bar rows (kRowsMax padded rows; rows past rcap are read by the scoring tiles but never kept)
// and later the K|V stages of phase C.
template <int D>
constexpr size_t pf_keys_off() { return (sizeof(PfSmem<D>) + 15) & ~(size_t)15; }
template <int D>
constexpr size_t pf_region_off() { return (pf_keys_off<D>() + (size_t)kRowsMax * 8 + 127) & ~(size_t)127; }
template <int D>
constexpr size_t pf_region_bytes(int rcap, int nstages) {
    const size_t a = (size_t)(rcap > 0 ? kRowsMax : 0) * row_elems<D>() * 2, b = (size_t)nstages * stage_bytes<D>();
    return a > b ? a : b;
}
template <int D>
constexpr size_t pf_smem_bytes(int rcap, int nstages) { return pf_region_off<D>() + pf_region_bytes<D>(rcap, nstages); }

// ---------------------------------------------------------------- tagged words
__device__ __forceinline__ uint64_t ll_word(uint32_t v, uint32_t tag) { return ((uint64_t)v << 32) | tag; }
__device__ __forceinline__ void ll_st(uint64_t* p, uint64_t w) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void ll_st2(uint64_t* p, uint64_t a, uint64_t b) {  // p 16-byte aligned
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
// Reads of other CTAs' words are strong (gpu-scope relaxed): a weak load may be served from a copy
// that is never refreshed and would not see the writer's update.
__device__ __forceinline__ uint64_t ll_ld(const uint64_t* p) {
    uint64_t w;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}
__device__ __forceinline__ void ll_ld2(const uint64_t* p, uint64_t& a, uint64_t& b) {  // p 16-byte aligned
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ bool ll_ok(uint64_t w, uint32_t tag) { return (uint32_t)w == tag; }
__device__ __forceinline__ uint32_t ll_val(uint64_t w) { return (uint32_t)(w >> 32); }

// Spins until every word addr(i) (i < n, n <= N) carries the tag; fills w[]; on expiry sets *bad
// and returns false.  Every round issues all n loads before looking at any of them (no branch on a
// loaded value between the loads: a GPU does not run past such a branch, so checking each word as
// it arrives would serialise the round trips).
template <int N, typename Addr>
__device__ __forceinline__ bool ll_wait_all(Addr addr, int n, uint64_t (&w)[N], uint32_t tag, const DevCtx& ctx,
                                            int* bad) {
    if (n <= 0) return true;
    uint64_t t0 = 0;
    while (true) {
#pragma unroll
        for (int i = 0; i < N; ++i) w[i] = ll_ld(addr(i < n ? i : n - 1));
        unsigned miss = 0u;
#pragma unroll
        for (int i = 0; i < N; ++i) miss |= (unsigned)((uint32_t)w[i] != tag);
        if (miss == 0u) return true;
        const uint64_t t = globaltimer_ns();
        if (t0 == 0) t0 = t;
        if (*bad || t - t0 > ctx.wait_limit_ns) {
            *bad = 1;
            return false;
        }
    }
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, x, off);
        x = y > x ? y : x;
    }
    return x;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Exact k-th largest nonzero key among n keys in global memory (the fallback of phase B): one byte
// at a time from the top, as radix_kth, streaming the keys from memory on every pass.  On return
// winner(key) = key != 0 && (key & mask) >= prefix picks min(K, #nonzero) keys.
__device__ void radix_kth_stream(const uint64_t* keys, int n, int K, RadixSelSmem& s, uint64_t& prefix,
                                 uint64_t& mask, int t) {
    const int lane = t & 31, warp = t >> 5;
    int nv = 0;
    for (int e = t; e < n; e += kThreads) nv += __ldcg(keys + e) != 0ull;
    if (t == 0) s.nvalid = 0;
    __syncthreads();
    nv = __reduce_add_sync(0xffffffffu, nv);
    if (lane == 0 && nv) atomicAdd(&s.nvalid, nv);
    __syncthreads();
    prefix = 0;
    mask = 0;
    if (s.nvalid <= K) {
        prefix = 1;
        mask = ~0ull;
        return;
    }
    int krem = K;
    for (int shift = 56; shift >= 0; shift -= 8) {
        s.hist[t] = 0;
        __syncthreads();
        for (int e = t; e < n; e += kThreads) {
            const uint64_t key = __ldcg(keys + e);
            if (key && (key & mask) == prefix) atomicAdd(&s.hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            int cnt[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cnt[i] = (int)s.hist[255 - 8 * lane - i];
                sum += cnt[i];
            }
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            const int excl = incl - sum;
            if (excl < krem && krem <= incl) {
                int run = excl;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run + cnt[i] >= krem) {
                        s.d = 255 - 8 * lane - i;
                        s.above = run;
                        s.eq = cnt[i];
                        break;
                    }
                    run += cnt[i];
                }
            }
        }
        __syncthreads();
        krem -= s.above;
        prefix |= (uint64_t)s.d << shift;
        mask |= 0xFFull << shift;
        if (s.eq == krem) break;
    }
}

// Workspace region of this path (zeroed before its first use): one tagged word per CTA (it has
// read the epoch), the published lists, the fallback's keys and arrival words, the owners' block
// ids per slot and the per-slot partial records, all tagged but the fallback keys.
struct PfLayout {
    size_t alive, part, keys, fb, blkid, rec, total;
};
PfLayout pf_layout(int groups, int ncand, int slots, int G, int d) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    PfLayout L;
    L.alive = 0;
    L.part = L.alive + up((size_t)groups * kMaxCpg * 8);
    L.keys = L.part + up((size_t)groups * kPubCopies * kMaxCpg * kPubWords * 8);
    L.fb = L.keys + up((size_t)groups * (ncand > 0 ? ncand : 1) * 8);
    L.blkid = L.fb + up((size_t)groups * kMaxCpg * 8);
    L.rec = L.blkid + up((size_t)groups * kMaxSlots * 8);
    L.total = L.rec + (size_t)groups * slots * G * (d + 2) * 8;
    return L;
}

// One slot's softmax partial, computed by one warp: the block's K and V rows (64 x D, padded rows)
// in shared memory, the G <= 16 query rows in sm.Qb (padded to 16 with zeros).  The logits are an
// m16n8k16 tile row per head (16 x 64), the softmax runs in registers (a head's row lives in the 4
// lanes of a quad), and P -- rounded to bf16 -- becomes the A fragments of P V directly.  Writes
// the record [G][m, l, o_0 .. o_{D-1}] as tagged words, o unnormalised.
template <int D>
__device__ __forceinline__ void slot_partial(const __nv_bfloat16* __restrict__ Qs, const __nv_bfloat16* __restrict__ Ks,
                                             const __nv_bfloat16* __restrict__ Vs, int lim, float scale_log2, int G,
                                             uint64_t* r, uint32_t tag, int lane) {
    constexpr int RE = row_elems<D>();
    const int gq = lane >> 2, t2 = 2 * (lane & 3), mi = lane >> 3, r8 = lane & 7;
    float sc[8][4];
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) sc[jn][0] = sc[jn][1] = sc[jn][2] = sc[jn][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, Qs + (lane & 15) * RE + 16 * ks + (lane >> 4) * 8);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            uint32_t b4[4];
            ldsm_x4(b4, Ks + (16 * jj + (mi >> 1) * 8 + r8) * RE + 16 * ks + (mi & 1) * 8);
            const uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
            mma16816(sc[2 * jj], a, b0);
            mma16816(sc[2 * jj + 1], a, b1);
        }
    }
    // rows gq and gq + 8; keys 8 jn + t2 (+1); logits in log2 units
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const bool ok = 8 * jn + t2 + u <= lim;
            sc[jn][u] = ok ? sc[jn][u] * scale_log2 : -INFINITY;
            sc[jn][2 + u] = ok ? sc[jn][2 + u] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[jn][u]);
            mx1 = fmaxf(mx1, sc[jn][2 + u]);
        }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // lim >= 0, so every row has a finite maximum
    float l0 = 0.f, l1 = 0.f;
    uint32_t pa[4][4];  // A fragments of P for the 4 key steps of P V
#pragma unroll
    for (int jn = 0; jn < 8; ++jn) {
        const float p0 = exp2f(sc[jn][0] - mx0), p1 = exp2f(sc[jn][1] - mx0);
        const float p2 = exp2f(sc[jn][2] - mx1), p3 = exp2f(sc[jn][3] - mx1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        pa[jn >> 1][(jn & 1) * 2] = pack_bf16(p0, p1);
        pa[jn >> 1][(jn & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    // P V in halves of D/2 columns (or all of D = 64): ldmatrix.trans of V gives both B fragments
    // of two column tiles at once
    constexpr int kHalf = D >= 128 ? 64 : D;
#pragma unroll
    for (int h0 = 0; h0 < D; h0 += kHalf) {
        float ov[kHalf / 8][4];
#pragma unroll
        for (int n = 0; n < kHalf / 8; ++n) ov[n][0] = ov[n][1] = ov[n][2] = ov[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int nn = 0; nn < kHalf / 16; ++nn) {
                uint32_t b4[4];
                ldsm_x4_t(b4, Vs + (16 * kk + (mi & 1) * 8 + r8) * RE + h0 + 16 * nn + (mi >> 1) * 8);
                const uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
                mma16816(ov[2 * nn], pa[kk], b0);
                mma16816(ov[2 * nn + 1], pa[kk], b1);
            }
        }
#pragma unroll
        for (int n = 0; n < kHalf / 8; ++n) {
            const int col = h0 + 8 * n + t2;
            if (gq < G)
                ll_st2(r + gq * (D + 2) + 2 + col, ll_word(__float_as_uint(ov[n][0]), tag),
                       ll_word(__float_as_uint(ov[n][1]), tag));
            if (gq + 8 < G)
                ll_st2(r + (gq + 8) * (D + 2) + 2 + col, ll_word(__float_as_uint(ov[n][2]), tag),
                       ll_word(__float_as_uint(ov[n][3]), tag));
        }
    }
    // the running maximum is kept in log2 units; the combine takes exponents base 2
    if ((lane & 3) == 0) {
        if (gq < G) ll_st2(r + gq * (D + 2), ll_word(__float_as_uint(mx0), tag), ll_word(__float_as_uint(l0), tag));
        if (gq + 8 < G)
            ll_st2(r + (gq + 8) * (D + 2), ll_word(__float_as_uint(mx1), tag), ll_word(__float_as_uint(l1), tag));
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
sparse_decode_pf_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                        const __nv_bfloat16* __restrict__ vc, const __nv_bfloat16* __restrict__ kbar,
                        const int32_t* __restrict__ idx_in, int32_t* __restrict__ idx_out,
                        __nv_bfloat16* __restrict__ o, int H, int Hkv, int pos, int Tmax, int nb_cap,
                        int topk, int n_init, int n_local, int slots, float scale, int cpg, int rcap,
                        int nstages, unsigned* epoch, unsigned char* ws, PfLayout lay, DevCtx ctx) {
    extern __shared__ __align__(128) unsigned char pf_smem_raw[];
    PfSmem<D>& sm = *reinterpret_cast<PfSmem<D>*>(pf_smem_raw);
    uint64_t* s_keys = reinterpret_cast<uint64_t*>(pf_smem_raw + pf_keys_off<D>());
    __nv_bfloat16* s_region = reinterpret_cast<__nv_bfloat16*>(pf_smem_raw + pf_region_off<D>());
    constexpr int RE = row_elems<D>();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / Hkv;
    const int bg = blockIdx.x / cpg, j = blockIdx.x % cpg;
    const int64_t b = bg / Hkv;
    const int g = bg % Hkv;
    const int c = pos / kBlk;
    const int lo = n_init, hi = c - n_local;
    const int ncand = hi - lo + 1;
    const int K = topk;
    // owner mode: the selection is made here and the CTAs attend their own winners
    const bool owner = idx_in == nullptr && K > 0 && ncand > K;
    const int nchunks = owner ? (ncand + kChunk - 1) / kChunk : 0;
    const int my_chunks = j < nchunks ? (nchunks - 1 - j) / cpg + 1 : 0;
    const int nrows = my_chunks * kChunk;  // <= rcap <= kRowsMax
    const __nv_bfloat16* qg = q + (b * H + (int64_t)g * G) * D;
    uint64_t* alive = reinterpret_cast<uint64_t*>(ws + lay.alive);
    uint64_t* part = reinterpret_cast<uint64_t*>(ws + lay.part) + (int64_t)bg * kPubCopies * kMaxCpg * kPubWords;
    uint64_t* gkeys = reinterpret_cast<uint64_t*>(ws + lay.keys) + (int64_t)bg * (ncand > 0 ? ncand : 1);
    uint64_t* fbw = reinterpret_cast<uint64_t*>(ws + lay.fb) + (int64_t)bg * kMaxCpg;
    uint64_t* done = reinterpret_cast<uint64_t*>(ws + lay.blkid) + (int64_t)bg * kMaxSlots;
    uint64_t* rec = reinterpret_cast<uint64_t*>(ws + lay.rec) + (int64_t)bg * slots * G * (D + 2);

    // ---------------------------------------------------------------- prefetch of k_bar
    if (owner && my_chunks > 0) {
        const __nv_bfloat16* kb = kbar + ((int64_t)bg * nb_cap + lo) * D;
        for (int e = tid; e < nrows * (D / 8); e += kThreads) {
            const int r = e / (D / 8), piece = e % (D / 8);
            const int cand = (j + (r / kChunk) * cpg) * kChunk + r % kChunk;
            const bool ok = cand < ncand;
            ptx::cp_async16(s_region + (size_t)r * RE + piece * 8,
                            kb + (ok ? (int64_t)cand * D + piece * 8 : 0), ok);
        }
    }
    ptx::cp_async_commit();
    // The next kernel in the stream may start now (it waits for this grid before reading anything
    // this grid writes); this kernel's own reads of q, the cache, idx_in and the workspace wait for
    // the previous kernel when it was launched as a programmatic dependent.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const uint32_t tag = 0x7F800001u + __ldcg(epoch) % 0x3FFFFFu;  // 0x7F800001 .. 0x7FBFFFFF
    if (tid == 0) {
        sm.bad = 0;
        ll_st(alive + blockIdx.x, ll_word(1u, tag));
    }
    int* bad = &sm.bad;
    // ---------------------------------------------------------------- the group's query rows
    for (int e = tid; e < kMaxG * (D / 8); e += kThreads) {
        const int h = e / (D / 8), c8 = (e % (D / 8)) * 8;
        *reinterpret_cast<uint4*>(&sm.Qb[h][c8]) = h < G ? ld16(qg + h * D + c8) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    bool fallback = false;
    if (owner) {
        if (tid < D) {
            float s = 0.f;
            for (int h = 0; h < G; ++h) s += __bfloat162float(sm.Qb[h][tid]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(s);
            sm.QS[0][tid] = hi;
            sm.QS[1][tid] = __float2bfloat16_rn(s - __bfloat162float(hi));
        }
        for (int e = tid; e < 14 * (D / 8); e += kThreads)
            *reinterpret_cast<uint4*>(&sm.QS[2 + e / (D / 8)][(e % (D / 8)) * 8]) = make_uint4(0u, 0u, 0u, 0u);
        if (tid <= kPub) sm.own[tid] = 0ull;
        if (lane <= kPub) sm.wtop[warp][lane] = 0ull;
        ptx::cp_async_wait<0>();
        __syncthreads();
        // ------------------------------------------------------------ A: scores of this CTA's rows
        // Warp w scores rows 32w .. 32w+31 as four 8-row tiles at once.  A operand: the QS tile
        // (row 0 = bf16(qbar), row 1 = bf16(qbar - row 0), the other rows zero), so the two rows
        // of the result hold the hi and lo parts of each score.
        {
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t af[4];
                ldsm_x4(af, &sm.QS[lane & 15][16 * ks + (lane >> 4) * 8]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t bfr[2];
                    ldsm_x2(bfr, s_region + (size_t)(32 * warp + 8 * i + (lane & 7)) * RE + 16 * ks + ((lane >> 3) & 1) * 8);
                    mma16816(acc[i], af, bfr);
                }
            }
            // lanes 0-3: row 0 (hi) at columns 2t, 2t+1 of each tile; lanes 4-7: row 1 (lo)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float s0 = acc[i][0] + __shfl_down_sync(0xffffffffu, acc[i][0], 4);
                const float s1 = acc[i][1] + __shfl_down_sync(0xffffffffu, acc[i][1], 4);
                if (lane < 4) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int r = 32 * warp + 8 * i + 2 * lane + u;
                        const int cand = (j + (r / kChunk) * cpg) * kChunk + r % kChunk;
                        s_keys[r] = r < nrows && cand < ncand ? sel_key(u ? s1 : s0, lo + cand) : 0ull;
                    }
                }
            }
        }
        __syncwarp();
        // best kPub + 1 keys of the warp's 32 by counting ranks (keys are distinct), then of the
        // CTA from the warps' lists
        {
            const uint64_t x = s_keys[32 * warp + lane];
            const ulonglong2* kv = reinterpret_cast<const ulonglong2*>(s_keys + 32 * warp);
            int n = 0;
#pragma unroll
            for (int y = 0; y < 16; ++y) {
                const ulonglong2 pr = kv[y];
                n += (pr.x > x) + (pr.y > x);
            }
            if (x != 0ull && n <= kPub) sm.wtop[warp][n] = x;
        }
        __syncthreads();
        if (tid < kWarps * (kPub + 1)) {
            const uint64_t* wt = &sm.wtop[0][0];
            const uint64_t x = wt[tid];
            int n = 0;
#pragma unroll 8
            for (int y = 0; y < kWarps * (kPub + 1); ++y) n += wt[y] > x;
            if (x != 0ull && n <= kPub) sm.own[n] = x;
        }
        __syncthreads();
        if (tid < kPubCopies * (kPub + 1)) {  // publish: two tagged words per key, in every copy
            const int t = tid % (kPub + 1), cp = tid / (kPub + 1);
            const uint64_t x = sm.own[t];
            ll_st2(part + ((int64_t)cp * kMaxCpg + j) * kPubWords + 2 * t, ll_word((uint32_t)(x >> 32), tag),
                   ll_word((uint32_t)x, tag));
        }

        // ------------------------------------------------------------ B: rank own keys within U
        // thread i < cpg reads list i (its kPub keys and the next one), polling until every word
        // carries this call's tag, and counts its keys above each of this CTA's keys
        int cnt[kPub + 1];
        uint64_t x = 0, ukey[kPub];
#pragma unroll
        for (int qq = 0; qq <= kPub; ++qq) cnt[qq] = 0;
#pragma unroll
        for (int t = 0; t < kPub; ++t) ukey[t] = 0ull;
        if (tid < cpg) {
            uint64_t w[2 * (kPub + 1)];
            const uint64_t* lst = part + ((int64_t)(j % kPubCopies) * kMaxCpg + tid) * kPubWords;
            {  // the list's words are their own readiness flags: one round trip after they land
                uint64_t t0 = 0;
                while (true) {
#pragma unroll
                    for (int i = 0; i <= kPub; ++i) ll_ld2(lst + 2 * i, w[2 * i], w[2 * i + 1]);
                    unsigned miss = 0u;
#pragma unroll
                    for (int i = 0; i < 2 * (kPub + 1); ++i) miss |= (unsigned)((uint32_t)w[i] != tag);
                    if (miss == 0u) break;
                    const uint64_t t = globaltimer_ns();
                    if (t0 == 0) t0 = t;
                    if (*bad || t - t0 > ctx.wait_limit_ns) {
                        *bad = 1;
                        break;
                    }
                }
            }
            uint64_t mine[kPub];
#pragma unroll
            for (int qq = 0; qq < kPub; ++qq) mine[qq] = sm.own[qq];
#pragma unroll
            for (int t = 0; t < kPub; ++t) {
                ukey[t] = ((uint64_t)ll_val(w[2 * t]) << 32) | ll_val(w[2 * t + 1]);
#pragma unroll
                for (int qq = 0; qq < kPub; ++qq) cnt[qq] += ukey[t] > mine[qq];
            }
            x = ((uint64_t)ll_val(w[2 * kPub]) << 32) | ll_val(w[2 * kPub + 1]);
        }
        x = warp_max_u64(x);
        if (lane == 0) sm.xmax[warp] = x;
#pragma unroll
        for (int qq = 0; qq < kPub; ++qq) {
            const int n = __reduce_add_sync(0xffffffffu, cnt[qq]);
            if (lane == 0) sm.rpart[warp][qq] = n;
        }
        __syncthreads();
        if (sm.bad) {
            if (tid == 0) {
                flag(ctx, kStatusTimeout);
                atomicAdd(epoch, 1u);
            }
            return;
        }
        if (tid == 0) {
            uint64_t m = 0;
            for (int w = 0; w < kWarps; ++w) m = sm.xmax[w] > m ? sm.xmax[w] : m;
            sm.query[kPub] = m;
        }
        __syncthreads();
        // X, the largest next key of any list: the number of published keys above it
        {
            const uint64_t X = sm.query[kPub];
#pragma unroll
            for (int t = 0; t < kPub; ++t) cnt[kPub] += ukey[t] > X;
        }
        {
            const int n = __reduce_add_sync(0xffffffffu, cnt[kPub]);
            if (lane == 0) sm.rpart[warp][kPub] = n;
        }
        __syncthreads();
        if (tid <= kPub) {
            int n = 0;
            for (int w = 0; w < kWarps; ++w) n += sm.rpart[w][tid];
            sm.rank[tid] = n;
        }
        __syncthreads();
        fallback = sm.query[kPub] != 0ull && sm.rank[kPub] < K;
        if (!fallback) {
            if (tid == 0) {
                int n = 0;
                for (int t = 0; t < kPub; ++t) {
                    if (sm.own[t] != 0ull && sm.rank[t] < K) {
                        sm.work_slot[n] = sm.rank[t];
                        sm.work_blk[n] = key_block(sm.own[t]);
                        ++n;
                    }
                }
                // init and local blocks: slots K .. slots-1, one per CTA from the last CTA down
                const int nf = n_init + n_local;
                for (int f = 0; f < nf; ++f) {
                    if ((cpg - 1 - (f % cpg)) != j) continue;
                    sm.work_slot[n] = K + f;
                    sm.work_blk[n] = f < n_init ? f : c - n_local + 1 + (f - n_init);
                    ++n;
                }
                sm.nwork = n;
            }
        } else {
            // every CTA publishes all its keys, then all meet (tagged arrival words); the winners of
            // an exact top-k over all of them, ascending by block, fill the slots between the init
            // and the local blocks
            for (int r = tid; r < nrows; r += kThreads) {
                const int cand = (j + (r / kChunk) * cpg) * kChunk + r % kChunk;
                if (cand < ncand) gkeys[cand] = s_keys[r];
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) ll_st(fbw + j, ll_word(1u, tag));
            {
                uint64_t ww[1];
                ll_wait_all([&](int) { return fbw + min(tid, cpg - 1); }, 1, ww, tag, ctx, bad);
            }
            __threadfence();
            __syncthreads();
            if (sm.bad) {
                if (tid == 0) {
                    flag(ctx, kStatusTimeout);
                    atomicAdd(epoch, 1u);
                }
                return;
            }
            uint64_t prefix, mask;
            radix_kth_stream(gkeys, ncand, K, sm.ss, prefix, mask, tid);
            if (tid == 0) sm.nwin = 0;
            __syncthreads();
            for (int e = tid; e < ncand; e += kThreads) {
                const uint64_t key = __ldcg(gkeys + e);
                if (key && (key & mask) >= prefix) {
                    const int w = atomicAdd(&sm.nwin, 1);
                    if (w < kCap) sm.wkeys[w] = key;
                }
            }
            __syncthreads();
            if (warp == 0) {
                const int nw = min(sm.nwin, K);
                int x0 = 2 * lane < nw ? key_block(sm.wkeys[2 * lane]) : 0x7fffffff;
                int x1 = 2 * lane + 1 < nw ? key_block(sm.wkeys[2 * lane + 1]) : 0x7fffffff;
                warp_sort64(x0, x1, lane);
                for (int s = lane; s < n_init; s += 32) sm.sel[s] = s;
                if (2 * lane < K) sm.sel[n_init + 2 * lane] = 2 * lane < nw ? x0 : -1;
                if (2 * lane + 1 < K) sm.sel[n_init + 2 * lane + 1] = 2 * lane + 1 < nw ? x1 : -1;
                for (int t = lane; t < n_local; t += 32) sm.sel[n_init + K + t] = c - n_local + 1 + t;
                for (int s = n_init + K + n_local + lane; s < slots; s += 32) sm.sel[s] = -1;
            }
        }
    } else {
        // list paths: the given selection (entries past the query's block flagged and left out),
        // or every block 0 .. c when there are at most k candidates, or the init and local blocks
        // when k = 0
        if (idx_in) {
            for (int s = tid; s < slots; s += kThreads) {
                int blk = idx_in[(int64_t)bg * slots + s];
                if (blk > c) {
                    flag(ctx, kStatusBounds);
                    blk = -1;
                }
                sm.sel[s] = blk;
            }
        } else if (ncand <= K) {
            for (int s = tid; s < slots; s += kThreads) sm.sel[s] = s <= c ? s : -1;
        } else {
            for (int s = tid; s < slots; s += kThreads) {
                int blk = -1;
                if (s < n_init) blk = s;
                else if (s < n_init + n_local) blk = c - n_local + 1 + (s - n_init);
                sm.sel[s] = blk;
            }
        }
    }
    __syncthreads();
    if (!owner || fallback) {
        if (tid == 0) {
            int n = 0;
            for (int s = j; s < slots; s += cpg) {
                sm.work_slot[n] = s;
                sm.work_blk[n] = sm.sel[s];
                ++n;
            }
            sm.nwork = n;
        }
    }
    __syncthreads();  // also: every thread is done with the k_bar rows the stages now overwrite

    // CTA 0 requests every CTA's alive word now and looks at them at the end (see there)
    uint64_t alive_w = 0;
    if (blockIdx.x == 0 && tid < (int)gridDim.x) alive_w = ll_ld(alive + tid);

    // ---------------------------------------------------------------- C: per-slot partials
    // Warp w < nstages attends items w, w + nstages, ... in its own stage: its lanes request the
    // block's K and V rows (16-byte asynchronous copies; rows past the query zero-filled), wait for
    // their own copies, and compute the slot's partial.  The slot's done word (tagged, carrying the
    // block id) follows its record.
    const int nwork = sm.nwork;
    const float scale_log2 = scale * 1.4426950408889634f;
    if (warp < nstages) {
        __nv_bfloat16* sk = s_region + (size_t)warp * (stage_bytes<D>() / 2);
        __nv_bfloat16* sv = sk + kBlk * RE;
        for (int w = warp; w < nwork; w += nstages) {
            const int slot = sm.work_slot[w];
            const int blk = sm.work_blk[w];
            uint64_t* r = rec + (int64_t)slot * G * (D + 2);
            if (blk < 0) {
                for (int hh = 0; hh < G; ++hh) {
                    for (int e = lane; e < D + 2; e += 32) {
                        const float v = e == 0 ? -INFINITY : 0.f;
                        ll_st(r + hh * (D + 2) + e, ll_word(__float_as_uint(v), tag));
                    }
                }
            } else {
                const __nv_bfloat16* kblk = kc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
                const __nv_bfloat16* vblk = vc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
                const int lim = min(kBlk - 1, pos - blk * kBlk);
                for (int e = lane; e < kBlk * (D / 8); e += 32) {
                    const int row = e / (D / 8), c8 = (e % (D / 8)) * 8;
                    const bool ok = row <= lim;
                    ptx::cp_async16(sk + row * RE + c8, kblk + (ok ? (int64_t)row * D + c8 : 0), ok);
                    ptx::cp_async16(sv + row * RE + c8, vblk + (ok ? (int64_t)row * D + c8 : 0), ok);
                }
                ptx::cp_async_commit();
                ptx::cp_async_wait<0>();
                __syncwarp();
                slot_partial<D>(&sm.Qb[0][0], sk, sv, lim, scale_log2, G, r, tag, lane);
                __syncwarp();  // the stage is reloaded by the warp's next item
            }
            __syncwarp();
            if (lane == 0) ll_st(done + slot, ll_word((uint32_t)blk, tag));
        }
    }

    // ---------------------------------------------------------------- D: combine, idx_out
    // idx_out comes from a CTA without a combine item when there is one
    if (idx_out && j == (cpg > G * (D / 32) ? cpg - 1 : 0)) {
        if (owner && !fallback) {
            if (warp == 0) {
                uint64_t ww[2];
                ll_wait_all([&](int i) { return done + min(2 * lane + i, K - 1); }, 2, ww, tag, ctx, bad);
                int x0 = 2 * lane < K ? (int)ll_val(ww[0]) : 0x7fffffff;
                int x1 = 2 * lane + 1 < K ? (int)ll_val(ww[1]) : 0x7fffffff;
                warp_sort64(x0, x1, lane);
                int32_t* dst = idx_out + (int64_t)bg * slots;
                for (int s = lane; s < n_init; s += 32) dst[s] = s;
                if (2 * lane < K) dst[n_init + 2 * lane] = x0;
                if (2 * lane + 1 < K) dst[n_init + 2 * lane + 1] = x1;
                for (int t = lane; t < n_local; t += 32) dst[n_init + K + t] = c - n_local + 1 + t;
                for (int s = n_init + K + n_local + lane; s < slots; s += 32) dst[s] = -1;
            }
        } else {
            for (int s = tid; s < slots; s += kThreads) idx_out[(int64_t)bg * slots + s] = sm.sel[s];
        }
    }
    constexpr int kPerWarp = (kMaxSlots + kWarps - 1) / kWarps;
    const int nmine = warp < slots ? (slots - 1 - warp) / kWarps + 1 : 0;  // warp w folds slots w, w+8, ..
    for (int item = j; item < G * (D / 32); item += cpg) {
        const int hh = item / (D / 32), d0 = (item % (D / 32)) * 32;
        // wait for the warp's slots (lane i polls the m word of slot warp + 8 i), then read their
        // records (every word checked again; a word not yet visible is read again)
        {
            uint64_t ww[1];
            if (lane < nmine)
                ll_wait_all([&](int) { return rec + ((int64_t)(warp + kWarps * lane) * G + hh) * (D + 2); }, 1, ww,
                            tag, ctx, bad);
            __syncwarp();
        }
        float ms[kPerWarp], ls[kPerWarp], os[kPerWarp];
        {
            uint64_t ww[3 * kPerWarp];
            auto addr = [&](int i) -> const uint64_t* {
                const int s = warp + kWarps * (i / 3), part3 = i % 3;
                return rec + ((int64_t)s * G + hh) * (D + 2) + (part3 < 2 ? part3 : 2 + d0 + lane);
            };
            ll_wait_all(addr, 3 * nmine, ww, tag, ctx, bad);
#pragma unroll
            for (int i = 0; i < kPerWarp; ++i) {
                ms[i] = -INFINITY;
                ls[i] = os[i] = 0.f;
                if (i < nmine) {
                    ms[i] = __uint_as_float(ll_val(ww[3 * i]));
                    ls[i] = __uint_as_float(ll_val(ww[3 * i + 1]));
                    os[i] = __uint_as_float(ll_val(ww[3 * i + 2]));
                }
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
                const float w8 = exp2f(ms[i] - M);
                L = fmaf(ls[i], w8, L);
                acc = fmaf(os[i], w8, acc);
            }
        }
        sm.cm[warp][lane] = M;
        sm.cl[warp][lane] = L;
        sm.co[warp][lane] = acc;
        __syncthreads();
        if (warp == 0 && !sm.bad) {
            float Mt = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) Mt = fmaxf(Mt, sm.cm[w][lane]);
            float Lt = 0.f, At = 0.f;
            if (Mt != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    if (sm.cm[w][lane] == -INFINITY) continue;
                    const float a = exp2f(sm.cm[w][lane] - Mt);
                    Lt += a * sm.cl[w][lane];
                    At += a * sm.co[w][lane];
                }
            }
            o[(b * H + (int64_t)g * G + hh) * D + d0 + lane] = __float2bfloat16_rn(Lt > 0.f ? At / Lt : 0.f);
        }
        __syncthreads();
    }
    // The epoch advances once every CTA of the grid has read it (each tagged its alive word after
    // reading it), so the next call on this workspace uses a new tag.
    if (blockIdx.x == 0) {
        for (int i0 = 0; i0 < (int)gridDim.x; i0 += kThreads) {
            if (i0 == 0 && (tid >= (int)gridDim.x || ll_ok(alive_w, tag))) continue;
            uint64_t ww[1];
            ll_wait_all([&](int) { return alive + min(i0 + tid, (int)gridDim.x - 1); }, 1, ww, tag, ctx, bad);
        }
        __syncthreads();
        if (tid == 0 && !sm.bad) atomicAdd(epoch, 1u);
    }
    __syncthreads();
    if (sm.bad && tid == 0) {
        flag(ctx, kStatusTimeout);
        atomicAdd(epoch, 1u);
    }
}

template <int D>
cudaError_t pf(const void* q, const void* kc, const void* vc, const void* kbar, const int32_t* idx_in,
               int32_t* idx_out, void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap, int topk,
               int n_init, int n_local, float scale, unsigned* epoch, void* ws, size_t ws_bytes, bool pdl,
               cudaStream_t st, DevCtx ctx) {
    const int slots = n_init + n_local + topk;
    const int G = H / Hkv;
    const int groups = B * Hkv;
    const int c = pos / kBlk;
    const int ncand = c - n_local - n_init + 1;
    if (topk > kCap || slots > kMaxSlots || G > kMaxG || groups > kMaxGroups) return cudaErrorNotSupported;
    auto kern = sparse_decode_pf_kernel<D>;
    const int smem_max = (int)pf_smem_bytes<D>(kRowsMax, kMaxStages);
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
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
            if (e != cudaSuccess) return e;
            int oc = 0, n = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&oc, kern, kThreads, smem_max);
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            if (oc < 1) return cudaErrorNotSupported;
            occ_of[dev] = oc;
            nsm_of[dev] = n;
        }
        occ = occ_of[dev];
        nsm = nsm_of[dev];
    }
    int cpg = min(occ * nsm / groups, kMaxCpg);
    if (cpg < 1) return cudaErrorNotSupported;
    const bool owner = idx_in == nullptr && topk > 0 && ncand > topk;
    int rcap = 0, nstages = 1;  // k_bar rows a CTA holds (a multiple of 8), K|V stages
    if (owner) {
        const int nchunks = (ncand + kChunk - 1) / kChunk;
        rcap = (nchunks + cpg - 1) / cpg * kChunk;
        if (rcap > kRowsMax) return cudaErrorNotSupported;
        nstages = kMaxStages;
    } else {
        cpg = min(cpg, max(slots, G * (D / 32)));
        nstages = min(kMaxStages, (slots + cpg - 1) / cpg);
    }
    const int smem = (int)pf_smem_bytes<D>(rcap, nstages);
    const PfLayout lay = pf_layout(groups, ncand > 0 ? ncand : 0, slots, G, D);
    if (lay.total > ws_bytes) return cudaErrorNotSupported;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(groups * cpg));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    // All CTAs must be resident at once (they wait for one another's words).  A plain call
    // launches cooperatively.  A programmatic dependent launches with the grid sized to the
    // occupancy instead: its CTAs may wait for resources that the previous kernel frees as it
    // finishes, and every CTA of this grid runs before any kernel that waits for this one can
    // start (those start only once all CTAs here have executed griddepcontrol.launch_dependents).
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kc),
                              static_cast<const __nv_bfloat16*>(vc), static_cast<const __nv_bfloat16*>(kbar), idx_in,
                              idx_out, static_cast<__nv_bfloat16*>(o), H, Hkv, pos, Tmax, nb_cap, topk, n_init,
                              n_local, slots, scale, cpg, rcap, nstages, epoch, static_cast<unsigned char*>(ws), lay,
                              ctx);
}

}  // namespace

size_t sparse_decode_pf_workspace(int B, int H, int Hkv, int pos, int topk, int n_init, int n_local, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || pos < 0) return 0;
    const int slots = n_init + n_local + topk;
    const int ncand = pos / kBlk - n_local - n_init + 1;
    return pf_layout(B * Hkv, ncand > 0 ? ncand : 0, slots, H / Hkv, d).total;
}

cudaError_t launch_sparse_decode_pf(DType dt, const void* q, const void* kc, const void* vc, const void* kbar,
                                    const int32_t* idx_in, int32_t* idx_out, void* o, int B, int H, int Hkv,
                                    int pos, int Tmax, int nb_cap, int d, int topk, int n_init, int n_local,
                                    float scale, unsigned* epoch, void* ws, size_t ws_bytes, bool pdl,
                                    cudaStream_t st, DevCtx ctx) {
    if (dt != DType::BF16 || (d != 64 && d != 128)) return cudaErrorNotSupported;
    return d == 64 ? pf<64>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init,
                            n_local, scale, epoch, ws, ws_bytes, pdl, st, ctx)
                   : pf<128>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init,
                             n_local, scale, epoch, ws, ws_bytes, pdl, st, ctx);
}

}  // namespace sala
