// Sparse decode in two launches for bf16, d = 64 or 128: the block-key table k_bar is prefetched
// and scored by every SM, then one thread-block cluster per (batch, KV group) attends the selected
// blocks and combines the partials in distributed shared memory.
//
// The step reads the whole block-key table of the group (8 MiB at 2^20 tokens and 2 KV heads) to
// score the candidates, and then only the ~67 selected K/V blocks (4 MiB).  Exchanging data between
// CTAs through global memory costs a round trip to the memory's home (on a two-die B200 often the
// other die) every time, so the design keeps exactly one global exchange, the one between the two
// kernels, where the kernel boundary itself makes the data visible:
//
//   score kernel (groups x cpg CTAs, no waits between CTAs).  Each CTA copies its share of k_bar --
//      4-block chunks dealt round robin, so blocks chosen together land in different CTAs -- into
//      shared memory as soon as it runs (16-byte asynchronous copies; before griddepcontrol.wait
//      when the call is a programmatic dependent, so the copy overlaps the previous layer's kernel).
//      It then scores its rows on the tensor cores (the group-summed query as bf16 hi + lo rows of
//      an m16n8k16 tile against 8 k_bar rows at a time), keeps its best kPub + 1 selection keys
//      (orderable score above the inverted block index: distinct, larger = better, ties to the lower
//      block) by counting ranks, and stores them, and all its keys, for the attend kernel.
//   attend kernel (groups clusters of CS CTAs), launched as a programmatic dependent of the score
//      kernel: before griddepcontrol.wait it loads the query rows and starts copying the init and
//      local blocks; after it, every CTA reads the group's lists U (kPub keys per scoring CTA).
//      With X = the largest (kPub+1)-th key of any CTA, no unlisted key can beat X; when at least
//      k keys of U exceed X, the winners are among those keys C, and every CTA ranks its share of C
//      against C: a key of rank r < k is the group's (r+1)-th best block.  When fewer than k keys
//      of U exceed X (some scoring CTA had more than kPub winners), the cluster instead takes an
//      exact radix select over all the group's keys.  The winners, by rank,
//      are broadcast to the cluster through distributed shared memory.  CTA r then attends slots
//      r, r + CS, ... (a warp per slot: K and V of the block by 16-byte asynchronous copies, the
//      G heads' logits and p v on warp-level tensor-core tiles, a softmax partial per head), folds
//      its slots into one partial per head, and after a cluster barrier combines the partials of
//      every CTA of the cluster for its heads into the output.
//
// With a given selection (idx_in), or at most k candidates, or k = 0, only the attend kernel runs.
#include <cooperative_groups.h>

#include <mutex>

#include "blocksel.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sala {
namespace {

namespace cg = cooperative_groups;
using namespace dec;

constexpr int kBlk = 64;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCap = 64;            // largest k
constexpr int kMaxSlots = 80;       // n_init + n_local + k
constexpr int kMaxG = 16;
constexpr int kPub = 8;             // keys per scoring CTA in U
constexpr int kListWords = 10;      // per list: kPub keys, the next key, padding
constexpr int kMaxCpg = 160;        // scoring CTAs per group (a B200 has 148 SMs)
constexpr int kMaxGroups = 16;
constexpr int kChunk = 4;           // k_bar rows per round-robin chunk
constexpr int kRowsMax = kThreads;  // k_bar rows a scoring CTA holds: 32 per warp (four 8-row tiles)
constexpr int kStages = 5;          // K|V stages of an attend CTA (one per warp 0 .. 4)
constexpr int kCS = 16;             // CTAs per attend cluster

template <int D>
constexpr int row_elems() { return D + 8; }  // padded rows: conflict-free ldmatrix
template <int D>
constexpr size_t stage_bytes() { return (size_t)2 * kBlk * row_elems<D>() * 2; }
// A head's softmax partial: maximum, sum, two unused words, then the D sums of p v -- rows of
// D + 4 floats, so the p v part is read and sent to the combining CTA 16 bytes at a time.
template <int D>
constexpr int part_row() { return D + 4; }

template <int D>
struct ScoreSmem {
    __nv_bfloat16 QS[16][D + 8];      // A tile: row 0 bf16(sum of the group's queries), row 1 the residual
    uint64_t wtop[kWarps][kPub + 1];  // per-warp best keys, largest first (0: none)
    uint64_t own[kPub + 1];           // this CTA's best keys, largest first
    alignas(16) uint64_t keys[kRowsMax];  // read two at a time (16-byte loads)
    alignas(128) __nv_bfloat16 rows[kRowsMax][D + 8];  // k_bar rows (rows past the CTA's share unused)
};

template <int D>
struct AttendSmem {
    __nv_bfloat16 Qb[kMaxG][D + 8];
    alignas(16) uint64_t u[kMaxCpg * kPub];  // C, the keys of U above X (read two at a time)
    int cnt_part[kWarps];             // per warp: nonzero keys of U
    int cnt_c[(kMaxCpg * kPub + kThreads - 1) / kThreads][kWarps];  // per (key slot, warp): keys above X
    uint64_t xpart[kWarps];
    int sel[kMaxSlots];               // slot -> block (-1: empty)
    int wblk[kCap];                   // CTA 0, with idx_out: the winners' blocks by rank
    int nloc;                         // winners among this CTA's share of U ...
    int loc_rank[kMaxCpg * kPub / kCS], loc_blk[kMaxCpg * kPub / kCS];  // ... their ranks and blocks
    uint64_t wkeys[kCap];
    int nwin;
    RadixSelSmem ss;
    float wt[kStages][kMaxG];         // fold: weight of each slot's partial per head
    float fm[kMaxG], fl[kMaxG];       // fold: largest maximum and weighted sum per head
    alignas(16) float recv[kMaxG / kCS][kCS][part_row<D>()];  // partials of the heads this CTA combines
    alignas(128) unsigned char stages[kStages * stage_bytes<D>()];
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, x, off);
        x = y > x ? y : x;
    }
    return x;
}

// Exact k-th largest nonzero key among n keys in global memory (the fallback): one byte at a time
// from the top, streaming the keys on every pass.  On return winner(key) = key != 0 &&
// (key & mask) >= prefix picks min(K, #nonzero) keys.
__device__ void radix_kth_stream(const uint64_t* keys, int n, int K, RadixSelSmem& s, uint64_t& prefix,
                                 uint64_t& mask, int t) {
    const int lane = t & 31, warp = t >> 5;
    int nv = 0;
    for (int e = t; e < n; e += kThreads) nv += keys[e] != 0ull;
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
            const uint64_t key = keys[e];
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

// One slot's softmax partial, computed by one warp: the block's K and V rows (64 x D, padded rows)
// in shared memory, the G <= 16 query rows in Qs (padded to 16 with zeros).  The logits are an
// m16n8k16 tile row per head (16 x 64), the softmax runs in registers (a head's row lives in the 4
// lanes of a quad), and P -- rounded to bf16 -- becomes the A fragments of P V directly.  Writes
// out[h][0] = the head's maximum logit (log2 units), out[h][1] = the sum of its probabilities and
// out[h][4 ..] = the unnormalised sum of p v, for heads h < G (rows of part_row<D>() floats).
template <int D>
__device__ __forceinline__ void slot_partial(const __nv_bfloat16* __restrict__ Qs, const __nv_bfloat16* __restrict__ Ks,
                                             const __nv_bfloat16* __restrict__ Vs, int lim, float scale_log2, int G,
                                             float* out, int lane) {
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
    // P V in halves of 64 columns (or all of D = 64): ldmatrix.trans of V gives the B fragments of
    // two column tiles at once
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
            if (gq < G) *reinterpret_cast<float2*>(out + gq * part_row<D>() + 4 + col) = make_float2(ov[n][0], ov[n][1]);
            if (gq + 8 < G)
                *reinterpret_cast<float2*>(out + (gq + 8) * part_row<D>() + 4 + col) = make_float2(ov[n][2], ov[n][3]);
        }
    }
    if ((lane & 3) == 0) {
        if (gq < G) *reinterpret_cast<float2*>(out + gq * part_row<D>()) = make_float2(mx0, l0);
        if (gq + 8 < G) *reinterpret_cast<float2*>(out + (gq + 8) * part_row<D>()) = make_float2(mx1, l1);
    }
}

// Round-robin dealing of a group's candidates to its scoring CTAs: row r of CTA j holds candidate
// (j + (r / kChunk) * cpg) * kChunk + r % kChunk (block n_init + candidate).
__device__ __forceinline__ int cand_of_row(int j, int r, int cpg) {
    return (j + (r / kChunk) * cpg) * kChunk + r % kChunk;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
decode_score_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kbar,
                    const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc, int H, int Hkv,
                    int pos, int Tmax, int nb_cap, int n_init, int n_local, int cpg, uint64_t* __restrict__ lists,
                    uint64_t* __restrict__ allkeys) {
    extern __shared__ __align__(128) unsigned char score_smem_raw[];
    ScoreSmem<D>& sm = *reinterpret_cast<ScoreSmem<D>*>(score_smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / Hkv;
    const int bg = blockIdx.x / cpg, j = blockIdx.x % cpg;
    const int64_t b = bg / Hkv;
    const int g = bg % Hkv;
    const int c = pos / kBlk;
    const int lo = n_init;
    const int ncand = c - n_local - lo + 1;  // > topk >= 1 on this path
    const int nchunks = (ncand + kChunk - 1) / kChunk;
    const int my_chunks = j < nchunks ? (nchunks - 1 - j) / cpg + 1 : 0;
    const int nrows = my_chunks * kChunk;  // <= kRowsMax (checked at launch)

    // k_bar rows first: they do not depend on the previous kernel
    const __nv_bfloat16* kb = kbar + ((int64_t)bg * nb_cap + lo) * D;
    for (int e = tid; e < nrows * (D / 8); e += kThreads) {
        const int r = e / (D / 8), piece = e % (D / 8);
        const int cand = cand_of_row(j, r, cpg);
        const bool ok = cand < ncand;
        ptx::cp_async16(&sm.rows[r][piece * 8], kb + (ok ? (int64_t)cand * D + piece * 8 : 0), ok);
    }
    ptx::cp_async_commit();
    // the group's query rows (G x D bf16, 128-byte lines) are pulled into L2 only: the previous
    // kernel's writes land there, so they are read for real after the wait
    if (tid < G * D / 64)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(q + (b * H + (int64_t)g * G) * D + 64 * tid));
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the attend kernel may start now: its own early reads come after the previous kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tid < D) {
        // every head's load in flight at once (a loop over a runtime G would wait for each load
        // before issuing the next)
        const __nv_bfloat16* qg = q + (b * H + (int64_t)g * G) * D + tid;
        float qv[kMaxG];
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) qv[h] = h < G ? __bfloat162float(qg[h * D]) : 0.f;
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) s += qv[h];
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

    // scores: warp w takes rows 32w .. 32w+31 as four 8-row tiles at once; the two rows of each
    // result hold the hi and lo parts of the scores
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
                ldsm_x2(bfr, &sm.rows[32 * warp + 8 * i + (lane & 7)][16 * ks + ((lane >> 3) & 1) * 8]);
                mma16816(acc[i], af, bfr);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float s0 = acc[i][0] + __shfl_down_sync(0xffffffffu, acc[i][0], 4);
            const float s1 = acc[i][1] + __shfl_down_sync(0xffffffffu, acc[i][1], 4);
            if (lane < 4) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int r = 32 * warp + 8 * i + 2 * lane + u;
                    const int cand = cand_of_row(j, r, cpg);
                    sm.keys[r] = r < nrows && cand < ncand ? sel_key(u ? s1 : s0, lo + cand) : 0ull;
                }
            }
        }
    }
    __syncwarp();
    // best kPub + 1 keys of the warp's 32 by counting ranks (keys are distinct), then of the CTA
    {
        const uint64_t x = sm.keys[32 * warp + lane];
        const ulonglong2* kv = reinterpret_cast<const ulonglong2*>(sm.keys + 32 * warp);
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
    if (tid <= kPub) lists[(int64_t)blockIdx.x * kListWords + tid] = sm.own[tid];
    // the CTA's two best blocks are likely winners: their K and V rows start towards L2 now, so the
    // attend kernel finds most of its blocks there (a hint; the selection does not depend on it)
    if (tid < 4 && sm.own[tid >> 1] != 0ull) {
        const int blk = key_block(sm.own[tid >> 1]);
        const __nv_bfloat16* base = (tid & 1) ? vc : kc;
        ptx::bulk_prefetch_l2(base + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D, kBlk * D * 2);
    }
    uint64_t* gk = allkeys + (int64_t)bg * ncand;
    for (int r = tid; r < nrows; r += kThreads) {
        const int cand = cand_of_row(j, r, cpg);
        if (cand < ncand) gk[cand] = sm.keys[r];
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
decode_attend_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                     const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ idx_in,
                     int32_t* __restrict__ idx_out, __nv_bfloat16* __restrict__ o, int H, int Hkv, int pos,
                     int Tmax, int topk, int n_init, int n_local, int slots, float scale, int cpg, bool early,
                     const uint64_t* __restrict__ lists, const uint64_t* __restrict__ allkeys, DevCtx ctx) {
    extern __shared__ __align__(128) unsigned char attend_smem_raw[];
    AttendSmem<D>& sm = *reinterpret_cast<AttendSmem<D>*>(attend_smem_raw);
    constexpr int RE = row_elems<D>();
    cg::cluster_group cl = cg::this_cluster();
    constexpr int CS = kCS;  // the launch's cluster size
    const int rk = (int)cl.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = H / Hkv;
    const int bg = blockIdx.x / CS;
    const int64_t b = bg / Hkv;
    const int g = bg % Hkv;
    const int c = pos / kBlk;
    const int lo = n_init;
    const int ncand = c - n_local - lo + 1;
    const int K = topk;
    const bool owner = cpg > 0;  // the score kernel ran: the selection is made here
    const int nitems = rk < slots ? (slots - 1 - rk) / CS + 1 : 0;  // slots rk, rk + CS, ... (<= kStages)
    const __nv_bfloat16* qg = q + (b * H + (int64_t)g * G) * D;
    const float scale_log2 = scale * 1.4426950408889634f;
    auto stage_k = [&](int w) { return reinterpret_cast<__nv_bfloat16*>(sm.stages + (size_t)w * stage_bytes<D>()); };
    auto issue = [&](int w, int blk) {  // warp w's lanes copy block blk's K and V rows into stage w
        __nv_bfloat16* sk = stage_k(w);
        __nv_bfloat16* sv = sk + kBlk * RE;
        const __nv_bfloat16* kb = kc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
        const __nv_bfloat16* vb = vc + ((int64_t)bg * Tmax + (int64_t)blk * kBlk) * D;
        const int lim = min(kBlk - 1, pos - blk * kBlk);
        for (int e = lane; e < kBlk * (D / 8); e += 32) {
            const int row = e / (D / 8), c8 = (e % (D / 8)) * 8;
            const bool ok = row <= lim;
            ptx::cp_async16(sk + row * RE + c8, kb + (ok ? (int64_t)row * D + c8 : 0), ok);
            ptx::cp_async16(sv + row * RE + c8, vb + (ok ? (int64_t)row * D + c8 : 0), ok);
        }
        ptx::cp_async_commit();
    };
    // init and local blocks: slots K .. K + n_init + n_local - 1 on the rank path
    auto forced_block = [&](int s) { const int f = s - K; return f < n_init ? f : c - n_local + 1 + (f - n_init); };

    // ---------------------------------------------------------------- before the score kernel ends
    // (only when it ran: its predecessor has then completed, so q and the cache are final)
    bool preloaded = false;
    if (early) {
        for (int e = tid; e < kMaxG * (D / 8); e += kThreads) {
            const int h = e / (D / 8), c8 = (e % (D / 8)) * 8;
            *reinterpret_cast<uint4*>(&sm.Qb[h][c8]) = h < G ? ld16(qg + h * D + c8) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (warp < nitems && rk + warp * CS >= K) {
            issue(warp, forced_block(rk + warp * CS));
            preloaded = true;
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cl.sync();  // every CTA of the cluster runs before any reaches into another's shared memory
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!early) {
        for (int e = tid; e < kMaxG * (D / 8); e += kThreads) {
            const int h = e / (D / 8), c8 = (e % (D / 8)) * 8;
            *reinterpret_cast<uint4*>(&sm.Qb[h][c8]) = h < G ? ld16(qg + h * D + c8) : make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // ---------------------------------------------------------------- the slot list
    bool rank_layout = false;  // slots 0 .. K-1: the winners by rank, then the forced blocks
    int nwin = 0;              // winners on the rank path (min(K, nonzero keys of U))
    if (owner) {
        // U, the group's lists, into registers; X, the largest key any list left out
        const int nu = cpg * kPub;
        const uint64_t* gl = lists + (int64_t)bg * cpg * kListWords;
        constexpr int kU = (kMaxCpg * kPub + kThreads - 1) / kThreads;
        uint64_t uv[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const int e = tid + kThreads * i;
            uv[i] = e < nu ? gl[(e / kPub) * kListWords + e % kPub] : 0ull;
        }
        uint64_t x = tid < cpg ? gl[tid * kListWords + kPub] : 0ull;  // cpg <= kThreads
        x = warp_max_u64(x);
        int nz = 0;
#pragma unroll
        for (int i = 0; i < kU; ++i) nz += uv[i] != 0ull;
        nz = __reduce_add_sync(0xffffffffu, nz);
        if (lane == 0) {
            sm.xpart[warp] = x;
            sm.cnt_part[warp] = nz;
        }
        __syncthreads();
        uint64_t X = 0ull;
        int nvalid = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            X = sm.xpart[w] > X ? sm.xpart[w] : X;
            nvalid += sm.cnt_part[w];
        }
        // C = the keys of U above X, in (key slot, thread) order.  A key at or below X has at
        // least |C| keys above it, so when |C| >= K only keys of C can win, and a key of C has
        // the same rank in C as in U (every key above it is in C).
        unsigned ab[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) ab[i] = __ballot_sync(0xffffffffu, uv[i] > X);
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kU; ++i) sm.cnt_c[i][warp] = __popc(ab[i]);
        }
        if (tid == 0) sm.nloc = 0;
        __syncthreads();
        const unsigned below = (1u << lane) - 1u;
        int rank_x = 0;  // |C|: the keys of U above X
        int pos[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            int before = 0, tot = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const int c = sm.cnt_c[i][w];
                tot += c;
                before += w < warp ? c : 0;
            }
            pos[i] = rank_x + before + __popc(ab[i] & below);
            rank_x += tot;
        }
        // X would be a winner when fewer than K keys of U beat it: the lists may then hide winners
        // (with fewer than K keys in U every key wins, and some list left keys out).
        rank_layout = X == 0ull || rank_x >= K;
        if (rank_layout) {
            // Every key's rank (the keys of C above it; keys are distinct) decides its slot: the
            // winner of rank r < K is attended in slot r by CTA r mod CS.  This CTA ranks its share
            // of C, eight threads per key, and writes each winner's block into the slot list of
            // the CTA that attends it (and, with idx_out, into CTA 0's list of winners).
#pragma unroll
            for (int i = 0; i < kU; ++i)
                if (uv[i] > X) sm.u[pos[i]] = uv[i];
            if (tid == 0 && (rank_x & 1)) sm.u[rank_x] = 0ull;  // even length (rank_x < nu here)
            __syncthreads();
            nwin = min(nvalid, K);
            const int nc = rank_x;
            const int per = (nc + CS - 1) / CS, e0 = rk * per, e1 = min(nc, e0 + per);
            const int sub = tid & 7;
            const ulonglong2* u2 = reinterpret_cast<const ulonglong2*>(sm.u);
            // the share holds at most kMaxCpg * kPub / CS = 80 keys: up to three per group of eight
            // threads, all ranked against each pair of C's keys as it is read
            constexpr int kPerThread = (kMaxCpg * kPub / kCS + kThreads / 8 - 1) / (kThreads / 8);
            uint64_t key[kPerThread];
            int r[kPerThread];
#pragma unroll
            for (int m = 0; m < kPerThread; ++m) {
                const int e = e0 + (tid >> 3) + (kThreads / 8) * m;
                key[m] = e < e1 ? sm.u[e] : 0ull;
                r[m] = 0;
            }
#pragma unroll 4
            for (int j = sub; j < (nc + 1) / 2; j += 8) {
                const ulonglong2 p2 = u2[j];
#pragma unroll
                for (int m = 0; m < kPerThread; ++m) r[m] += (p2.x > key[m]) + (p2.y > key[m]);
            }
#pragma unroll
            for (int m = 0; m < kPerThread; ++m) {
                r[m] += __shfl_xor_sync(0xffffffffu, r[m], 1);
                r[m] += __shfl_xor_sync(0xffffffffu, r[m], 2);
                r[m] += __shfl_xor_sync(0xffffffffu, r[m], 4);
                if (sub == 0 && key[m] != 0ull && r[m] < K) {
                    const int w = atomicAdd(&sm.nloc, 1);
                    sm.loc_rank[w] = r[m];
                    sm.loc_blk[w] = key_block(key[m]);
                }
            }
            // the share's winners, gathered above, go out together: one thread each
            __syncthreads();
            if (tid < sm.nloc) {
                const int r = sm.loc_rank[tid], blk = sm.loc_blk[tid];
                *cl.map_shared_rank(&sm.sel[r], r % CS) = blk;
                if (idx_out) *cl.map_shared_rank(&sm.wblk[r], 0) = blk;
            }
            // this CTA's own slots that no winner fills: the forced blocks, and -1 past the winners
            for (int s = rk; s < slots; s += CS) {
                if (s >= K) sm.sel[s] = forced_block(s);
                else if (s >= nwin) sm.sel[s] = -1;
            }
        } else {
            // exact top-k over all the group's keys (written by the score kernel); the winners,
            // ascending by block, fill the slots between the init and the local blocks
            uint64_t prefix, mask;
            const uint64_t* gk = allkeys + (int64_t)bg * ncand;
            radix_kth_stream(gk, ncand, K, sm.ss, prefix, mask, tid);
            if (tid == 0) sm.nwin = 0;
            __syncthreads();
            for (int e = tid; e < ncand; e += kThreads) {
                const uint64_t key = gk[e];
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
    } else if (idx_in) {
        // a given selection: entries past the query's block are flagged and left out
        for (int s = tid; s < slots; s += kThreads) {
            int blk = idx_in[(int64_t)bg * slots + s];
            if (blk > c) {
                flag(ctx, kStatusBounds);
                blk = -1;
            }
            sm.sel[s] = blk;
        }
    } else if (ncand <= K) {
        for (int s = tid; s < slots; s += kThreads) sm.sel[s] = s <= c ? s : -1;  // every block 0 .. c
    } else {
        for (int s = tid; s < slots; s += kThreads) {  // k = 0: the init and local blocks
            int blk = -1;
            if (s < n_init) blk = s;
            else if (s < n_init + n_local) blk = c - n_local + 1 + (s - n_init);
            sm.sel[s] = blk;
        }
    }
    // With the score kernel's lists, winners were written into other CTAs' slot lists: a cluster
    // barrier (the same on both of that path's branches, so every CTA of the cluster meets it).
    if (owner) cl.sync();
    else __syncthreads();

    // ---------------------------------------------------------------- attention of this CTA's slots
    // warp w < nitems attends slot rk + w CS in stage w and leaves the slot's partial (per head:
    // max, sum, sum of p v) at the start of the stage
    if (warp < nitems) {
        int blk = sm.sel[rk + warp * CS];
        if (blk >= 0 && !in_bounds(ctx, blk <= c)) blk = -1;
        float* out = reinterpret_cast<float*>(stage_k(warp));
        if (blk >= 0) {
            if (!(preloaded && rank_layout)) {  // the early copy is this slot's block only on the rank path
                if (preloaded) {
                    ptx::cp_async_wait<0>();
                    __syncwarp();
                }
                issue(warp, blk);
            }
            ptx::cp_async_wait<0>();
            __syncwarp();
            const __nv_bfloat16* sk = stage_k(warp);
            const int lim = min(kBlk - 1, pos - blk * kBlk);
            slot_partial<D>(&sm.Qb[0][0], sk, sk + kBlk * RE, lim, scale_log2, G, out, lane);
        } else {
            ptx::cp_async_wait<0>();
            __syncwarp();
            for (int e = lane; e < G * part_row<D>(); e += 32) out[e] = e % part_row<D>() == 0 ? -INFINITY : 0.f;
        }
    }
    __syncthreads();
    // fold the CTA's slots into one partial per head: per head the largest maximum over the slots
    // and each slot's weight 2^(m - M), then the weighted sums; the partial of head h goes straight
    // into the shared memory of CTA h mod kCS, which combines that head
    if (tid < G) {
        const int h = tid;
        float m[kStages];
        float M = -INFINITY;
#pragma unroll
        for (int t = 0; t < kStages; ++t) {
            m[t] = t < nitems ? reinterpret_cast<const float*>(stage_k(t))[h * part_row<D>()] : -INFINITY;
            M = fmaxf(M, m[t]);
        }
        float L = 0.f;
#pragma unroll
        for (int t = 0; t < kStages; ++t) {
            const float w8 = m[t] == -INFINITY ? 0.f : exp2f(m[t] - M);
            sm.wt[t][h] = w8;
            if (t < nitems) L = fmaf(reinterpret_cast<const float*>(stage_k(t))[h * part_row<D>() + 1], w8, L);
        }
        sm.fm[h] = M;
        sm.fl[h] = L;
    }
    __syncthreads();
    // per head: (maximum, sum) as one 8-byte store, then the weighted p v sums 16 bytes at a time
    constexpr int kQ = D / 4 + 1;
    for (int e = tid; e < G * kQ; e += kThreads) {
        const int h = e / kQ, q4 = e % kQ;
        float* dst = cl.map_shared_rank(&sm.recv[h / kCS][rk][0], h % kCS);
        if (q4 == 0) {
            *reinterpret_cast<float2*>(dst) = make_float2(sm.fm[h], sm.fl[h]);
        } else {
            const int col = 4 + 4 * (q4 - 1);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int t = 0; t < kStages; ++t) {
                if (t < nitems) {
                    const float4 pv = *reinterpret_cast<const float4*>(
                        reinterpret_cast<const float*>(stage_k(t)) + h * part_row<D>() + col);
                    const float w8 = sm.wt[t][h];
                    v.x = fmaf(pv.x, w8, v.x);
                    v.y = fmaf(pv.y, w8, v.y);
                    v.z = fmaf(pv.z, w8, v.z);
                    v.w = fmaf(pv.w, w8, v.w);
                }
            }
            *reinterpret_cast<float4*>(dst + col) = v;
        }
    }
    cl.sync();  // every CTA's partials have landed where they are combined
    // CTA rk combines heads rk, rk + kCS, ... over the partials of every CTA of the cluster
    for (int h = rk; h < G; h += kCS) {
        if (tid < D) {
            const int hh = h / kCS;
            float mp[kCS], lp[kCS], op[kCS];
#pragma unroll
            for (int p = 0; p < kCS; ++p) {
                mp[p] = sm.recv[hh][p][0];
                lp[p] = sm.recv[hh][p][1];
                op[p] = sm.recv[hh][p][4 + tid];
            }
            float M = -INFINITY;
#pragma unroll
            for (int p = 0; p < kCS; ++p) M = fmaxf(M, mp[p]);
            float L = 0.f, A = 0.f;
#pragma unroll
            for (int p = 0; p < kCS; ++p) {
                const float w8 = mp[p] == -INFINITY ? 0.f : exp2f(mp[p] - M);
                L = fmaf(lp[p], w8, L);
                A = fmaf(op[p], w8, A);
            }
            o[(b * H + (int64_t)g * G + h) * D + tid] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
        }
    }
    if (idx_out && rk == 0) {
        int32_t* dst = idx_out + (int64_t)bg * slots;
        if (rank_layout) {  // the winners ascending by block (k <= 64: one warp sorts them)
            for (int s = tid; s < n_init; s += kThreads) dst[s] = s;
            if (warp == 0) {
                int x0 = 2 * lane < nwin ? sm.wblk[2 * lane] : 0x7fffffff;
                int x1 = 2 * lane + 1 < nwin ? sm.wblk[2 * lane + 1] : 0x7fffffff;
                warp_sort64(x0, x1, lane);
                if (2 * lane < K) dst[n_init + 2 * lane] = 2 * lane < nwin ? x0 : -1;
                if (2 * lane + 1 < K) dst[n_init + 2 * lane + 1] = 2 * lane + 1 < nwin ? x1 : -1;
            }
            for (int t = tid; t < n_local; t += kThreads) dst[n_init + K + t] = c - n_local + 1 + t;
        } else {
            for (int s = tid; s < slots; s += kThreads) dst[s] = sm.sel[s];
        }
    }
}

struct PfLayout {
    size_t lists, keys, total;
};
PfLayout pf_layout(int groups, int ncand) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    PfLayout L;
    L.lists = 0;
    L.keys = up((size_t)groups * kMaxCpg * kListWords * sizeof(uint64_t));
    L.total = L.keys + (size_t)groups * (ncand > 0 ? ncand : 1) * sizeof(uint64_t);
    return L;
}

struct DevInfo {
    int nsm = 0, clusters = 0;
};

template <int D>
cudaError_t dev_info(DevInfo* out) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static DevInfo info[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorNotSupported;
    std::lock_guard<std::mutex> lk(mu);
    if (info[dev].nsm == 0) {
        DevInfo d;
        e = cudaDeviceGetAttribute(&d.nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(decode_score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(ScoreSmem<D>));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(decode_attend_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(AttendSmem<D>));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(decode_attend_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kCS);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = sizeof(AttendSmem<D>);
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = kCS;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&d.clusters, decode_attend_kernel<D>, &cfg);
        if (e != cudaSuccess) {
            cudaGetLastError();
            d.clusters = -1;  // no clusters of this size: this path is never taken
        }
        info[dev] = d;
    }
    *out = info[dev];
    return cudaSuccess;
}

template <int D>
cudaError_t pf(const void* q, const void* kc, const void* vc, const void* kbar, const int32_t* idx_in,
               int32_t* idx_out, void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap, int topk,
               int n_init, int n_local, float scale, void* ws, size_t ws_bytes, bool pdl, cudaStream_t st,
               DevCtx ctx) {
    const int slots = n_init + n_local + topk;
    const int G = H / Hkv;
    const int groups = B * Hkv;
    const int ncand = pos / kBlk - n_local - n_init + 1;
    if (topk > kCap || slots > kMaxSlots || slots > kStages * kCS || G > kMaxG || groups > kMaxGroups)
        return cudaErrorNotSupported;
    DevInfo info;
    cudaError_t e = dev_info<D>(&info);
    if (e != cudaSuccess) return e;
    if (info.clusters < groups) return cudaErrorNotSupported;  // every group's cluster resident at once
    const bool owner = idx_in == nullptr && topk > 0 && ncand > topk;
    int cpg = 0;
    if (owner) {
        cpg = min(kMaxCpg, info.nsm / groups);
        if (cpg < 1) return cudaErrorNotSupported;
        const int nchunks = (ncand + kChunk - 1) / kChunk;
        if ((nchunks + cpg - 1) / cpg * kChunk > kRowsMax) return cudaErrorNotSupported;
    }
    const PfLayout lay = pf_layout(groups, ncand);
    if (lay.total > ws_bytes) return cudaErrorNotSupported;
    unsigned char* w = static_cast<unsigned char*>(ws);
    uint64_t* lists = reinterpret_cast<uint64_t*>(w + lay.lists);
    uint64_t* keys = reinterpret_cast<uint64_t*>(w + lay.keys);
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    cudaLaunchAttribute pdl_attr;
    pdl_attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr.val.programmaticStreamSerializationAllowed = 1;
    if (owner) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(groups * cpg));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = sizeof(ScoreSmem<D>);
        cfg.stream = st;
        cfg.attrs = &pdl_attr;
        cfg.numAttrs = pdl ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, decode_score_kernel<D>, qb, static_cast<const __nv_bfloat16*>(kbar),
                               static_cast<const __nv_bfloat16*>(kc), static_cast<const __nv_bfloat16*>(vc), H,
                               Hkv, pos, Tmax, nb_cap, n_init, n_local, cpg, lists, keys);
        if (e != cudaSuccess) return e;
    }
    // the attend kernel: a programmatic dependent of the score kernel when that ran (its early
    // reads come after the score kernel's own wait), else of the previous kernel when asked
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(groups * kCS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sizeof(AttendSmem<D>);
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kCS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1] = pdl_attr;
    cfg.attrs = at;
    cfg.numAttrs = (owner || pdl) ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, decode_attend_kernel<D>, qb, static_cast<const __nv_bfloat16*>(kc),
                              static_cast<const __nv_bfloat16*>(vc), idx_in, idx_out, static_cast<__nv_bfloat16*>(o),
                              H, Hkv, pos, Tmax, topk, n_init, n_local, slots, scale, cpg, owner,
                              static_cast<const uint64_t*>(lists), static_cast<const uint64_t*>(keys), ctx);
}

}  // namespace

size_t sparse_decode_pf_workspace(int B, int H, int Hkv, int pos, int topk, int n_init, int n_local, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || pos < 0) return 0;
    const int ncand = pos / kBlk - n_local - n_init + 1;
    return pf_layout(B * Hkv, ncand > 0 ? ncand : 0).total;
}

cudaError_t launch_sparse_decode_pf(DType dt, const void* q, const void* kc, const void* vc, const void* kbar,
                                    const int32_t* idx_in, int32_t* idx_out, void* o, int B, int H, int Hkv,
                                    int pos, int Tmax, int nb_cap, int d, int topk, int n_init, int n_local,
                                    float scale, void* ws, size_t ws_bytes, bool pdl, cudaStream_t st,
                                    DevCtx ctx) {
    if (dt != DType::BF16 || (d != 64 && d != 128)) return cudaErrorNotSupported;
    return d == 64 ? pf<64>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init,
                            n_local, scale, ws, ws_bytes, pdl, st, ctx)
                   : pf<128>(q, kc, vc, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, topk, n_init,
                             n_local, scale, ws, ws_bytes, pdl, st, ctx);
}

}  // namespace sala
