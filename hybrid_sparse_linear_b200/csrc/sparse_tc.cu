// Block-sparse softmax attention prefill on the 5th-generation tensor cores (sm_100a).
//
// Work unit ("tile"): 8 consecutive query tokens x the 16 query heads of one KV group = 128 rows,
// the M of one tcgen05 MMA (row r = head * 8 + token).  The Q tile lives in TMEM (A operand of the
// S MMA), written one tile ahead by the softmax warps, so shared memory holds only K/V.  The 8 tokens
// share their query block (8 divides 64), hence the forced blocks and the diagonal; their
// top-k choices differ, so the tile walks the UNION of the 8 selections (ascending) and each
// row masks the blocks its token did not choose.  Executed FLOPs exceed the algorithmic ones by
// the union overhead; the sum over each row's own selected keys is exact.
//
// The union is consumed two blocks at a time (a "pair", 128 keys):
//   S    = Q [K_a; K_b]^T        M=128 N=128 K=128  (A = Q from TMEM; the two K tiles sit back
//                                                    to back in shared memory: one B operand)
//   P    = online softmax of S, masked per row by each block's selection bit and, on the
//          diagonal block, by causality                              (registers, fp32)
//   O   += P [V_a; V_b]          M=128 N=128 K=128  (A = P from TMEM, bf16, aliasing S)
// S is double-buffered in TMEM so the next pair's S runs on the tensor core while the softmax
// warps work on this one; K/V pairs stream through a 3-stage ring, so a pair's blocks are requested
// two pairs before they are needed.  O is rescaled only when a row's running max grows by more than 8 in
// log2 units (the stale max keeps exp2 below 256 and cancels in O / l).
//
// Roles (320 threads, persistent: one CTA per SM walks tiles blockIdx.x, +gridDim.x, ...):
// warps 0-7 softmax + epilogue: warp w reads TMEM lanes 32(w%4).. (its 32 rows) and owns one
// 64-key half of each pair (w < 4: the first block, w >= 4: the second), so every scheduler runs
// two softmax warps; the two halves of a row exchange their maxima through shared memory and keep
// one running max, two partial sums.  Warp 8 stages the next tile's selection rows in shared
// memory with coalesced loads, merges them into the union list and issues the TMA loads; warp 9
// allocates TMEM and issues the MMAs (one thread).  Every wait is bounded; a timeout sets the
// status word, the roles wind down, and the kernel waits (bounded) for its own copies and MMAs
// before it frees TMEM and returns.
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128;          // head dim
constexpr int kG = 16;           // query heads per KV group
constexpr int kTQ = 8;           // query tokens per tile
constexpr int kBlk = 64;         // keys per block
constexpr int kMaxSlots = 128;   // selection slots per row the kernel accepts
constexpr int kMaxList = kTQ * kMaxSlots;
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;

// Shared memory (offsets from a 1024-aligned base).
constexpr int kStages = 3;                            // K/V pair stages
constexpr int kHalfK = 8192;                          // one K box: [64 rows x 128 B]
constexpr int kPairBytes = 8 * kHalfK;                // K_a|K_b (d 0-63), K_a|K_b (d 64-127), V_a, V_b
constexpr int kOffKV = 0;
constexpr int kOffList = kOffKV + kStages * kPairBytes;
constexpr int kListBytes = kMaxList * 5;              // int32 ids + uint8 token masks
constexpr int kOffStage = kOffList + 2 * kListBytes;  // staged selection rows of one tile
constexpr int kSmemBytes = kOffStage + kTQ * kMaxSlots * 4 + 1024;

// TMEM columns: O [0,128), S buffers [128,256) and [256,384), Q buffers [384,448) and [448,512).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 128, kColQ0 = 384;

struct Bars {
    uint64_t q_full, q_seen;
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t list_full[2], list_empty[2];
    uint64_t fin;
    uint32_t tmem_base;
    int list_n[2];
    int abort;
    float xmax[2][128];  // per-half row maxima of the current pair
    float xl[128];       // second-half partial row sums, for the epilogue
    int sm_stop;         // set by a softmax thread whose wait failed; read after a barrier
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                              volatile int* abort) {
    if (*abort) return false;
    if (!mbar_wait(bar, parity, ctx)) {
        *abort = 1;
        return false;
    }
    return true;
}

// Max of 64 values held as raw fp32 bit patterns, 8 independent chains.
__device__ __forceinline__ float max64(const uint32_t* x) {
    float m[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) m[a] = __uint_as_float(x[a]);
#pragma unroll
    for (int j = 8; j < 64; j += 8)
#pragma unroll
        for (int a = 0; a < 8; ++a) m[a] = fmaxf(m[a], __uint_as_float(x[j + a]));
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Softmax numerators of one 64-key half: p = 2^(x * sl2 - m), packed to bf16 pairs; returns the
// sum of the fp32 p.  Keys j > lim are masked (lim = 63: none).
__device__ __forceinline__ float exp_half(const uint32_t* x, float sl2, float neg_m, int lim,
                                          uint32_t* pk) {
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float p0 = ex2(fmaf(__uint_as_float(x[2 * j]), sl2, neg_m));
        float p1 = ex2(fmaf(__uint_as_float(x[2 * j + 1]), sl2, neg_m));
        p0 = (2 * j <= lim) ? p0 : 0.f;
        p1 = (2 * j + 1 <= lim) ? p1 : 0.f;
        s[j & 3] += p0 + p1;
        pk[j] = pack_bf16x2(p0, p1);
    }
    return (s[0] + s[1]) + (s[2] + s[3]);
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_prefill_tc_kernel(const __nv_bfloat16* __restrict__ q,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out, int H,
                         int Hkv, int N, int slots, float sl2, int n_tiles, DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_per_seq = (N + kTQ - 1) / kTQ;
    volatile int* abort = &bars.abort;

    if (warp == 9) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.q_full, 8);
        mbar_init(&bars.q_seen, 1);
        for (int b = 0; b < kStages; ++b) {
            mbar_init(&bars.kv_full[b], 1);
            mbar_init(&bars.kv_empty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 8);
            mbar_init(&bars.pv_done[b], 1);
            mbar_init(&bars.list_full[b], 1);
            mbar_init(&bars.list_empty[b], 2);
        }
        mbar_init(&bars.fin, 1);
        bars.abort = 0;
        bars.sm_stop = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    auto list_id = [&](int lb) { return reinterpret_cast<int32_t*>(sm + kOffList + lb * kListBytes); };
    auto list_mask = [&](int lb) { return sm + kOffList + lb * kListBytes + kMaxList * 4; };

    if (warp == 8) {
        // ---------------------------------------------------------------- producer
        int32_t* stage = reinterpret_cast<int32_t*>(sm + kOffStage);
        int it = 0, gp = 0;
        int last_phase[kStages];
        for (int e = 0; e < kStages; ++e) last_phase[e] = -1;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            const int lb = it & 1;
            if (it >= 2 && !wait_or_abort(&bars.list_empty[lb], ((it - 2) >> 1) & 1, ctx, abort)) break;
            const int64_t bg = tile / tiles_per_seq;
            const int i0 = (tile % tiles_per_seq) * kTQ;
            const int c = i0 / kBlk;
            const int n_act = min(kTQ, N - i0);
            // Stage the tile's selection rows (contiguous in memory) with coalesced loads.
            const int32_t* src = idx + (bg * N + i0) * (int64_t)slots;
            for (int e = lane; e < n_act * slots; e += 32) stage[e] = src[e];
            __syncwarp();
            // 8-way merge of the ascending rows, one lane per token.
            const int32_t* row = stage + lane * slots;
            const bool active = lane < n_act;
            int p = 0, n = 0, prev = -1;
            while (true) {
                int head = 0x7fffffff;
                if (active && p < slots) {
                    const int v = row[p];
                    if (v >= 0) head = v;
                }
                const int m = __reduce_min_sync(0xffffffffu, head);
                if (m == 0x7fffffff) break;
                const unsigned msk = __ballot_sync(0xffffffffu, head == m);
                if (head == m) ++p;
                if (m > c) {  // in the future of every token of the tile
                    if (lane == 0) flag(ctx, kStatusBounds);
                    continue;
                }
                if (lane == 0) {
                    if (m == prev) {
                        list_mask(lb)[n - 1] |= (uint8_t)msk;
                    } else if (n < kMaxList) {
                        list_id(lb)[n] = m;
                        list_mask(lb)[n] = (uint8_t)msk;
                        ++n;
                    }
                }
                n = __shfl_sync(0xffffffffu, n, 0);
                prev = m;
            }
            if (lane == 0) {
                bars.list_n[lb] = n;
                mbar_arrive(&bars.list_full[lb]);
            }
            __syncwarp();
            int stop = 0;
            if (lane == 0) {
                for (int u = 0; u < n; u += 2, ++gp) {
                    const int s = gp % kStages, r = gp / kStages;
                    if (r >= 1 && !wait_or_abort(&bars.kv_empty[s], (r - 1) & 1, ctx, abort)) {
                        stop = 1;
                        break;
                    }
                    const int nb = min(2, n - u);
                    uint8_t* st = sm + kOffKV + s * kPairBytes;
                    mbar_arrive_expect_tx(&bars.kv_full[s], nb * 4 * kHalfK);
                    for (int e = 0; e < nb; ++e) {
                        const int y = list_id(lb)[u + e] * kBlk;
                        tma_load_3d(st + e * kHalfK, &tmK, &bars.kv_full[s], 0, y, (int)bg);
                        tma_load_3d(st + 2 * kHalfK + e * kHalfK, &tmK, &bars.kv_full[s], 64, y, (int)bg);
                        tma_load_3d(st + 4 * kHalfK + e * 2 * kHalfK, &tmV, &bars.kv_full[s], 0, y, (int)bg);
                        tma_load_3d(st + 5 * kHalfK + e * 2 * kHalfK, &tmV, &bars.kv_full[s], 64, y, (int)bg);
                    }
                    last_phase[s] = r;
                }
            }
            gp = __shfl_sync(0xffffffffu, gp, 0);
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop || *abort) break;
        }
        if (lane == 0)
            for (int e = 0; e < kStages; ++e)
                if (last_phase[e] >= 0) (void)mbar_wait(&bars.kv_full[e], last_phase[e] & 1, ctx);
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS2 = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idS1 = idesc_bf16_f32(128, 64, false, false);
            const uint32_t idPV = idesc_bf16_f32(128, kD, false, true);
            int it = 0, gp = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++it) {
                const int lb = it & 1;
                ok = wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort);
                if (!ok) break;
                const int n = bars.list_n[lb];
                const int np = (n + 1) >> 1;
                mbar_arrive(&bars.list_empty[lb]);
                ok = wait_or_abort(&bars.q_full, it & 1, ctx, abort);  // Q(tile) is in TMEM
                if (!ok) break;
                mbar_arrive(&bars.q_seen);
                tc_fence_after();
                const uint32_t aQ = tmem + kColQ0 + (it & 1) * 64;
                auto issue_s = [&](int j, int g) -> bool {
                    const int st = g % kStages, b = g & 1;
                    if (!wait_or_abort(&bars.kv_full[st], (g / kStages) & 1, ctx, abort)) return false;
                    tc_fence_after();
                    const uint32_t kb = smem_u32(sm + kOffKV + st * kPairBytes);
                    const uint32_t dS = tmem + kColS0 + b * 128;
                    const uint32_t id = (2 * j + 1 < n) ? idS2 : idS1;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint64_t bd = sdesc_sw128(kb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 32, 16, 1024);
                        mma_ts(dS, aQ + ks * 8, bd, id, ks > 0);
                    }
                    mma_commit(&bars.s_full[b]);
                    return true;
                };
                if (np > 0) ok = issue_s(0, gp);
                for (int j = 0; j < np && ok; ++j) {
                    const int g = gp + j;
                    if (j + 1 < np) {
                        ok = issue_s(j + 1, g + 1);
                        if (!ok) break;
                    }
                    ok = wait_or_abort(&bars.p_full[g & 1], (g >> 1) & 1, ctx, abort);
                    if (!ok) break;
                    tc_fence_after();
                    const int s = g & 1, st = g % kStages;
                    const uint32_t vb = smem_u32(sm + kOffKV + st * kPairBytes + 4 * kHalfK);
                    const uint32_t aP = tmem + kColS0 + s * 128;
                    const int ksteps = (2 * j + 1 < n) ? 8 : 4;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const uint64_t b = sdesc_sw128(vb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 16 * 128, kHalfK, 1024);
                        mma_ts(tmem + kColO, aP + ks * 8, b, idPV, (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars.kv_empty[st]);
                    mma_commit(&bars.pv_done[s]);
                }
                gp += np;
            }
            mma_commit(&bars.fin);
            (void)mbar_wait(&bars.fin, 0, ctx);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        // The 8 softmax warps meet at named barriers (bar.sync 2 / 1, 256 threads), which have
        // no time limit.  So they never leave a loop one by one: a failed (timed-out) wait
        // records sm_stop and the thread carries on without touching TMEM; after the next
        // barrier every softmax thread reads the same sm_stop and they all leave together.
        const int r = tid & 127;            // row = TMEM lane
        const int half = tid >> 7;          // 0: first block of a pair, 1: second
        const int t = r % kTQ, hh = r / kTQ;
        const uint32_t lane_base = tmem_lane_base(warp);
        // Q rows of a tile -> registers (this thread: row r, columns 64*half .. +63), then TMEM.
        auto load_q = [&](int T, uint4 (&qv)[8]) {
            const int64_t bgT = T / tiles_per_seq;
            const int iT = (T % tiles_per_seq) * kTQ + t;
            if (iT < N) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    q + (((bgT / Hkv) * H + (bgT % Hkv) * kG + hh) * (int64_t)N + iT) * kD + half * 64);
#pragma unroll
                for (int e = 0; e < 8; ++e) qv[e] = src[e];
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) qv[e] = make_uint4(0, 0, 0, 0);
            }
        };
        auto store_q = [&](int buf, const uint4 (&qv)[8]) {
            tmem_st32(tmem + lane_base + kColQ0 + buf * 64 + half * 32,
                      *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.q_full);
        };
        {
            uint4 qv[8];
            load_q(blockIdx.x, qv);
            store_q(0, qv);
        }
        // sm_stop holds the index of the first barrier after which everybody must leave: a
        // failure before barrier k (nbar == k-1 completed) names k, one after it names k+1, so a
        // thread that reads the flag right after barrier k never sees a later failure early.
        volatile int* sm_stop = &bars.sm_stop;
        int nbar = 0;                       // named barriers (id 2) passed so far
        bool dead = false;                  // this thread saw a failed wait
        auto fail = [&]() {
            dead = true;
            atomicCAS(&bars.sm_stop, 0, nbar + 1);
            *abort = 1;
        };
        auto stop_now = [&]() { const int v = *sm_stop; return v != 0 && v <= nbar; };
        int it = 0, gp = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!dead && !mbar_wait(&bars.list_full[lb], (it >> 1) & 1, ctx)) fail();
            asm volatile("bar.sync 2, 256;" ::: "memory");
            ++nbar;
            if (stop_now()) break;
            const int n = bars.list_n[lb];
            const int np = (n + 1) >> 1;
            const int32_t* ids = list_id(lb);
            const uint8_t* msks = list_mask(lb);
            const int64_t bg = tile / tiles_per_seq;
            const int i0 = (tile % tiles_per_seq) * kTQ;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            float m_run = -INFINITY, l = 0.f;  // running max (scaled log2 units), partial sum
            bool stop = false;
            // Q of this CTA's next tile: loaded now, written to TMEM after the first pair (by then
            // the MMA thread has taken this tile's Q, see q_seen), into the other Q buffer.
            const int next = tile + gridDim.x;
            bool q_pending = next < n_tiles;
            uint4 qv[8];
            if (q_pending) load_q(next, qv);
            auto flush_q = [&]() {
                if (!q_pending) return;
                q_pending = false;
                if (!dead && !mbar_wait(&bars.q_seen, it & 1, ctx)) fail();
                if (!__any_sync(0xffffffffu, dead)) store_q((it + 1) & 1, qv);
            };
            for (int j = 0; j < np; ++j) {
                const int g = gp + j, s = g & 1;
                const int u = 2 * j + half;     // this warp's union block
                const bool has = u < n;
                const int blk = has ? ids[u] : -1;
                const bool sel = has && ((msks[u] >> t) & 1);
                // last visible key of this half (-1: none)
                const int lim = !sel ? -1 : (blk == c ? i - blk * kBlk : kBlk - 1);
                if (!dead && !mbar_wait(&bars.s_full[s], (g >> 1) & 1, ctx)) fail();
                tc_fence_after();
                const uint32_t colS = tmem + lane_base + kColS0 + s * 128;
                uint32_t x[64];
                const bool ld = __any_sync(0xffffffffu, has && !dead);
                if (ld) {
                    tmem_ld32(colS + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
                    tmem_ld32(colS + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
                    tmem_ld_wait();
                }
                if (lim >= 0 && lim < kBlk - 1)
#pragma unroll
                    for (int jj = 0; jj < 64; ++jj) x[jj] = jj <= lim ? x[jj] : __float_as_uint(-INFINITY);
                const float mh = (lim >= 0 && ld) ? max64(x) * sl2 : -INFINITY;
                bars.xmax[half][r] = mh;
                // Both halves have loaded their S columns before either overwrites S with P.
                asm volatile("bar.sync 2, 256;" ::: "memory");
                ++nbar;
                if (stop_now()) { stop = true; break; }
                const float mx = fmaxf(mh, bars.xmax[half ^ 1][r]);
                const bool grow = mx > m_run + 8.f;
                // O holds this row's earlier pairs once m_run is finite: rescale it (first half).
                const bool need_rescale = grow && m_run != -INFINITY;
                if (half == 0 && __any_sync(0xffffffffu, need_rescale)) {
                    if (j >= 1 && !dead) {
                        const int gq = g - 1;
                        if (!mbar_wait(&bars.pv_done[gq & 1], (gq >> 1) & 1, ctx)) fail();
                    }
                    if (!__any_sync(0xffffffffu, dead)) {
                        tc_fence_after();
                        const float alpha = need_rescale ? ex2(m_run - mx) : 1.f;
#pragma unroll 1
                        for (int c0 = 0; c0 < kD; c0 += 32) {
                            uint32_t orr[32];
                            tmem_ld32(tmem + lane_base + kColO + c0, orr);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 32; ++q) orr[q] = __float_as_uint(__uint_as_float(orr[q]) * alpha);
                            tmem_st16(tmem + lane_base + kColO + c0, *reinterpret_cast<uint32_t(*)[16]>(&orr[0]));
                            tmem_st16(tmem + lane_base + kColO + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&orr[16]));
                        }
                        tmem_st_wait();
                    }
                }
                if (grow) {
                    l = (m_run == -INFINITY) ? 0.f : l * ex2(m_run - mx);
                    m_run = mx;
                }
                if (ld && !__any_sync(0xffffffffu, dead)) {
                    uint32_t pk[32];
                    if (lim >= 0) {
                        l += exp_half(x, sl2, -m_run, lim, pk);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) pk[q] = 0u;
                    }
                    tmem_st16(colS + half * 32, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                    tmem_st16(colS + half * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[s]);
                flush_q();
            }
            if (stop) break;
            flush_q();
            // Epilogue: l = sum of both halves; each half writes 64 of the 128 output columns.
            if (half == 1) bars.xl[r] = l;
            asm volatile("bar.sync 2, 256;" ::: "memory");
            ++nbar;
            if (half == 0) bars.xmax[0][r] = l + bars.xl[r];  // broadcast of the row total
            asm volatile("bar.sync 2, 256;" ::: "memory");
            ++nbar;
            const float ltot = bars.xmax[0][r];
            const int64_t orow = (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
            if (np > 0) {
                const int gl = gp + np - 1;
                if (!dead && !mbar_wait(&bars.pv_done[gl & 1], (gl >> 1) & 1, ctx)) fail();
                if (!__any_sync(0xffffffffu, dead)) {
                    tc_fence_after();
                    const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
#pragma unroll 1
                    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
                        uint32_t orr[32];
                        tmem_ld32(tmem + lane_base + kColO + c0, orr);
                        tmem_ld_wait();
                        if (i < N) {
                            uint4 w[4];
                            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                wp[q] = pack_bf16x2(__uint_as_float(orr[2 * q]) * inv,
                                                    __uint_as_float(orr[2 * q + 1]) * inv);
                            uint4* d4 = reinterpret_cast<uint4*>(out + orow + c0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) d4[q] = w[q];
                        }
                    }
                    tc_fence_before();
                }
            } else if (i < N) {
                uint4* d4 = reinterpret_cast<uint4*>(out + orow + half * 64);
                for (int q = 0; q < 8; ++q) d4[q] = make_uint4(0, 0, 0, 0);
            }
            gp += np;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (tid == 0) mbar_arrive(&bars.list_empty[lb]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool sparse_prefill_tc_supported(int H, int Hkv, int d) {
    return d == kD && Hkv > 0 && H == Hkv * kG;
}

cudaError_t launch_sparse_prefill_tc(const void* q, const void* k, const void* v,
                                     const int32_t* idx, void* o, int B, int H, int Hkv, int N,
                                     int d, int slots, float scale, cudaStream_t st, DevCtx ctx) {
    if (d != kD || H != Hkv * kG || slots > kMaxSlots) return cudaErrorNotSupported;
    CUtensorMap tmK, tmV;
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    auto make3 = [&](CUtensorMap* m, const void* base, uint64_t rows, uint64_t planes,
                     uint32_t box_rows, uint32_t box_planes) -> bool {
        cuuint64_t dims[3] = {(cuuint64_t)kD, rows, planes};
        cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * rows};
        cuuint32_t box[3] = {64, box_rows, box_planes};
        cuuint32_t estr[3] = {1, 1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!make3(&tmK, k, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1) ||
        !make3(&tmV, v, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1))
        return cudaErrorInvalidValue;
    static int num_sms = 0;
    if (!num_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (num_sms <= 0) num_sms = 148;
    }
    cudaError_t e = ensure_smem<sparse_prefill_tc_kernel>(kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles_per_seq = (N + kTQ - 1) / kTQ;
    const int n_tiles = tiles_per_seq * B * Hkv;
    const int grid = n_tiles < num_sms ? n_tiles : num_sms;
    const float sl2 = scale * 1.4426950408889634f;
    sparse_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        static_cast<const __nv_bfloat16*>(q), tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), H, Hkv,
        N, slots, sl2, n_tiles, ctx);
    return cudaGetLastError();
}

}  // namespace sala
