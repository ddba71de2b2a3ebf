// Block-sparse softmax attention prefill on the 5th-generation tensor cores (sm_100a).
//
// Work unit: 16 consecutive query tokens of one KV group, split into two tiles A (tokens 0-7) and
// B (tokens 8-15) of 128 rows each (row = head * 8 + token, the 16 query heads of the group), the
// M of one tcgen05 MMA.  The 16 tokens share their query block (16 divides 64), hence the forced
// blocks and the diagonal; their top-k choices differ, so the unit walks the UNION of the 16
// selections (ascending) and each row masks the blocks its token did not choose.  Executed FLOPs
// exceed the algorithmic ones by that union overhead; each row's own sum over its selected keys
// is exact.
//
// The union is consumed two blocks at a time (a "pair", 128 keys), and the two tiles ping-pong on
// the tensor core (the structure FlashAttention-4 uses on this architecture):
//   S_X  = Q_X [K_a; K_b]^T      M=128 N=128 K=128  (X = A, B; Q from shared memory, the two K
//                                                    tiles back to back in shared memory)
//   P_X  = online softmax of S_X (per row: selection mask per block, causal mask on the diagonal)
//   O_X += P_X [V_a; V_b]        M=128 N=128 K=128  (A = P_X from TMEM, aliasing S_X)
// Issue order per pair: PV_A, S_A(next), PV_B, S_B(next), so the softmax of one tile overlaps the
// MMAs of the other.  O_X is rescaled only when a row's running max grows by more than 8 in log2
// units (the stale max keeps exp2 below 256 and cancels in O / l).
//
// Roles (384 threads, persistent: one CTA per SM walks units blockIdx.x, +gridDim.x, ...):
// warps 0-3 softmax + epilogue of tile A, warps 4-7 of tile B (thread = row = TMEM lane; each
// thread owns its whole row, so the two warpgroups never wait for each other inside a unit);
// warp 8 stages the next unit's 16 selection rows with coalesced loads, merges them into the union
// list and issues the TMA loads (Q tiles, then a 2-stage ring of K/V pairs); warp 9 allocates TMEM
// and issues the MMAs (one thread); warps 10-11 only complete the third warpgroup.  Every wait is bounded; a timeout sets the status word, the
// roles wind down, and the kernel waits (bounded) for its own copies and MMAs before it frees TMEM.
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128;          // head dim
constexpr int kG = 16;           // query heads per KV group
constexpr int kTQ = 8;           // query tokens per tile
constexpr int kUT = 16;          // query tokens per unit (two tiles)
constexpr int kBlk = 64;         // keys per block
constexpr int kMaxSlots = 80;    // selection slots per row the kernel accepts
constexpr int kMaxList = kUT * kMaxSlots;
constexpr int kThreads = 384;
// Register split (setmaxnreg): the two softmax warpgroups hold a whole S row per thread; the
// third warpgroup (producer, MMA issuer, two idle warps) needs little.  256 * 216 + 128 * 72 =
// 384 * 168, the per-thread count the block is launched with.
constexpr int kRegsLaunch = 168, kRegsSoftmax = 216, kRegsOther = 72;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch, "register split");
constexpr int kStages = 2;       // K/V pair stages

// Shared memory (offsets from a 1024-aligned base).
constexpr int kQBytes = 128 * kD * 2;                 // one Q tile: 2 sub-tiles [128 rows x 128 B]
constexpr int kHalfK = 8192;                          // one K box: [64 rows x 128 B]
constexpr int kPairBytes = 8 * kHalfK;                // K_a|K_b (d 0-63), K_a|K_b (d 64-127), V_a, V_b
constexpr int kOffQ = 0;                              // Q_A, Q_B
constexpr int kOffKV = 2 * kQBytes;
constexpr int kOffList = kOffKV + kStages * kPairBytes;
constexpr int kListBytes = kMaxList * 6;              // int32 ids + uint16 token masks
constexpr int kOffStage = kOffList + 2 * kListBytes;  // staged selection rows of one unit
constexpr int kSmemBytes = kOffStage + kUT * kMaxSlots * 4 + 1024;

// TMEM columns: O_A [0,128), O_B [128,256), S_A [256,384), S_B [384,512).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], p_full[2], pv_done[2];  // per tile
    uint64_t list_full[2], list_empty[2];
    uint64_t fin;
    uint32_t tmem_base;
    int list_n[2];
    int abort;
    int sm_stop;
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

__device__ __forceinline__ uint32_t (&sub32(uint32_t (&a)[128], int k))[32] {
    return *reinterpret_cast<uint32_t(*)[32]>(a + 32 * k);
}

// Max over 64 raw fp32 values, four independent chains of three-input maxima.
__device__ __forceinline__ float max64(const uint32_t* s) {
    float m[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t* x = s + 16 * c;
        float v = fmaxf(__uint_as_float(x[0]), __uint_as_float(x[1]));
#pragma unroll
        for (int k = 2; k < 16; k += 2) v = fmax3(v, __uint_as_float(x[k]), __uint_as_float(x[k + 1]));
        m[c] = v;
    }
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Max over the values at positions 0..lim of 64 (-inf when lim < 0).
__device__ __forceinline__ float max64_masked(const uint32_t* s, int lim) {
    float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < 64; ++k)
        m[k & 3] = fmaxf(m[k & 3], k <= lim ? __uint_as_float(s[k]) : -INFINITY);
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// p = 2^(s * sl2 + nb) for 64 keys, packed to 32 bf16 pairs and stored to TMEM columns
// taddr .. taddr+31 in two pieces of 16; sums added to a0..a3.  kMasked zeroes the keys past lim
// (the causal edge).
template <bool kMasked>
__device__ __forceinline__ void exp_block(const uint32_t* s, float sl2, float nb, int lim,
                                          uint32_t taddr, float& a0, float& a1, float& a2,
                                          float& a3) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int k = 32 * h + 2 * q;
            float y0, y1;
            fma2_bcast(y0, y1, __uint_as_float(s[k]), __uint_as_float(s[k + 1]), sl2, nb);
            float p0 = ex2(y0), p1 = ex2(y1);
            if (kMasked) {
                p0 = k <= lim ? p0 : 0.f;
                p1 = k + 1 <= lim ? p1 : 0.f;
            }
            if (q & 1) add2(a2, a3, p0, p1);
            else add2(a0, a1, p0, p1);
            pk[q] = pack_bf16x2(p0, p1);
        }
        tmem_st16(taddr + 16 * h, pk);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out, int H,
                         int Hkv, int N, int slots, float sl2, int n_units, DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int units_per_seq = (N + kUT - 1) / kUT;
    volatile int* abort = &bars.abort;

    if (warp == 9) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_empty, 1);
        for (int b = 0; b < kStages; ++b) {
            mbar_init(&bars.kv_full[b], 1);
            mbar_init(&bars.kv_empty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 4);
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
    auto list_mask = [&](int lb) {
        return reinterpret_cast<uint16_t*>(sm + kOffList + lb * kListBytes + kMaxList * 4);
    };

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (warp == 8) {
            // ---------------------------------------------------------------- producer
            int32_t* stage = reinterpret_cast<int32_t*>(sm + kOffStage);
            int it = 0, gp = 0;
            uint32_t q_issued = 0;
            int last0 = -1, last1 = -1;
            for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
                const int lb = it & 1;
                if (it >= 2 && !wait_or_abort(&bars.list_empty[lb], ((it - 2) >> 1) & 1, ctx, abort)) break;
                const int64_t bg = unit / units_per_seq;
                const int i0 = (unit % units_per_seq) * kUT;
                const int c = i0 / kBlk;
                const int n_act = min(kUT, N - i0);
                // Stage the unit's selection rows (contiguous in memory) with coalesced loads.
                const int32_t* src = idx + (bg * N + i0) * (int64_t)slots;
                for (int e = lane; e < n_act * slots; e += 32) stage[e] = src[e];
                __syncwarp();
                // 16-way merge of the ascending rows, one lane per token.
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
                    if (m > c) {  // in the future of every token of the unit
                        if (lane == 0) flag(ctx, kStatusBounds);
                        continue;
                    }
                    if (lane == 0) {
                        if (m == prev) {
                            list_mask(lb)[n - 1] |= (uint16_t)msk;
                        } else if (n < kMaxList) {
                            list_id(lb)[n] = m;
                            list_mask(lb)[n] = (uint16_t)msk;
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
                    // Q tiles A and B: 16 heads x 8 tokens x 128 columns each.
                    if (it >= 1 && !wait_or_abort(&bars.q_empty, (it - 1) & 1, ctx, abort)) stop = 1;
                    if (!stop) {
                        mbar_arrive_expect_tx(&bars.q_full, 2 * kQBytes);
                        const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
                        for (int x = 0; x < 2; ++x) {
                            uint8_t* qd = sm + kOffQ + x * kQBytes;
                            tma_load_3d(qd, &tmQ, &bars.q_full, 0, i0 + x * kTQ, z);
                            tma_load_3d(qd + kQBytes / 2, &tmQ, &bars.q_full, 64, i0 + x * kTQ, z);
                        }
                        q_issued = it + 1;
                    }
                    for (int u = 0; u < n && !stop; u += 2, ++gp) {
                        const int s = gp & 1, r = gp >> 1;
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
                        if (s == 0) last0 = r; else last1 = r;
                    }
                }
                gp = __shfl_sync(0xffffffffu, gp, 0);
                stop = __shfl_sync(0xffffffffu, stop, 0);
                if (stop || *abort) break;
            }
            if (lane == 0) {
                if (q_issued) (void)mbar_wait(&bars.q_full, (q_issued - 1) & 1, ctx);
                if (last0 >= 0) (void)mbar_wait(&bars.kv_full[0], last0 & 1, ctx);
                if (last1 >= 0) (void)mbar_wait(&bars.kv_full[1], last1 & 1, ctx);
            }
        } else if (warp == 9) {
            // ---------------------------------------------------------------- MMA issuer
            if (lane == 0) {
                const uint32_t idS2 = idesc_bf16_f32(128, 128, false, false);
                const uint32_t idS1 = idesc_bf16_f32(128, 64, false, false);
                const uint32_t idPV = idesc_bf16_f32(128, kD, false, true);
                int it = 0, gp = 0;
                bool ok = true;
                for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++it) {
                    const int lb = it & 1;
                    ok = wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort);
                    if (!ok) break;
                    const int n = bars.list_n[lb];
                    const int np = (n + 1) >> 1;
                    mbar_arrive(&bars.list_empty[lb]);
                    ok = wait_or_abort(&bars.q_full, it & 1, ctx, abort);
                    if (!ok) break;
                    tc_fence_after();
                    // S_x(j) of tile x; waits for the pair's K/V only when asked.
                    auto issue_s = [&](int x, int j, bool wait_kv) -> bool {
                        const int g = gp + j, s = g & 1;
                        if (wait_kv && !wait_or_abort(&bars.kv_full[s], (g >> 1) & 1, ctx, abort)) return false;
                        tc_fence_after();
                        const uint32_t q0 = smem_u32(sm + kOffQ + x * kQBytes);
                        const uint32_t kb = smem_u32(sm + kOffKV + s * kPairBytes);
                        const uint32_t id = (2 * j + 1 < n) ? idS2 : idS1;
    #pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks) {
                            const uint64_t a = sdesc_sw128(q0 + (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32, 16, 1024);
                            const uint64_t b = sdesc_sw128(kb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 32, 16, 1024);
                            mma_ss(tmem + kColS + x * 128, a, b, id, ks > 0);
                        }
                        mma_commit(&bars.s_full[x]);
                        return true;
                    };
                    auto issue_pv = [&](int x, int j) -> bool {
                        const int g = gp + j, s = g & 1;
                        if (!wait_or_abort(&bars.p_full[x], g & 1, ctx, abort)) return false;
                        tc_fence_after();
                        const uint32_t vb = smem_u32(sm + kOffKV + s * kPairBytes + 4 * kHalfK);
                        const uint32_t aP = tmem + kColS + x * 128;
                        const int ksteps = (2 * j + 1 < n) ? 8 : 4;
                        for (int ks = 0; ks < ksteps; ++ks) {
                            const uint64_t b = sdesc_sw128(vb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 16 * 128, kHalfK, 1024);
                            mma_ts(tmem + kColO + x * 128, aP + ks * 8, b, idPV, (j > 0 || ks > 0) ? 1u : 0u);
                        }
                        mma_commit(&bars.pv_done[x]);
                        return true;
                    };
                    if (np > 0) ok = issue_s(0, 0, true) && issue_s(1, 0, false);
                    for (int j = 0; j < np && ok; ++j) {
                        const bool more = j + 1 < np;
                        ok = issue_pv(0, j);
                        if (ok && more) ok = issue_s(0, j + 1, true);
                        if (ok) ok = issue_pv(1, j);
                        if (ok) mma_commit(&bars.kv_empty[(gp + j) & 1]);
                        if (ok && more) ok = issue_s(1, j + 1, false);
                    }
                    mma_commit(&bars.q_empty);  // every MMA reading this unit's Q has been issued
                    gp += np;
                }
                mma_commit(&bars.fin);
                (void)mbar_wait(&bars.fin, 0, ctx);
            }
            __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ---------------------------------------------------------------- softmax + epilogue
        // Warpgroup x (0: tile A, 1: tile B); thread = row r of the tile = TMEM lane r.  The two
        // warpgroups meet only at one named barrier per unit (bar.sync 1, 256 threads).  A failed
        // (timed-out) wait is recorded in sm_stop; every softmax thread reads sm_stop right after
        // that barrier and all leave together (a failure before barrier k names k, one after it
        // names k+1), so no thread is ever left waiting at a barrier.
        const int x = warp >> 2;
        const int r = tid & 127;
        const int t = x * kTQ + r % kTQ, hh = r / kTQ;   // token within the unit, head
        const uint32_t lane_base = tmem_lane_base(warp);
        const uint32_t colO = tmem + lane_base + kColO + x * 128;
        const uint32_t colS = tmem + lane_base + kColS + x * 128;
        volatile int* sm_stop = &bars.sm_stop;
        int nbar = 0;
        bool dead = false;
        auto fail = [&]() {
            dead = true;
            atomicCAS(&bars.sm_stop, 0, nbar + 1);
            *abort = 1;
        };
        int it = 0, gp = 0;
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!dead && !mbar_wait(&bars.list_full[lb], (it >> 1) & 1, ctx)) fail();
            const int n = dead ? 0 : bars.list_n[lb];
            const int np = (n + 1) >> 1;
            const int32_t* ids = list_id(lb);
            const uint16_t* msks = list_mask(lb);
            const int64_t bg = unit / units_per_seq;
            const int i0 = (unit % units_per_seq) * kUT;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            float m_run = -INFINITY, l = 0.f;  // running max (scaled log2 units), row sum
            for (int j = 0; j < np; ++j) {
                const int g = gp + j;
                const bool two = 2 * j + 1 < n;
                const int blk_a = ids[2 * j];
                const int blk_b = two ? ids[2 * j + 1] : -1;
                const bool sel_a = (msks[2 * j] >> t) & 1;
                const bool sel_b = two && ((msks[2 * j + 1] >> t) & 1);
                // last visible key of each block (-1: none)
                const int lim_a = !sel_a ? -1 : (blk_a == c ? i - blk_a * kBlk : kBlk - 1);
                const int lim_b = !sel_b ? -1 : (blk_b == c ? i - blk_b * kBlk : kBlk - 1);
                if (!dead && !mbar_wait(&bars.s_full[x], g & 1, ctx)) fail();
                tc_fence_after();
                const bool go = !__any_sync(0xffffffffu, dead);
                // The pair's S row is read from TMEM once, into 128 registers.  Blocks the token did
                // not select drop out through the exponent bias (2^-inf = 0); the causal mask inside
                // the diagonal block, the one block a token sees in part, costs a select per element
                // on the pair that holds it only.
                const bool diag = (blk_a == c) || (blk_b == c);  // uniform over the CTA
                uint32_t sr[128];
                float mx = -INFINITY;
                if (go) {
                    tmem_ld32(colS, sub32(sr, 0));
                    tmem_ld32(colS + 32, sub32(sr, 1));
                    if (two) {
                        tmem_ld32(colS + 64, sub32(sr, 2));
                        tmem_ld32(colS + 96, sub32(sr, 3));
                    }
                    tmem_ld_wait();
                    float ma, mb = -INFINITY;
                    if (diag) {
                        ma = max64_masked(sr, lim_a);
                        if (two) mb = max64_masked(sr + 64, lim_b);
                    } else {
                        ma = lim_a >= 0 ? max64(sr) : -INFINITY;
                        if (two && lim_b >= 0) mb = max64(sr + 64);
                    }
                    mx = fmaxf(ma, mb);
                }
                mx *= sl2;
                const bool grow = mx > m_run + 8.f;
                const bool need_rescale = grow && m_run != -INFINITY;
                const float alpha = need_rescale ? ex2(m_run - mx) : 1.f;
                if (grow) {
                    l = (m_run == -INFINITY) ? 0.f : l * alpha;
                    m_run = mx;
                }
                // p = 2^(s * sl2 - m) as bf16 pairs over the first 64 columns of S (already read).
                if (go && !__any_sync(0xffffffffu, dead)) {
                    const float nb_a = lim_a >= 0 ? -m_run : -INFINITY;
                    const float nb_b = lim_b >= 0 ? -m_run : -INFINITY;
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                    if (diag) exp_block<true>(sr, sl2, nb_a, lim_a, colS, a0, a1, a2, a3);
                    else exp_block<false>(sr, sl2, nb_a, lim_a, colS, a0, a1, a2, a3);
                    if (two) {
                        if (diag) exp_block<true>(sr + 64, sl2, nb_b, lim_b, colS + 32, a0, a1, a2, a3);
                        else exp_block<false>(sr + 64, sl2, nb_b, lim_b, colS + 32, a0, a1, a2, a3);
                    }
                    l += (a0 + a1) + (a2 + a3);
                }
                // Rescale O_x by 2^(m_old - m_new) where the max grew past the threshold (before
                // this thread releases P, so before PV(j) can add into O_x).
                if (go && __any_sync(0xffffffffu, need_rescale)) {
                    if (j >= 1) {  // the previous PV into O_x must be complete
                        if (!dead && !mbar_wait(&bars.pv_done[x], (g - 1) & 1, ctx)) fail();
                    }
                    if (!__any_sync(0xffffffffu, dead)) {
                        tc_fence_after();
#pragma unroll 1
                        for (int c0 = 0; c0 < kD; c0 += 32) {
                            uint32_t orr[32];
                            tmem_ld32(colO + c0, orr);
                            tmem_ld_wait();
#pragma unroll
                            for (int q = 0; q < 32; ++q) orr[q] = __float_as_uint(__uint_as_float(orr[q]) * alpha);
                            tmem_st32(colO + c0, orr);
                        }
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[x]);
            }
            // Epilogue: O_x / l -> bf16 -> global.
            const int64_t orow = (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
            if (np > 0) {
                const int gl = gp + np - 1;
                if (!dead && !mbar_wait(&bars.pv_done[x], gl & 1, ctx)) fail();
                if (!__any_sync(0xffffffffu, dead)) {
                    tc_fence_after();
                    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                    for (int c0 = 0; c0 < kD; c0 += 32) {
                        uint32_t orr[32];
                        tmem_ld32(colO + c0, orr);
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
            } else if (i < N && !dead) {
                uint4* d4 = reinterpret_cast<uint4*>(out + orow);
                for (int q = 0; q < kD / 8; ++q) d4[q] = make_uint4(0, 0, 0, 0);
            }
            gp += np;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            ++nbar;
            if (tid == 0 && !dead) mbar_arrive(&bars.list_empty[lb]);
            const int v = *sm_stop;
            if (v != 0 && v <= nbar) break;
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
    CUtensorMap tmQ, tmK, tmV;
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
    if (!make3(&tmQ, q, (uint64_t)N, (uint64_t)B * H, kTQ, kG) ||
        !make3(&tmK, k, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1) ||
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
    // setmaxnreg.inc waits until the block's pool has the registers, so launch only when the
    // compiled per-thread count covers the split.
    static int regs_ok = -1;
    if (regs_ok < 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, sparse_prefill_tc_kernel);
        if (e != cudaSuccess) return e;
        regs_ok = fa.numRegs * kThreads >= 256 * kRegsSoftmax + 128 * kRegsOther ? 1 : 0;
    }
    if (!regs_ok) return cudaErrorNotSupported;
    const int units_per_seq = (N + kUT - 1) / kUT;
    const int n_units = units_per_seq * B * Hkv;
    const int grid = n_units < num_sms ? n_units : num_sms;
    const float sl2 = scale * 1.4426950408889634f;
    sparse_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), H, Hkv, N, slots, sl2, n_units, ctx);
    return cudaGetLastError();
}

}  // namespace sala
