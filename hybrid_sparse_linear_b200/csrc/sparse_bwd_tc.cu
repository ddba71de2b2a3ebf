// Tensor-core passes of the block-sparse attention backward (sm_100a), selection held fixed.
// Notation (per query row i of a KV group, key j):  P_ij = exp(scale q_i.k_j - lse_i) on the
// visible keys, dP_ij = do_i . v_j, D_i = do_i . o_i, dS_ij = P_ij (dP_ij - D_i);
//   dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij do_i.
//
// dq pass (query side): the forward's work units.  A unit is 16 consecutive tokens of one KV
// group as two 128-row tiles (row = head * 8 + token) walking the union of their selections, K
// and V of each union block loaded once for both tiles.  D_i = do_i . o_i comes from the training
// forward's output carried to ~2^-16 (o plus its bf16 residual, P taken as hi + lo in its P V):
// dP_ij - D_i cancels where the softmax is peaked, so D must match the P the backward forms
// (from the same lse and ex2) far better than a bf16 o does.  Per block and active tile X:
//   S_X  = Q_X K_b^T      M=128 N=64 K=128    (TMEM)
//   dP_X = dO_X V_b^T     M=128 N=64 K=128    (TMEM)
//   dS_X = P (dP - D) as two bf16 terms hi + lo (hi over S_X's columns, lo over dP_X's), and
//   dQ_X += hi K_b + lo K_b   M=128 N=128 K=64   (A from TMEM, B = K_b N-major).  The rows of dS sum to zero while the keys of a group share
//   a large common part, so dq = scale sum_j dS_ij k_j cancels: one bf16 term would leave an
//   error of ~2^-9 sum_j |dS_ij| |k_j|, near 1 % of max |dq| on peaked selections.
// TMEM holds dQ_A, dQ_B (128 columns each) and one S | dP pair per tile (128 columns each), so
// a tile's chain is S, dP -> dS -> dQ; the two tiles' chains, each issued by its own thread,
// interleave on the tensor core.  The epilogue scales dQ by `scale` and writes bf16.
//
// dk / dv pass (key side): one persistent CTA per SM takes an equal share of the transposed
// selection (all (batch, group, key block) token lists laid end to end).  A segment is the part
// of one block's list inside the share; its K and V sit in a shared buffer, and its
// tokens go in tiles of 8 (16 heads each: row = slot * 16 + head), their Q and dO rows gathered
// by TMA, 16 rows per token.  Per tile:
//   S = Q K_b^T, dP = dO V_b^T                       (M=128 N=64 K=128, K-major operands)
//   P, dS = P (dP - D) as bf16 rows in shared memory (the row's causal edge on the diagonal)
//   dV_b^T += dO^T P,  dK_b^T += Q^T dS            (M=128 (d) N=64 (keys) K=128 (rows); A and
//                                                    B read M- / N-major)
// dK^T, dV^T accumulate in TMEM over the segment (two buffers, so one drains while the next
// fills); at the segment's end four epilogue warps add them into fp32 dk / dv accumulators.
//
// Every wait is bounded; a timeout sets the status word and the roles wind down.
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128;        // head dim
constexpr int kG = 16;         // query heads per KV group
constexpr int kBlk = 64;       // keys per block
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kHalfQ = 16384;  // one [128 rows x 128 B] half of a Q / dO tile
constexpr int kTileBytes = 2 * kHalfQ;
constexpr int kHalfBlk = 8192;  // one [64 rows x 128 B] half of K_b or V_b
constexpr int kKVBytes = 4 * kHalfBlk;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                              volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (!mbar_wait(bar, parity, ctx)) {
        *abort = 1;
        return false;
    }
    return true;
}

// dS for 32 keys k0 .. k0+31 of one row from raw S and dP (TMEM words), as two bf16 terms
// dS = hi + lo (lo = the rounding residual of hi), each packed to 16 bf16 pairs.  Keys past lim
// (causal edge, unselected block, padding row) give exact zeros.
__device__ __forceinline__ void ds_half(const uint32_t (&s)[32], const uint32_t (&dp)[32], int k0,
                                        int lim, float sl2, float nl, float dv,
                                        uint32_t (&hi)[16], uint32_t (&lo)[16]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const int k = k0 + 2 * q;
        const float p0 = k <= lim ? ex2(fmaf(__uint_as_float(s[2 * q]), sl2, nl)) : 0.f;
        const float p1 = k + 1 <= lim ? ex2(fmaf(__uint_as_float(s[2 * q + 1]), sl2, nl)) : 0.f;
        const float d0 = p0 * (__uint_as_float(dp[2 * q]) - dv);
        const float d1 = p1 * (__uint_as_float(dp[2 * q + 1]) - dv);
        hi[q] = pack_bf16x2(d0, d1);
        lo[q] = pack_bf16x2(d0 - __uint_as_float(hi[q] << 16), d1 - __uint_as_float(hi[q] & 0xffff0000u));
    }
}

// ================================================================================== dq pass
namespace dqp {

constexpr int kTQ = 8;           // tokens per tile
constexpr int kUT = 16;          // tokens per unit
constexpr int kMaxSlots = 80;
constexpr int kMaxList = kUT * kMaxSlots;
constexpr int kThreads = 384;
constexpr int kStages = 2;
constexpr int kOffDO = 2 * kTileBytes;                // Q_A, Q_B, then dO_A, dO_B
constexpr int kOffRing = 4 * kTileBytes;
constexpr int kOffList = kOffRing + kStages * kKVBytes;
constexpr int kListBytes = kMaxList * 6;              // int32 ids + uint16 token masks
constexpr int kOffStage = kOffList + 2 * kListBytes;
constexpr int kSmemBytes = kOffStage + kUT * kMaxSlots * 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256;  // S_X at kColS + 128 X, dP_X at +64; dQ_X at 128 X

struct Bars {
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], p_full[2], dq_done[2];
    uint64_t q_full, q_empty;
    uint64_t list_full[2], list_empty[2];
    uint64_t fin[2];
    uint32_t tmem_base;
    int list_n[2];
    int abort;
    int sm_stop;
};

}  // namespace dqp

__global__ void __launch_bounds__(dqp::kThreads, 1)
sparse_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const int32_t* __restrict__ idx, const float* __restrict__ lse,
                    const float* __restrict__ delta, __nv_bfloat16* __restrict__ dq, int H,
                    int Hkv, int N, int slots, float sl2, float scale, int n_units, DevCtx ctx) {
    using namespace dqp;
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
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 2);  // released by both issuers
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 4);
            mbar_init(&bars.dq_done[b], 1);
            mbar_init(&bars.list_full[b], 1);
            mbar_init(&bars.list_empty[b], 4);  // producer, both issuers, softmax
            mbar_init(&bars.fin[b], 1);
        }
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_empty, 2);
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
    auto stage_ptr = [&](uint32_t e) { return sm + kOffRing + (e % kStages) * kKVBytes; };
    auto full_bar = [&](uint32_t e) { return &bars.kv_full[e % kStages]; };
    auto empty_bar = [&](uint32_t e) { return &bars.kv_empty[e % kStages]; };
    auto round_of = [](uint32_t e) { return (e / kStages) & 1u; };

    if (warp == 11) {
        // ---------------------------------------------------------------- union lists
        // Unit u+1's union list (double-buffered) is built while unit u is consumed: the 16
        // selection rows are staged with all loads in flight, then merged one lane per token.
        int32_t* stage = reinterpret_cast<int32_t*>(sm + kOffStage);
        int it = 0;
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            if (it >= 2 && !wait_or_abort(&bars.list_empty[lb], ((it - 2) >> 1) & 1, ctx, abort)) break;
            const int64_t bg = unit / units_per_seq;
            const int i0 = (unit % units_per_seq) * kUT;
            const int c = i0 / kBlk;
            const int n_act = min(kUT, N - i0);
            const int total = n_act * slots;
            const int32_t* src = idx + (bg * N + i0) * (int64_t)slots;
            {
                constexpr int kPer = kMaxList / 32;
                int32_t v[kPer];
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    const int e = lane + 32 * j;
                    v[j] = e < total ? __ldg(src + e) : -1;
                }
#pragma unroll
                for (int j = 0; j < kPer; ++j) {
                    const int e = lane + 32 * j;
                    if (e < total) stage[e] = v[j];
                }
            }
            __syncwarp();
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
            __syncwarp();
            if (lane == 0) {
                bars.list_n[lb] = n;
                mbar_arrive(&bars.list_full[lb]);
            }
            __syncwarp();
            if (*abort) break;
        }
    } else if (warp == 8) {
        // ---------------------------------------------------------------- producer
        int it = 0;
        uint32_t rc = 0, kq = 0;
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            int stop = 0;
            if (lane == 0) {
                if (!wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort)) stop = 1;
                const int n = stop ? 0 : bars.list_n[lb];
                const int64_t bg = unit / units_per_seq;
                const int i0 = (unit % units_per_seq) * kUT;
                if (n > 0) {
                    if (kq >= 1 && !wait_or_abort(&bars.q_empty, (kq - 1) & 1, ctx, abort)) stop = 1;
                    if (!stop) {
                        const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
                        mbar_arrive_expect_tx(&bars.q_full, 4 * kTileBytes);
                        for (int q = 0; q < 2; ++q) {
                            uint8_t* dq_ = sm + q * kTileBytes;
                            uint8_t* dd = sm + kOffDO + q * kTileBytes;
                            tma_load_3d(dq_, &tmQ, &bars.q_full, 0, i0 + q * kTQ, z);
                            tma_load_3d(dq_ + kHalfQ, &tmQ, &bars.q_full, 64, i0 + q * kTQ, z);
                            tma_load_3d(dd, &tmDO, &bars.q_full, 0, i0 + q * kTQ, z);
                            tma_load_3d(dd + kHalfQ, &tmDO, &bars.q_full, 64, i0 + q * kTQ, z);
                        }
                        ++kq;
                    }
                    for (int e = 0; e < n && !stop; ++e, ++rc) {
                        if (rc >= kStages && !wait_or_abort(empty_bar(rc), round_of(rc - kStages), ctx, abort)) {
                            stop = 1;
                            break;
                        }
                        uint8_t* st = stage_ptr(rc);
                        uint64_t* fb = full_bar(rc);
                        mbar_arrive_expect_tx(fb, kKVBytes);
                        const int y = list_id(lb)[e] * kBlk;
                        tma_load_3d(st, &tmK, fb, 0, y, (int)bg);
                        tma_load_3d(st + kHalfBlk, &tmK, fb, 64, y, (int)bg);
                        tma_load_3d(st + 2 * kHalfBlk, &tmV, fb, 0, y, (int)bg);
                        tma_load_3d(st + 3 * kHalfBlk, &tmV, fb, 64, y, (int)bg);
                    }
                }
                if (!stop) mbar_arrive(&bars.list_empty[lb]);
            }
            rc = __shfl_sync(0xffffffffu, rc, 0);
            kq = __shfl_sync(0xffffffffu, kq, 0);
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop || *abort) break;
        }
        if (lane == 0) {  // every copy this warp started has landed before the block exits
            if (kq > 0) (void)mbar_wait(&bars.q_full, (kq - 1) & 1, ctx);
            for (uint32_t e = rc > kStages ? rc - kStages : 0; e < rc; ++e)
                (void)mbar_wait(full_bar(e), round_of(e), ctx);
        }
    } else if (warp == 9 || warp == 10) {
        // ---------------------------------------------------------------- MMA issuers
        // Warp 9 issues tile A's MMAs, warp 10 tile B's (one thread each).  Per active block:
        // S and dP, then, once the tile's softmax has written dS, dQ += dS K and the stage goes
        // back; a block the tile did not choose goes back at once.  An issuer holds no stage
        // while it waits for another, and its S of the next block is issued after the dQ that
        // reads this block's dS from the same TMEM columns (MMAs of one thread run in order).
        const int x = warp - 9;
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, kBlk, false, false);
            const uint32_t idDQ = idesc_bf16_f32(128, kD, false, true);
            const uint32_t tDQ = tmem + x * 128;
            const uint32_t tS = tmem + kColS + x * 128, tP = tS + 64;
            const uint32_t dhi = sdesc_sw128_hi(1024);
            const uint32_t q_lo = sdesc_sw128_lo(smem_u32(sm + x * kTileBytes), 16);
            const uint32_t do_lo = sdesc_sw128_lo(smem_u32(sm + kOffDO + x * kTileBytes), 16);
            const uint32_t k_lo = sdesc_sw128_lo(smem_u32(sm + kOffRing), 16);
            const uint32_t v_lo = sdesc_sw128_lo(smem_u32(sm + kOffRing + 2 * kHalfBlk), 16);
            const uint32_t kmn_lo = sdesc_sw128_lo(smem_u32(sm + kOffRing), kHalfBlk);
            int it = 0;
            uint32_t rc = 0, kq = 0, a = 0;
            bool ok = true;
            for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++it) {
                const int lb = it & 1;
                ok = wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort);
                if (!ok) break;
                const int n = bars.list_n[lb];
                if (n > 0) {
                    ok = wait_or_abort(&bars.q_full, kq & 1, ctx, abort);
                    ++kq;
                    tc_fence_after();
                    bool accum = false;
                    for (int b = 0; b < n && ok; ++b) {
                        const uint32_t e = rc + b;
                        const bool act = ((list_mask(lb)[b] >> (8 * x)) & 0xffu) != 0;
                        if (!(ok = wait_or_abort(full_bar(e), round_of(e), ctx, abort))) break;
                        if (!act) {
                            mbar_arrive(empty_bar(e));
                            continue;
                        }
                        tc_fence_after();
                        const uint32_t so = (e % kStages) * (kKVBytes >> 4);
#pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks) {
                            const uint32_t ao = ((ks >> 2) * kHalfQ + (ks & 3) * 32) >> 4;
                            const uint32_t bo = so + (((ks >> 2) * kHalfBlk + (ks & 3) * 32) >> 4);
                            mma_ss_lohi(tS, q_lo + ao, k_lo + bo, dhi, idS, ks > 0 ? 1u : 0u);
                        }
#pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks) {
                            const uint32_t ao = ((ks >> 2) * kHalfQ + (ks & 3) * 32) >> 4;
                            const uint32_t bo = so + (((ks >> 2) * kHalfBlk + (ks & 3) * 32) >> 4);
                            mma_ss_lohi(tP, do_lo + ao, v_lo + bo, dhi, idS, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(&bars.s_full[x]);
                        if (!(ok = wait_or_abort(&bars.p_full[x], a & 1u, ctx, abort))) break;
                        {
                            tc_fence_after();
#pragma unroll
                            for (int ks = 0; ks < kBlk / 16; ++ks)
                                mma_ts_lohi(tDQ, tS + ks * 8, kmn_lo + so + ((ks * 16 * 128) >> 4),
                                            dhi, idDQ, (accum || ks > 0) ? 1u : 0u);
#pragma unroll
                            for (int ks = 0; ks < kBlk / 16; ++ks)  // the residual term, over dP_X
                                mma_ts_lohi(tDQ, tP + ks * 8, kmn_lo + so + ((ks * 16 * 128) >> 4),
                                            dhi, idDQ, 1u);
                            mma_commit(&bars.dq_done[x]);
                            accum = true;
                        }
                        mma_commit(empty_bar(e));
                        ++a;
                    }
                    mma_commit(&bars.q_empty);
                    rc += n;
                }
                mbar_arrive(&bars.list_empty[lb]);
            }
            mma_commit(&bars.fin[x]);
            (void)mbar_wait(&bars.fin[x], 0, ctx);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- dS + epilogue
        // Warpgroup x (0: tile A, 1: tile B); thread = row r of the tile = TMEM lane r.  The
        // warpgroups meet once per unit at a named barrier; a failed wait is recorded in sm_stop
        // and all leave together after the barrier it names, as in the forward.
        const int x = warp >> 2;
        const int r = tid & 127;
        const int t = x * kTQ + r % kTQ, hh = r / kTQ;
        const uint32_t lane_base = tmem_lane_base(warp);
        const uint32_t colDQ = tmem + lane_base + x * 128;
        const uint32_t colS = tmem + lane_base + kColS + x * 128, colP = colS + 64;
        volatile int* sm_stop = &bars.sm_stop;
        int nbar = 0;
        bool dead = false;
        auto fail = [&]() {
            dead = true;
            atomicCAS(&bars.sm_stop, 0, nbar + 1);
            *abort = 1;
        };
        int it = 0;
        uint32_t a = 0, ndq = 0;  // S rounds of this tile; dQ rounds before this unit
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!dead && !mbar_wait(&bars.list_full[lb], (it >> 1) & 1, ctx)) fail();
            const int n = dead ? 0 : bars.list_n[lb];
            const int32_t* ids = list_id(lb);
            const uint16_t* msks = list_mask(lb);
            const int64_t bg = unit / units_per_seq;
            const int i0 = (unit % units_per_seq) * kUT;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            const int64_t row = ((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i;
            const float nl = i < N ? -__ldg(lse + row) * kLog2e : 0.f;
            const float dv = i < N ? __ldg(delta + row) : 0.f;
            int last = -1;  // the tile's last dQ round (its dq_done phase)
            for (int b = 0; b < n; ++b) {
                const unsigned msk = msks[b];
                if (((msk >> (8 * x)) & 0xffu) == 0) continue;
                const int blk = ids[b];
                const bool sel = (msk >> t) & 1u;
                const int lim = (!sel || i >= N) ? -1 : (blk == c ? i - blk * kBlk : kBlk - 1);
                if (!dead && !mbar_wait(&bars.s_full[x], a & 1u, ctx)) fail();
                tc_fence_after();
                if (!__any_sync(0xffffffffu, dead)) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t sr[32], pr[32], hi[16], lo[16];
                        tmem_ld32(colS + 32 * h, sr);
                        tmem_ld32(colP + 32 * h, pr);
                        tmem_ld_wait();
                        ds_half(sr, pr, 32 * h, lim, sl2, nl, dv, hi, lo);
                        tmem_st16(colS + 16 * h, hi);  // columns already read
                        tmem_st16(colP + 16 * h, lo);
                    }
                }
                tmem_st_wait();
                ++last;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[x]);
                ++a;
            }
            last = last >= 0 ? (int)(ndq + last) : -1;
            ndq = last >= 0 ? (uint32_t)last + 1 : ndq;
            // Epilogue: scale * dQ_x -> bf16 -> global (zeros when the tile saw no block).
            if (last >= 0) {
                if (!dead && !mbar_wait(&bars.dq_done[x], (uint32_t)last & 1u, ctx)) fail();  // last dQ round
                if (!__any_sync(0xffffffffu, dead)) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < kD; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(colDQ + c0, v);
                        tmem_ld_wait();
                        if (i < N) {
                            uint4 w[4];
                            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                wp[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * scale,
                                                    __uint_as_float(v[2 * q + 1]) * scale);
                            uint4* d4 = reinterpret_cast<uint4*>(dq + row * kD + c0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) d4[q] = w[q];
                        }
                    }
                    tc_fence_before();
                }
            } else if (i < N && !dead) {
                uint4* d4 = reinterpret_cast<uint4*>(dq + row * kD);
                for (int q = 0; q < kD / 8; ++q) d4[q] = make_uint4(0, 0, 0, 0);
            }
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

// ================================================================================== dk / dv pass
namespace dkvp {

// warps 0-7 dS (two per row: keys 0-31 and 32-63), 8-11 epilogue, 12 producer, 13 S|dP issuer
// (and TMEM owner), 14 dV issuer, 15 dK issuer
constexpr int kThreads = 512;
constexpr int kTok = 8;        // tokens per tile (x 16 heads = 128 rows)
constexpr int kRingBytes = 2 * kTileBytes;          // Q tile then dO tile
constexpr int kOffRing = kKVBytes;                  // after the K|V buffer
constexpr int kOffP = kOffRing + 2 * kRingBytes;    // two buffers of P [128 rows x 128 B] + dS
constexpr int kPBytes = 16384;
constexpr int kSmemBytes = kOffP + 4 * kPBytes + 1024;
static_assert(kSmemBytes <= 232448 - 512, "shared memory");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 256;  // dK^T at kColAcc + 128 w, dV^T at +64; S_u at 128 u, dP_u +64

struct Bars {
    uint64_t kv_full, kv_empty;
    uint64_t ring_full[2], ring_empty[2];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full[2], pds_free[2];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t fin[3];
    uint32_t tmem_base;
    int abort;
};

// The CTA's work: items of kItem consecutive positions of the concatenated token lists, taken
// in turn (item blockIdx.x, + gridDim.x, ...) so that all CTAs move through the lists together,
// one chunk of query tokens at a time; within an item, segment by segment: key = the list
// ((b * Hkv + g) * n_chunks + chunk) * nb + j, [p0, p1) its part inside the item.  Every role
// walks it alike.
struct WalkCtx {
    const int* off;
    const int* item_key;
    int64_t T;
    int stride;
};
struct Walk {
    int item;
    int key;
    int64_t t1, p0, p1;
    __device__ bool enter(const WalkCtx& c) {
        const int64_t t0 = (int64_t)item * kItem;
        if (t0 >= c.T) return false;
        t1 = min(c.T, t0 + kItem);
        key = __ldg(c.item_key + item);
        p0 = t0;
        p1 = min((int64_t)__ldg(c.off + key + 1), t1);
        return true;
    }
    __device__ bool start(const WalkCtx& c, int first) {
        item = first;
        return enter(c);
    }
    __device__ bool next(const WalkCtx& c) {
        if (p1 < t1) {
            p0 = p1;
            do {
                ++key;
            } while (__ldg(c.off + key + 1) <= p0);
            p1 = min((int64_t)__ldg(c.off + key + 1), t1);
            return true;
        }
        item += c.stride;
        return enter(c);
    }
};

// A tile cursor over the same walk: tile = up to kTok consecutive list positions of one segment.
struct Cursor {
    Walk w;
    int64_t pos;
    bool ok;
    __device__ void start(const WalkCtx& c, int first) {
        ok = w.start(c, first);
        pos = w.p0;
    }
    __device__ int n() const { return (int)min((int64_t)kTok, w.p1 - pos); }
    __device__ void advance(const WalkCtx& c) {
        pos += kTok;
        if (pos >= w.p1) {
            ok = ok && w.next(c);
            pos = w.p0;
        }
    }
};

}  // namespace dkvp

__global__ void __launch_bounds__(dkvp::kThreads, 1)
sparse_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const int* __restrict__ off, const int* __restrict__ item_key,
                     const int* __restrict__ list,
                     const float* __restrict__ lse, const float* __restrict__ delta,
                     float* __restrict__ dk_acc, float* __restrict__ dv_acc, int H, int Hkv, int N,
                     int nb, int n_chunks, int n_keys, float sl2, DevCtx ctx) {
    using namespace dkvp;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &bars.abort;

    if (warp == 13) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.kv_full, 1);
        mbar_init(&bars.kv_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.p_full[b], 8);       // eight dS warps
            mbar_init(&bars.pds_free[b], 2);     // the dV and dK issuers
            mbar_init(&bars.ring_full[b], 1);
            mbar_init(&bars.ring_empty[b], 3);   // all three issuers read a tile
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.s_free[b], 8);
            mbar_init(&bars.acc_full[b], 2);     // dK and dV of a segment
            mbar_init(&bars.acc_empty[b], 4);
        }
        for (int b = 0; b < 3; ++b) mbar_init(&bars.fin[b], 1);
        bars.abort = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    const WalkCtx wc{off, item_key, (int64_t)__ldg(off + n_keys), (int)gridDim.x};
    auto ring = [&](uint32_t t) { return sm + kOffRing + (t & 1) * kRingBytes; };
    auto kvbuf = [&](uint32_t) { return sm; };
    auto sP = [&](uint32_t t) { return sm + kOffP + (t & 1) * 2 * kPBytes; };
    auto sDS = [&](uint32_t t) { return sm + kOffP + (t & 1) * 2 * kPBytes + kPBytes; };
    Walk wk;

    if (warp == 12) {
        // ---------------------------------------------------------------- producer
        // Per segment its K and V (once the buffer's segment two back is done), then per tile the
        // Q and dO rows of its tokens: lane u < 8 gathers token u (a short last tile repeats its
        // last token; those rows are masked), 16 heads x 128 B per box.
        uint32_t seg = 0, t = 0, kv_iss = 0;  // segments walked, tiles and K|V pairs issued
        bool stop = false;
        int tok_next = 0;
        bool have_next = false;
        for (bool more = wk.start(wc, blockIdx.x); more && !stop; more = wk.next(wc), ++seg) {
            const int64_t bg = wk.key / (nb * n_chunks);
            const int j = wk.key % nb;
            const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
            if (lane == 0) {
                if (seg >= 1 && !wait_or_abort(&bars.kv_empty, (seg - 1) & 1, ctx, abort))
                    stop = true;
                if (!stop) {
                    uint8_t* kv = kvbuf(seg);
                    uint64_t* fb = &bars.kv_full;
                    mbar_arrive_expect_tx(fb, kKVBytes);
                    tma_load_3d(kv, &tmK, fb, 0, j * kBlk, (int)bg);
                    tma_load_3d(kv + kHalfBlk, &tmK, fb, 64, j * kBlk, (int)bg);
                    tma_load_3d(kv + 2 * kHalfBlk, &tmV, fb, 0, j * kBlk, (int)bg);
                    tma_load_3d(kv + 3 * kHalfBlk, &tmV, fb, 64, j * kBlk, (int)bg);
                    ++kv_iss;
                }
            }
            stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
            for (int64_t pos = wk.p0; pos < wk.p1 && !stop; pos += kTok, ++t) {
                const int n = (int)min((int64_t)kTok, wk.p1 - pos);
                // this tile's tokens came one tile ahead when it is not an item's first (positions
                // pos .. pos + 7, clamped to the item); a short tile repeats its last token
                const int raw = !have_next ? (lane < kTok ? __ldg(list + min(pos + lane, wk.t1 - 1)) : 0)
                                           : tok_next;
                const int tok = __shfl_sync(0xffffffffu, raw, min(lane, n - 1));
                have_next = pos + n < wk.t1;
                tok_next = (lane < kTok && have_next) ? __ldg(list + min(pos + n + lane, wk.t1 - 1)) : 0;
                if (lane == 0) {
                    if (t >= 2 && !wait_or_abort(&bars.ring_empty[t & 1], ((t - 2) >> 1) & 1, ctx, abort))
                        stop = true;
                    if (!stop) mbar_arrive_expect_tx(&bars.ring_full[t & 1], kRingBytes);
                }
                stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
                if (stop) break;
                if (lane < kTok) {
                    uint8_t* dst = ring(t) + lane * 2048;
                    uint64_t* fb = &bars.ring_full[t & 1];
                    tma_load_3d(dst, &tmQ, fb, 0, tok, z);
                    tma_load_3d(dst + kHalfQ, &tmQ, fb, 64, tok, z);
                    tma_load_3d(dst + kTileBytes, &tmDO, fb, 0, tok, z);
                    tma_load_3d(dst + kTileBytes + kHalfQ, &tmDO, fb, 64, tok, z);
                }
                __syncwarp();
            }
            if (*abort) stop = true;
        }
        if (lane == 0) {  // every copy this warp started has landed before the block exits
            if (kv_iss > 0) (void)mbar_wait(&bars.kv_full, (kv_iss - 1) & 1, ctx);
            for (uint32_t e = t > 2 ? t - 2 : 0; e < t; ++e)
                (void)mbar_wait(&bars.ring_full[e & 1], (e >> 1) & 1, ctx);
        }
    } else if (warp == 13) {
        // ---------------------------------------------------------------- S | dP issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, kBlk, false, false);
            const uint32_t dhi = sdesc_sw128_hi(1024);
            uint32_t seg = 0, t = 0;
            bool ok = true;
            for (bool more = wk.start(wc, blockIdx.x); more && ok; more = wk.next(wc), ++seg) {
                if (!(ok = wait_or_abort(&bars.kv_full, seg & 1, ctx, abort))) break;
                const uint32_t k_lo = sdesc_sw128_lo(smem_u32(kvbuf(seg)), 16);
                const uint32_t v_lo = sdesc_sw128_lo(smem_u32(kvbuf(seg) + 2 * kHalfBlk), 16);
                for (int64_t pos = wk.p0; pos < wk.p1; pos += kTok, ++t) {
                    const uint32_t u = t & 1;
                    if (!(ok = wait_or_abort(&bars.ring_full[u], (t >> 1) & 1, ctx, abort))) break;
                    if (t >= 2 && !(ok = wait_or_abort(&bars.s_free[u], ((t - 2) >> 1) & 1, ctx, abort))) break;
                    tc_fence_after();
                    const uint32_t q_lo = sdesc_sw128_lo(smem_u32(ring(t)), 16);
                    const uint32_t do_lo = sdesc_sw128_lo(smem_u32(ring(t) + kTileBytes), 16);
                    const uint32_t tS = tmem + u * 128, tP = tS + 64;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t ao = ((ks >> 2) * kHalfQ + (ks & 3) * 32) >> 4;
                        const uint32_t bo = ((ks >> 2) * kHalfBlk + (ks & 3) * 32) >> 4;
                        mma_ss_lohi(tS, q_lo + ao, k_lo + bo, dhi, idS, ks > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t ao = ((ks >> 2) * kHalfQ + (ks & 3) * 32) >> 4;
                        const uint32_t bo = ((ks >> 2) * kHalfBlk + (ks & 3) * 32) >> 4;
                        mma_ss_lohi(tP, do_lo + ao, v_lo + bo, dhi, idS, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(&bars.s_full[u]);
                    mma_commit(&bars.ring_empty[u]);
                    if (pos + kTok >= wk.p1) mma_commit(&bars.kv_empty);
                }
            }
            mma_commit(&bars.fin[0]);
            (void)mbar_wait(&bars.fin[0], 0, ctx);
        }
        __syncwarp();
    } else if (warp == 14 || warp == 15) {
        // ---------------------------------------------------------------- dV, dK issuers
        // Warp 14: dV^T += dO^T P; warp 15: dK^T += Q^T dS (one thread each, separate TMEM
        // accumulators).  A is the tile read M-major (d contiguous, the two 64-column halves
        // 16 KiB apart), B the P / dS rows read N-major; K runs over the 128 rows in steps of 16
        // (2 KiB).
        const bool isV = warp == 14;
        if (lane == 0) {
            const uint32_t idD = idesc_bf16_f32(128, kBlk, true, true);
            const uint32_t dhi = sdesc_sw128_hi(1024);

            uint32_t seg = 0, t = 0;
            bool ok = true;
            for (bool more = wk.start(wc, blockIdx.x); more && ok; more = wk.next(wc), ++seg) {
                const uint32_t w = seg & 1;
                const uint32_t tK = tmem + kColAcc + w * 128, tV = tK + 64;
                for (int64_t pos = wk.p0; pos < wk.p1; pos += kTok, ++t) {
                    const uint32_t u = t & 1;
                    const bool first = pos == wk.p0;
                    if (!(ok = wait_or_abort(&bars.ring_full[u], (t >> 1) & 1, ctx, abort))) break;
                    if (!(ok = wait_or_abort(&bars.p_full[u], (t >> 1) & 1, ctx, abort))) break;
                    if (first && seg >= 2 &&
                        !(ok = wait_or_abort(&bars.acc_empty[w], ((seg - 2) >> 1) & 1, ctx, abort)))
                        break;
                    tc_fence_after();
                    const uint32_t q_lo = sdesc_sw128_lo(smem_u32(ring(t)), kHalfQ);
                    const uint32_t do_lo = sdesc_sw128_lo(smem_u32(ring(t) + kTileBytes), kHalfQ);
                    const uint32_t p_lo = sdesc_sw128_lo(smem_u32(sP(t)), kHalfQ);
                    const uint32_t ds_lo = sdesc_sw128_lo(smem_u32(sDS(t)), kHalfQ);
                    const uint32_t tD = isV ? tV : tK;
                    const uint32_t a_lo = isV ? do_lo : q_lo, b_lo = isV ? p_lo : ds_lo;
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {
                        const uint32_t o = (ks * 16 * 128) >> 4;
                        mma_ss_lohi(tD, a_lo + o, b_lo + o, dhi, idD, (first && ks == 0) ? 0u : 1u);
                    }
                    mma_commit(&bars.pds_free[u]);
                    mma_commit(&bars.ring_empty[u]);
                    if (pos + kTok >= wk.p1) mma_commit(&bars.acc_full[w]);
                }
            }
            mma_commit(&bars.fin[isV ? 1 : 2]);
            (void)mbar_wait(&bars.fin[isV ? 1 : 2], 0, ctx);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ---------------------------------------------------------------- P and dS rows
        // Thread = tile row r = TMEM lane r (token slot r / 16, head r % 16), keys 32 kh ..
        // 32 kh + 31 of it: warps 0-3 take the first half of every row, warps 4-7 the second.  P and dS go to
        // shared memory as 128-byte rows with the 128-byte swizzle (16-byte chunk c of row r at
        // chunk c ^ (r & 7)), the layout the dK | dV issuer's descriptors read.
        // The row's token, lse and D are global loads, the latter two dependent on the first:
        // tokens are fetched two tiles ahead and lse, D one tile ahead of their use.
        const int r = tid & 127, slot = r >> 4, hh = r & 15, kh = warp >> 2;
        const uint32_t lane_base = tmem_lane_base(warp);
        auto row_of = [&](const Cursor& c) {
            const int64_t bg = c.w.key / (nb * n_chunks);
            return ((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N;
        };
        auto tok_at = [&](const Cursor& c) {
            return (c.ok && slot < c.n()) ? __ldg(list + c.pos + slot) : -1;
        };
        // the tile after c1 starts at c1.pos + c1.n() when that is inside c1's item; its token
        // is fetched from there and kept if that tile turns out to start there
        auto pos_after = [&](const Cursor& c) { return c.ok ? c.pos + c.n() : (int64_t)-1; };
        auto tok_ahead = [&](const Cursor& c) {
            const int64_t p = pos_after(c);
            return (p >= 0 && p + slot < c.w.t1) ? __ldg(list + p + slot) : -1;
        };
        Cursor cur, c1;
        cur.start(wc, blockIdx.x);
        c1 = cur;
        c1.advance(wc);
        int tok0 = tok_at(cur), tok1 = tok_at(c1);
        float nl0 = 0.f, dv0 = 0.f;
        if (tok0 >= 0) {
            nl0 = -__ldg(lse + row_of(cur) + tok0) * kLog2e;
            dv0 = __ldg(delta + row_of(cur) + tok0);
        }
        uint32_t t = 0;
        bool ok = true;
        for (; cur.ok && ok; ++t) {
            float nl1 = 0.f, dv1 = 0.f;
            if (tok1 >= 0) {
                const int64_t r1 = row_of(c1) + tok1;
                nl1 = -__ldg(lse + r1) * kLog2e;
                dv1 = __ldg(delta + r1);
            }
            const int64_t p2 = pos_after(c1);
            const int tok2 = tok_ahead(c1);
            {
                const int j = cur.w.key % nb;
                const uint32_t u = t & 1;
                const float nl = nl0, dv = dv0;
                const int lim = tok0 >= 0 ? min(kBlk - 1, tok0 - j * kBlk) : -1;
                if (!(ok = wait_or_abort(&bars.s_full[u], (t >> 1) & 1, ctx, abort))) break;
                // the dK | dV MMAs of the tile two back are done with this P | dS buffer
                if (t >= 2 && !(ok = wait_or_abort(&bars.pds_free[u], ((t - 2) >> 1) & 1, ctx, abort))) break;
                tc_fence_after();
                uint4* prow = reinterpret_cast<uint4*>(sP(t) + r * 128);
                uint4* srow = reinterpret_cast<uint4*>(sDS(t) + r * 128);
                {
                    const int h = kh;
                    uint32_t sr[32], pr[32], pkP[16], pkS[16];
                    tmem_ld32(tmem + lane_base + u * 128 + 32 * h, sr);
                    tmem_ld32(tmem + lane_base + u * 128 + 64 + 32 * h, pr);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int k = 32 * h + 2 * q;
                        const float p0 = k <= lim ? ex2(fmaf(__uint_as_float(sr[2 * q]), sl2, nl)) : 0.f;
                        const float p1 = k + 1 <= lim ? ex2(fmaf(__uint_as_float(sr[2 * q + 1]), sl2, nl)) : 0.f;
                        pkP[q] = pack_bf16x2(p0, p1);
                        pkS[q] = pack_bf16x2(p0 * (__uint_as_float(pr[2 * q]) - dv),
                                             p1 * (__uint_as_float(pr[2 * q + 1]) - dv));
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int cc = (4 * h + c) ^ (r & 7);
                        prow[cc] = make_uint4(pkP[4 * c], pkP[4 * c + 1], pkP[4 * c + 2], pkP[4 * c + 3]);
                        srow[cc] = make_uint4(pkS[4 * c], pkS[4 * c + 1], pkS[4 * c + 2], pkS[4 * c + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.s_free[u]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[u]);
            }
            cur = c1;
            c1.advance(wc);
            tok0 = tok1;
            tok1 = (c1.ok && c1.pos == p2) ? (slot < c1.n() ? tok2 : -1) : tok_at(c1);
            nl0 = nl1;
            dv0 = dv1;
        }
    } else if (warp < 12) {
        // ---------------------------------------------------------------- epilogue
        // Thread = TMEM lane = column d of dK_b^T / dV_b^T; key by key, a warp adds 32
        // consecutive floats (128 bytes) of one key row into the fp32 accumulators.
        const int d = tid - 256;
        const uint32_t lane_base = tmem_lane_base(warp);
        uint32_t seg = 0;
        bool ok = true;
        for (bool more = wk.start(wc, blockIdx.x); more && ok; more = wk.next(wc), ++seg) {
            const int64_t bg = wk.key / (nb * n_chunks);
            const int j = wk.key % nb;
            const uint32_t w = seg & 1;
            if (!(ok = wait_or_abort(&bars.acc_full[w], (seg >> 1) & 1, ctx, abort))) break;
            tc_fence_after();
            const int nk = min(kBlk, N - j * kBlk);
            float* dkp = dk_acc + (bg * N + (int64_t)j * kBlk) * kD + d;
            float* dvp = dv_acc + (bg * N + (int64_t)j * kBlk) * kD + d;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                const uint32_t col = tmem + lane_base + kColAcc + w * 128 + (c >> 1) * 64 + (c & 1) * 32;
                tmem_ld32(col, v);
                tmem_ld_wait();
                float* dst = (c < 2 ? dkp : dvp) + (int64_t)((c & 1) * 32) * kD;
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    if ((c & 1) * 32 + q < nk) atomicAdd(dst + (int64_t)q * kD, __uint_as_float(v[q]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.acc_empty[w]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// 3-D tensor map over [planes][rows][128] bf16 with a {64, box_rows, box_planes} box, 128-byte
// swizzle.
bool make_map(EncodeTiledFn fn, CUtensorMap* m, const void* base, uint64_t rows, uint64_t planes,
              uint32_t box_rows, uint32_t box_planes) {
    cuuint64_t dims[3] = {(cuuint64_t)kD, rows, planes};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * rows};
    cuuint32_t box[3] = {64, box_rows, box_planes};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() { return device_sm_count(); }

}  // namespace

cudaError_t launch_sparse_dq_tc(const void* q, const void* k, const void* v, const void* dout,
                                const int32_t* idx, const float* lse, const float* delta, void* dq,
                                int B, int H, int Hkv, int N, int slots, float scale,
                                cudaStream_t st, DevCtx ctx) {
    if (H != Hkv * kG || slots > dqp::kMaxSlots) return cudaErrorNotSupported;
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tmQ, tmDO, tmK, tmV;
    if (!make_map(fn, &tmQ, q, (uint64_t)N, (uint64_t)B * H, dqp::kTQ, kG) ||
        !make_map(fn, &tmDO, dout, (uint64_t)N, (uint64_t)B * H, dqp::kTQ, kG) ||
        !make_map(fn, &tmK, k, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1) ||
        !make_map(fn, &tmV, v, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem<sparse_dq_tc_kernel>(dqp::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int units_per_seq = (N + dqp::kUT - 1) / dqp::kUT;
    const int n_units = units_per_seq * B * Hkv;
    const int grid = n_units < num_sms() ? n_units : num_sms();
    sparse_dq_tc_kernel<<<grid, dqp::kThreads, dqp::kSmemBytes, st>>>(
        tmQ, tmDO, tmK, tmV, idx, lse, delta, static_cast<__nv_bfloat16*>(dq), H, Hkv, N, slots,
        scale * kLog2e, scale, n_units, ctx);
    return cudaGetLastError();
}

cudaError_t launch_sparse_dkv_tc(const void* q, const void* k, const void* v, const void* dout,
                                 const float* lse, const float* delta, const SparseBwdCsr& c,
                                 float* dk_acc, float* dv_acc, int B, int H, int Hkv, int N,
                                 float scale, cudaStream_t st, DevCtx ctx) {
    if (H != Hkv * kG) return cudaErrorNotSupported;
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tmQ, tmDO, tmK, tmV;
    if (!make_map(fn, &tmQ, q, (uint64_t)N, (uint64_t)B * H, 1, kG) ||
        !make_map(fn, &tmDO, dout, (uint64_t)N, (uint64_t)B * H, 1, kG) ||
        !make_map(fn, &tmK, k, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1) ||
        !make_map(fn, &tmV, v, (uint64_t)N, (uint64_t)B * Hkv, kBlk, 1))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem<sparse_dkv_tc_kernel>(dkvp::kSmemBytes);
    if (e != cudaSuccess) return e;
    sparse_dkv_tc_kernel<<<num_sms(), dkvp::kThreads, dkvp::kSmemBytes, st>>>(
        tmQ, tmDO, tmK, tmV, c.off, c.item_key, c.list, lse, delta, dk_acc, dv_acc, H, Hkv, N, c.nb,
        c.n_chunks, c.n_keys, scale * kLog2e, ctx);
    return cudaGetLastError();
}

}  // namespace sala
