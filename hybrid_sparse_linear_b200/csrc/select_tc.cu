// Block selection on the 5th-generation tensor cores (sm_100a): scores of 128 query rows against
// 128 candidate blocks per MMA, exact per-row top-k with a provable floor.
//
// Tile: 128 consecutive query rows (two query blocks) of one (batch, KV group).  The group-summed
// query qbar_r = sum_{h in g} q_{h,r} is formed in fp32 and split into two bf16 terms
// hi = bf16(qbar), lo = bf16(qbar - hi), so score = hi.kbar + lo.kbar carries ~16 significant bits
// of qbar on bf16 tensor cores (kbar itself is bf16, exact).
//
// Floor: the pilot vector p = sum_r qbar_r ranks the candidates that every row of the tile may
// take; its top-k become seeds.  For a row r with at least k seeds, its k-th best key is at least
// the smallest key among its own k seed keys (k real candidates reach that key), so any candidate
// whose key is below that floor can never enter row r's top-k and is skipped.  The seeds only
// decide how much work is skipped, never the result: the selection is exact.
//
// Main pass, per 128-candidate tile: MMA (2 x 8 K-steps, N = 128) -> TMEM (double-buffered) ->
// warps 0-3 copy row r's 128 scores to shared memory -> warps 0-7 run the warp-level top-k of 16
// rows each (best 64 keys per row in registers, two per lane; only candidates above both the
// floor and the current k-th key are inserted).  Key = (orderable score, ~block), so ties go to
// the lower block index.  Output as the CUDA-core path: init ids, sorted top-k ids, local ids.
//
// Roles (320 threads): warps 0-7 workers, warp 8 TMA producer (kbar tiles), warp 9 TMEM owner and
// MMA issuer.  Every wait is bounded; the 8 workers leave their loops only together (see the
// sparse prefill kernel for the same named-barrier discipline).
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128, kRows = 128, kCand = 128, kBlk = 64, kCap = 64;
constexpr int kThreads = 320, kWorkers = 256;
constexpr int kSub = 128 * 128;                        // [128 rows x 128 B] = 16 KiB
constexpr int kOffAhi = 0, kOffAlo = 2 * kSub;         // A operands (hi, lo), 2 sub-tiles each
constexpr int kOffKb = 4 * kSub;                       // kbar tiles, 2 stages x 2 sub-tiles
constexpr int kOffSeedB = 8 * kSub;                    // seed kbar rows [64 x 128 d], 2 sub-tiles of 8 KiB
constexpr int kSCStride = kCand + 4;                   // floats per row of the score tile
constexpr int kOffSC = kOffSeedB + 2 * 8192;
constexpr int kOffPList = kOffSC + kRows * kSCStride * 4;  // 8 warp lists x 64 keys
constexpr int kSmemBytes = kOffPList + 8 * kCap * 8 + 1024;

constexpr uint32_t kColS0 = 0, kColSeed = 256, kTmemCols = 512;

struct Bars {
    uint64_t a_ready, seed_ready, seed_done;
    uint64_t kv_full[2], kv_empty[2], s_full[2], s_free[2];
    uint64_t fin;
    uint32_t tmem_base;
    int abort;
    int sm_stop;
    float pilot[kD];
    float ppart[8][kD];
    uint64_t floor_key[kRows];
    int seeds[kCap];
    int n_seeds;
};

__device__ __forceinline__ uint64_t shfl64(uint64_t x, int src) { return __shfl_sync(0xffffffffu, x, src); }

__device__ __forceinline__ uint64_t kth_key(uint64_t l0, uint64_t l1, int K) {
    return shfl64(((K - 1) & 1) ? l1 : l0, (K - 1) >> 1);
}

// Offer one key per lane to the warp's descending list (keeps the best K <= 64); keys at or below
// `floor` are dropped.
__device__ __forceinline__ void offer(uint64_t& l0, uint64_t& l1, uint64_t key, uint64_t floor,
                                      int K, int lane) {
    uint64_t thr = kth_key(l0, l1, K);
    if (floor > thr) thr = floor - 1;  // a key equal to the floor may still enter
    bool take = key > thr;
    unsigned m = __ballot_sync(0xffffffffu, take);
    while (m) {
        const int src = __ffs(m) - 1;
        const uint64_t kn = shfl64(key, src);
        const int p = __popc(__ballot_sync(0xffffffffu, l0 > kn)) + __popc(__ballot_sync(0xffffffffu, l1 > kn));
        const uint64_t prev1 = __shfl_up_sync(0xffffffffu, l1, 1);
        const int q0 = 2 * lane, q1 = 2 * lane + 1;
        const uint64_t n0 = q0 < p ? l0 : (q0 == p ? kn : prev1);
        const uint64_t n1 = q1 < p ? l1 : (q1 == p ? kn : l0);
        l0 = n0;
        l1 = n1;
        if (lane == src) take = false;
        thr = kth_key(l0, l1, K);
        if (floor > thr) thr = floor - 1;
        m = __ballot_sync(0xffffffffu, take && key > thr);
    }
}

// Top-64 (descending) of two descending 64-key lists held two per lane: elementwise max against
// the reversed second list gives a bitonic sequence holding the top half, then a bitonic clean.
__device__ __forceinline__ void merge_desc(uint64_t& a0, uint64_t& a1, uint64_t b0, uint64_t b1, int lane) {
    const uint64_t r0 = shfl64(b1, 31 - lane), r1 = shfl64(b0, 31 - lane);  // reversed B
    a0 = a0 > r0 ? a0 : r0;
    a1 = a1 > r1 ? a1 : r1;
#pragma unroll
    for (int s = 32; s >= 2; s >>= 1) {
        const int lm = s >> 1;
        const uint64_t y0 = shfl64(a0, lane ^ lm), y1 = shfl64(a1, lane ^ lm);
        const bool low = (lane & lm) == 0;  // this lane holds the lower position of the pair
        a0 = low ? (a0 > y0 ? a0 : y0) : (a0 < y0 ? a0 : y0);
        a1 = low ? (a1 > y1 ? a1 : y1) : (a1 < y1 ? a1 : y1);
    }
    const uint64_t hi = a0 > a1 ? a0 : a1, lo = a0 > a1 ? a1 : a0;
    a0 = hi;
    a1 = lo;
}

// Ascending bitonic sort of 64 ints held two per lane.
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

__global__ void __launch_bounds__(kThreads, 1)
topk_tc_kernel(const __grid_constant__ CUtensorMap tmKb, const __nv_bfloat16* __restrict__ q,
               const __nv_bfloat16* __restrict__ kbar, int32_t* __restrict__ idx, int H, int Hkv,
               int Nq, int nb, int topk, int n_init, int n_local, int slots, DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = H / Hkv;
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    const int r0 = blockIdx.x * kRows;
    const int nrows = min(kRows, Nq - r0);
    const int K = min(topk, kCap);
    // Candidate ranges: rows of the first query block of the tile (c0) and of the second (c0+1).
    const int c0 = r0 / kBlk;
    const int c_last = (r0 + nrows - 1) / kBlk;
    const int lo = n_init;
    const int hi_all = c0 - n_local;        // valid for every row of the tile
    const int hi = c_last - n_local;        // largest candidate of the tile
    const int ncand_all = hi_all - lo + 1;
    const bool rank = (hi - lo + 1) > topk && K > 0;  // some row has more candidates than k
    const int n_tiles = rank ? (hi - lo + kCand) / kCand : 0;
    volatile int* abort = &bars.abort;

    if (warp == 9) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.a_ready, 8);
        mbar_init(&bars.seed_ready, 8);
        mbar_init(&bars.seed_done, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.s_free[s], 4);
        }
        mbar_init(&bars.fin, 1);
        bars.abort = 0;
        bars.sm_stop = 0;
        bars.n_seeds = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0 && n_tiles > 0) {
            int issued0 = -1, issued1 = -1;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t & 1, r = t >> 1;
                if (r >= 1 && !mbar_wait(&bars.kv_empty[s], (r - 1) & 1, ctx)) { *abort = 1; break; }
                uint8_t* st = sm + kOffKb + s * 2 * kSub;
                mbar_arrive_expect_tx(&bars.kv_full[s], 2 * kSub);
                const int y = lo + t * kCand;
                tma_load_3d(st, &tmKb, &bars.kv_full[s], 0, y, (int)bg);
                tma_load_3d(st + kSub, &tmKb, &bars.kv_full[s], 64, y, (int)bg);
                if (s == 0) issued0 = r; else issued1 = r;
            }
            if (issued0 >= 0) (void)mbar_wait(&bars.kv_full[0], issued0 & 1, ctx);
            if (issued1 >= 0) (void)mbar_wait(&bars.kv_full[1], issued1 & 1, ctx);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            const uint32_t ahi = smem_u32(sm + kOffAhi), alo = smem_u32(sm + kOffAlo);
            bool ok = mbar_wait(&bars.a_ready, 0, ctx);
            // Seed scores: [128 rows] x [64 seeds], only when the floor is used.
            if (ok) ok = mbar_wait(&bars.seed_ready, 0, ctx);
            if (ok && bars.n_seeds == K) {
                tc_fence_after();
                const uint32_t sb = smem_u32(sm + kOffSeedB);
                const uint32_t id64 = idesc_bf16_f32(128, 64, false, false);
                for (int part = 0; part < 2; ++part) {
                    const uint32_t a = part ? alo : ahi;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_ss(tmem + kColSeed, sdesc_sw128(a + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024),
                               sdesc_sw128(sb + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id64,
                               (part > 0 || ks > 0) ? 1u : 0u);
                }
            }
            mma_commit(&bars.seed_done);
            const uint32_t id128 = idesc_bf16_f32(128, kCand, false, false);
            for (int t = 0; t < n_tiles && ok; ++t) {
                const int s = t & 1, r = t >> 1;
                if (!mbar_wait(&bars.kv_full[s], r & 1, ctx)) { ok = false; break; }
                if (r >= 1 && !mbar_wait(&bars.s_free[s], (r - 1) & 1, ctx)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kb = smem_u32(sm + kOffKb + s * 2 * kSub);
                for (int part = 0; part < 2; ++part) {
                    const uint32_t a = part ? alo : ahi;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_ss(tmem + kColS0 + s * kCand,
                               sdesc_sw128(a + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024),
                               sdesc_sw128(kb + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024), id128,
                               (part > 0 || ks > 0) ? 1u : 0u);
                }
                mma_commit(&bars.s_full[s]);
                mma_commit(&bars.kv_empty[s]);
            }
            if (!ok) *abort = 1;
            mma_commit(&bars.fin);
            (void)mbar_wait(&bars.fin, 0, ctx);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ workers (warps 0-7)
        volatile int* sm_stop = &bars.sm_stop;
        int nbar = 0;
        bool dead = false;
        auto fail = [&]() {
            dead = true;
            atomicCAS(&bars.sm_stop, 0, nbar + 1);
            *abort = 1;
        };
        auto sync_workers = [&]() {
            asm volatile("bar.sync 1, 256;" ::: "memory");
            ++nbar;
        };
        auto stop_now = [&]() { const int v = *sm_stop; return v != 0 && v <= nbar; };
        // (1) group-summed queries -> A (hi, lo), pilot partial sums.  Warp w: rows 16w..16w+15,
        // lane l: columns 4l..4l+3.
        {
            float pp[4] = {0.f, 0.f, 0.f, 0.f};
            const int sub = lane >> 4, chunk = (lane & 15) >> 1, within = (lane & 1) * 8;
            for (int rr = 0; rr < 16; ++rr) {
                const int row = warp * 16 + rr;
                float a[4] = {0.f, 0.f, 0.f, 0.f};
                if (row < nrows) {
                    for (int h = 0; h < G; ++h) {
                        const uint2 v = *reinterpret_cast<const uint2*>(
                            q + ((b * H + (int64_t)g * G + h) * Nq + r0 + row) * kD + 4 * lane);
                        a[0] += __uint_as_float(v.x << 16);
                        a[1] += __uint_as_float(v.x & 0xffff0000u);
                        a[2] += __uint_as_float(v.y << 16);
                        a[3] += __uint_as_float(v.y & 0xffff0000u);
                    }
                }
                uint32_t hb[2], lb2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(a[2 * e]), h1 = __float2bfloat16_rn(a[2 * e + 1]);
                    const float r0f = a[2 * e] - __bfloat162float(h0), r1f = a[2 * e + 1] - __bfloat162float(h1);
                    hb[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    lb2[e] = pack_bf16x2(r0f, r1f);
                }
                const int off = sub * kSub + row * 128 + ((chunk ^ (row & 7)) << 4) + within;
                *reinterpret_cast<uint2*>(sm + kOffAhi + off) = make_uint2(hb[0], hb[1]);
                *reinterpret_cast<uint2*>(sm + kOffAlo + off) = make_uint2(lb2[0], lb2[1]);
#pragma unroll
                for (int e = 0; e < 4; ++e) pp[e] += a[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) bars.ppart[warp][4 * lane + e] = pp[e];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.a_ready);
        }
        sync_workers();
        if (tid < kD) {
            float p = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) p += bars.ppart[w][tid];
            bars.pilot[tid] = p;
        }
        sync_workers();
        // (2) seeds: top-K candidates of [lo, hi_all] by the pilot score (every row may take them).
        const bool seeded = rank && ncand_all >= K;
        if (seeded) {
            uint64_t l0 = 0, l1 = 0;
            const int nbatch = (ncand_all + 31) / 32;
            for (int bt = warp; bt < nbatch; bt += 8) {
                const int blk = lo + bt * 32 + lane;
                uint64_t key = 0;
                if (blk <= hi_all) {
                    const uint4* row = reinterpret_cast<const uint4*>(kbar + (bg * nb + blk) * (int64_t)kD);
                    float s = 0.f;
#pragma unroll 4
                    for (int c = 0; c < kD / 8; ++c) {
                        const uint4 v = row[c];
                        const float* pv = bars.pilot + 8 * c;
                        s = fmaf(pv[0], __uint_as_float(v.x << 16), s);
                        s = fmaf(pv[1], __uint_as_float(v.x & 0xffff0000u), s);
                        s = fmaf(pv[2], __uint_as_float(v.y << 16), s);
                        s = fmaf(pv[3], __uint_as_float(v.y & 0xffff0000u), s);
                        s = fmaf(pv[4], __uint_as_float(v.z << 16), s);
                        s = fmaf(pv[5], __uint_as_float(v.z & 0xffff0000u), s);
                        s = fmaf(pv[6], __uint_as_float(v.w << 16), s);
                        s = fmaf(pv[7], __uint_as_float(v.w & 0xffff0000u), s);
                    }
                    key = sel_key(s, blk);
                }
                offer(l0, l1, key, 0ull, K, lane);
            }
            uint64_t* pl = reinterpret_cast<uint64_t*>(sm + kOffPList) + warp * kCap;
            pl[2 * lane] = l0;
            pl[2 * lane + 1] = l1;
            sync_workers();
#pragma unroll
            for (int span = 4; span >= 1; span >>= 1) {
                if (warp < span) {
                    uint64_t* pa = reinterpret_cast<uint64_t*>(sm + kOffPList) + warp * kCap;
                    const uint64_t* pb = reinterpret_cast<const uint64_t*>(sm + kOffPList) + (warp + span) * kCap;
                    uint64_t a0 = pa[2 * lane], a1 = pa[2 * lane + 1];
                    merge_desc(a0, a1, pb[2 * lane], pb[2 * lane + 1], lane);
                    pa[2 * lane] = a0;
                    pa[2 * lane + 1] = a1;
                }
                sync_workers();
            }
            if (warp == 0) {
                const uint64_t* pl0 = reinterpret_cast<const uint64_t*>(sm + kOffPList);
                if (2 * lane < K) bars.seeds[2 * lane] = key_block(pl0[2 * lane]);
                if (2 * lane + 1 < K) bars.seeds[2 * lane + 1] = key_block(pl0[2 * lane + 1]);
                if (lane == 0) bars.n_seeds = K;
            }
            sync_workers();
            // seed kbar rows -> B operand (K-major, 128-byte swizzle), zero rows past K
            for (int e = tid; e < kCap * 16; e += kWorkers) {
                const int j = e >> 4, cc = e & 15;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (j < K) v = reinterpret_cast<const uint4*>(kbar + (bg * nb + bars.seeds[j]) * (int64_t)kD)[cc];
                const int off = (cc >> 3) * 8192 + j * 128 + (((cc & 7) ^ (j & 7)) << 4);
                *reinterpret_cast<uint4*>(sm + kOffSeedB + off) = v;
            }
            fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.seed_ready);
        // (3) per-row floors from the rows' own seed scores (warps 0-3 read TMEM lanes = rows).
        if (warp < 4) {
            uint64_t fk = 0;
            if (seeded && n_tiles > 0) {
                if (!mbar_wait(&bars.seed_done, 0, ctx)) fail();
                tc_fence_after();
                if (!__any_sync(0xffffffffu, dead)) {
                    uint32_t x[64];
                    const uint32_t lb = tmem_lane_base(warp);
                    tmem_ld32(tmem + lb + kColSeed, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
                    tmem_ld32(tmem + lb + kColSeed + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
                    tmem_ld_wait();
                    fk = ~0ull;
#pragma unroll
                    for (int j = 0; j < kCap; ++j) {
                        if (j < K) {
                            const uint64_t k2 = sel_key(__uint_as_float(x[j]), bars.seeds[j]);
                            fk = k2 < fk ? k2 : fk;
                        }
                    }
                }
            }
            bars.floor_key[tid] = fk;
        }
        sync_workers();
        if (stop_now()) dead = true;
        // (4) main pass
        uint64_t L0[16], L1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) L0[i] = L1[i] = 0ull;
        bool stop = dead;
        for (int t = 0; t < n_tiles && !stop; ++t) {
            const int s = t & 1, r = t >> 1;
            if (warp < 4) {
                if (!dead && !mbar_wait(&bars.s_full[s], r & 1, ctx)) fail();
                tc_fence_after();
                if (!__any_sync(0xffffffffu, dead)) {
                    const uint32_t lb = tmem_lane_base(warp);
                    float* dst = reinterpret_cast<float*>(sm + kOffSC) + tid * kSCStride;
#pragma unroll 1
                    for (int c0 = 0; c0 < kCand; c0 += 32) {
                        uint32_t x[32];
                        tmem_ld32(tmem + lb + kColS0 + s * kCand + c0, x);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(dst + c0 + j) =
                                make_float4(__uint_as_float(x[j]), __uint_as_float(x[j + 1]),
                                            __uint_as_float(x[j + 2]), __uint_as_float(x[j + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.s_free[s]);
            }
            sync_workers();
            if (stop_now()) { stop = true; break; }
            const int j0 = lo + t * kCand;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int row = warp * 16 + i;
                const int lim = row < nrows ? (r0 + row) / kBlk - n_local : -1;
                if (lim - lo + 1 <= topk) continue;  // row takes every candidate
                const uint64_t fl = bars.floor_key[row];
                const float* src = reinterpret_cast<const float*>(sm + kOffSC) + row * kSCStride;
#pragma unroll
                for (int qq = 0; qq < kCand / 32; ++qq) {
                    const int blk = j0 + qq * 32 + lane;
                    const uint64_t key = blk <= lim ? sel_key(src[qq * 32 + lane], blk) : 0ull;
                    offer(L0[i], L1[i], key, fl, K, lane);
                }
            }
            sync_workers();
        }
        // (5) output rows: init ids, sorted top-k ids, local ids, -1 padding.
        if (!stop) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int row = warp * 16 + i;
                if (row >= nrows) continue;
                const int rq = r0 + row;
                const int c = rq / kBlk;
                const int ncand = c - n_local - n_init + 1;
                int32_t* out = idx + (bg * Nq + rq) * (int64_t)slots;
                if (ncand <= topk) {
                    for (int s = lane; s < slots; s += 32) out[s] = s <= c ? s : -1;
                    continue;
                }
                int x0 = (2 * lane < K && L0[i]) ? key_block(L0[i]) : 0x7fffffff;
                int x1 = (2 * lane + 1 < K && L1[i]) ? key_block(L1[i]) : 0x7fffffff;
                sort64_asc(x0, x1, lane);
                for (int s = lane; s < n_init; s += 32) out[s] = s;
                if (2 * lane < K) out[n_init + 2 * lane] = x0;
                if (2 * lane + 1 < K) out[n_init + 2 * lane + 1] = x1;
                for (int u = lane; u < n_local; u += 32) out[n_init + K + u] = c - n_local + 1 + u;
                for (int s = n_init + K + n_local + lane; s < slots; s += 32) out[s] = -1;
            }
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

bool block_topk_tc_supported(int H, int Hkv, int Nq, int q_pos0, int nb, int d, int topk) {
    (void)H; (void)Hkv;
    return d == kD && q_pos0 == 0 && Nq > 16 && topk <= kCap;
}

cudaError_t launch_block_topk_tc(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                 int Hkv, int Nq, int nb, int topk, int n_init, int n_local,
                                 cudaStream_t st, DevCtx ctx) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tm;
    const uint64_t rows = nb > 0 ? (uint64_t)nb : 1;
    cuuint64_t dims[3] = {(cuuint64_t)kD, rows, (cuuint64_t)B * Hkv};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * rows};
    cuuint32_t box[3] = {64, kCand, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kbar), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem<topk_tc_kernel>(kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(Nq, kRows), (unsigned)(B * Hkv));
    topk_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        tm, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kbar), idx, H,
        Hkv, Nq, nb, topk, n_init, n_local, n_init + n_local + topk, ctx);
    return cudaGetLastError();
}

}  // namespace sala
