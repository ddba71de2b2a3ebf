// Block selection on the 5th-generation tensor cores (sm_100a): scores of 128 query rows against
// 128 candidate blocks per MMA, exact per-row top-k behind a provable floor.
//
// Tile: 128 consecutive query rows (two query blocks) of one (batch, KV group).  The group-summed
// query qbar_r = sum_{h in g} q_{h,r} is formed in fp32 and split into two bf16 terms
// hi = bf16(qbar), lo = bf16(qbar - hi), so score = hi.kbar + lo.kbar carries ~16 significant bits
// of qbar on bf16 tensor cores (kbar itself is bf16, exact).
//
// Floor: the pilot vector p = sum_r qbar_r ranks the candidates that every row of the tile may
// take; its best 2k become seeds.  Row r's k-th best score is at least the k-th best of its own
// seed scores (k real candidates reach it), so a candidate scoring below that floor can never
// enter row r's top-k (the floor kept is that score rounded down to 16 bits of its orderable
// form, a lower bound as well).  The seeds only decide how much work is skipped, never the
// result: the selection is exact.
//
// Main pass, per 128-candidate tile: MMA (2 x 8 K-steps, N = 128) -> TMEM (double-buffered) ->
// one thread per query row reads its 128 scores straight from TMEM, compares each with the row's
// floor, and appends the few that pass to the row's buffer in shared memory, in ascending block
// order.  A full buffer is cut back to its best k, order kept (the floor rises to the k-th
// score); at the end the buffer's smallest keys are dropped until k remain (a bitwise select of
// the k-th best score when many more than k are left), and the rest are taken in buffer order.
// Key = (orderable score, ~block), so ties go to the lower block index.  Output as the
// CUDA-core path: init ids, top-k ids ascending, local ids.
//
// The producer warp also stages, by bulk copies, what the phases before the main pass read:
// each query head's rows of the tile for the group sum, and the candidates' kbar rows for the
// pilot scores, in areas the later phases take over.
//
// Roles (320 threads): warps 0-7 workers (the main pass runs on warps 0-3, thread = row = TMEM
// lane), warp 8 TMA producer (kbar tiles), warp 9 TMEM owner and MMA issuer.  Every wait is
// bounded; the 8 workers leave only together (the sparse prefill kernel's named-barrier
// discipline).
#include "blocksel.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128, kRows = 128, kCand = 128, kBlk = 64, kCap = 64;
constexpr int kThreads = 320, kWorkers = 256;
constexpr int kMaxG = 16;
constexpr int kBufCap = 88;                            // buffered keys per row
static_assert(kBufCap <= 96, "keep_best reads three keys per lane");
constexpr int kSub = 128 * 128;                        // [128 rows x 128 B] = 16 KiB
constexpr int kOffAhi = 0, kOffAlo = 2 * kSub;         // A operands (hi, lo), 2 sub-tiles each
constexpr int kOffKb = 4 * kSub;                       // kbar tiles, 2 stages x 2 sub-tiles
constexpr int kOffBuf = 8 * kSub;                      // row buffers [128][kBufCap] keys
constexpr int kBufBytes = kRows * kBufCap * 8;
constexpr int kSmemBytes = kOffBuf + kBufBytes + 1024;
// Before the main pass the buffer area holds, in turn: the pilot partial sums, the pilot keys of
// one chunk of candidates, and the seeds' kbar rows (the B operand of the seed MMA).
constexpr int kOffPPart = kOffBuf;                     // [8][128] floats
constexpr int kPilotChunk = 16 * kWorkers;             // keys per radix-select chunk
constexpr int kOffPKeys = kOffBuf;                     // [kPilotChunk] keys
constexpr int kSeeds = 2 * kCap;                       // pilot seeds (the floor uses the k-th)
constexpr int kOffSeedB = kOffBuf + kPilotChunk * 8;   // [128 seeds x 128 d], 2 sub-tiles
static_assert(kOffSeedB + 2 * kSub <= kOffBuf + kBufBytes, "buffer area too small");
// While the group sum runs, the A operand area and the buffer area hold four stages of one query
// head's 128 rows each ([128 rows x 256 B], as in global memory): stages 0-1 in A, 2-3 in the
// buffers.  A is written only once every head has been summed.
constexpr int kQStages = 4, kQStageBytes = kRows * kD * 2;
static_assert(2 * kQStageBytes == kOffKb - kOffAhi && 2 * kQStageBytes <= kBufBytes, "Q stages");
// The pilot scores read the candidates' kbar rows in pieces of 128 rows ([128 rows x 256 B]),
// copied into three stages: the two kbar tile stages (the main pass loads them afterwards) and
// the seed operand area (written once every piece has been scored).
constexpr int kSdStages = 3, kSdRows = 128, kSdStageBytes = kSdRows * kD * 2;
static_assert(2 * kSdStageBytes == 4 * kSub && kSdStageBytes <= 2 * kSub, "seed stages");

constexpr uint32_t kColS0 = 0, kColSeed = 256, kTmemCols = 512;

struct Bars {
    uint64_t a_ready, seed_ready, seed_done;
    uint64_t q_full[kQStages], q_empty[kQStages];
    uint64_t sd_full[kSdStages], sd_empty[kSdStages];
    uint64_t kv_full[2], kv_empty[2], s_full[2], s_free[2];
    uint64_t fin;
    uint32_t tmem_base;
    int abort;
    int sm_stop;
    float pilot[kD];
    float floor_s[kRows];
    int buf_n[kRows];
    uint64_t carry[kSeeds];
    int seeds[kSeeds];
    int n_seeds, n_win;
    RadixSelSmem rs;
};

// K-th largest of R independent arrays of up to 128 orderable scores held four per lane (0 marks
// an empty slot; every array holds at least K scores), returned to every lane: the largest t with
// #(x >= t) >= K, decided one bit at a time from the top, one warp-wide count per bit.  The R rows
// are interleaved so that each one's reduction latency hides behind the others'.  With kBits < 32
// the low 32 - kBits bits of t stay zero: t is then the K-th largest with those bits cleared, a
// lower bound of it (all a floor needs).
template <int R, int kBits>
__device__ __forceinline__ void kth_largest(const uint32_t (&x)[R][4], int K, uint32_t (&t)[R]) {
#pragma unroll
    for (int r = 0; r < R; ++r) t[r] = 0u;
#pragma unroll 4
    for (int bit = 31; bit >= 32 - kBits; --bit) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t c = t[r] | (1u << bit);
            const int cnt = __reduce_add_sync(0xffffffffu, (int)(x[r][0] >= c) + (int)(x[r][1] >= c) +
                                                               (int)(x[r][2] >= c) + (int)(x[r][3] >= c));
            t[r] = cnt >= K ? c : t[r];
        }
    }
}

__device__ __forceinline__ float from_orderable(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// The K best keys of a row buffer of n keys (n <= 96), in buffer order: those whose orderable
// score beats s_k (the K-th best score), then the first K - #beating of those that tie with it.
// Buffers are appended in ascending block order, so "first" is "lowest block", the tie rule of
// the keys.  One warp; emit(pos, key) is called for the kept keys, pos = 0 .. kept-1 in order;
// returns the number kept.  All reads happen before the first emit, so emit may write the
// buffer in place.
template <typename Emit>
__device__ __forceinline__ int keep_best(const uint64_t* buf, int n, int K, uint32_t s_k, int lane,
                                         Emit emit) {
    uint64_t key[3];
    bool gt[3], eq[3];
    int n_gt = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int p = lane + 32 * j;
        key[j] = p < n ? buf[p] : 0ull;
        const uint32_t o = (uint32_t)(key[j] >> 32);
        gt[j] = p < n && o > s_k;
        eq[j] = p < n && o == s_k;
        n_gt += __popc(__ballot_sync(0xffffffffu, gt[j]));
    }
    __syncwarp();
    const int need = K - n_gt;
    const unsigned below = (1u << lane) - 1u;
    int base = 0, eq_base = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const unsigned ue = __ballot_sync(0xffffffffu, eq[j]);
        const bool take = gt[j] || (eq[j] && eq_base + __popc(ue & below) < need);
        const unsigned ut = __ballot_sync(0xffffffffu, take);
        if (take) emit(base + __popc(ut & below), key[j]);
        base += __popc(ut);
        eq_base += __popc(ue);
    }
    return base;
}

__global__ void __launch_bounds__(kThreads, 1)
topk_tc_kernel(const __grid_constant__ CUtensorMap tmKb, const __nv_bfloat16* __restrict__ q,
               const __nv_bfloat16* __restrict__ kbar, int32_t* __restrict__ idx, int H, int Hkv,
               int Hs, int Nq, int nb, int topk, int n_init, int n_local, int slots, DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Selection group (b, g) of Hs per batch: the G = H / Hs query heads g*G .. g*G+G-1, scored
    // against their KV head's kbar (Hs = Hkv: the KV group; Hs = H: one query head).
    const int G = H / Hs;
    // Heaviest tiles first: a tile's work grows with its candidate count, i.e. with its row
    // index, so the launch order walks row tiles from the last to the first (all groups of one
    // row tile together) and the lightest tiles fill the tail.
    const int n_rt = (Nq + kRows - 1) / kRows;
    const int n_bg = (int)(gridDim.x / n_rt);
    const int64_t bg = blockIdx.x % n_bg;
    const int64_t b = bg / Hs;
    const int g = (int)(bg % Hs);
    const int64_t kv_plane = b * Hkv + g / (Hs / Hkv);
    const int r0 = (n_rt - 1 - (int)(blockIdx.x / n_bg)) * kRows;
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
    // Seeds (the pilot's best kSeeds candidates of [lo, hi_all]) are used when every row may take
    // that many; the pilot scores go through a radix select in chunks of kNew candidates.
    const bool seeded = rank && ncand_all >= kSeeds;
    constexpr int kNew = kPilotChunk - kSeeds;
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
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&bars.q_full[s], 1);
            mbar_init(&bars.q_empty[s], 8);  // the worker warps
        }
        for (int s = 0; s < kSdStages; ++s) {
            mbar_init(&bars.sd_full[s], 1);
            mbar_init(&bars.sd_empty[s], 8);
        }
        bars.abort = 0;
        bars.sm_stop = 0;
        bars.n_seeds = 0;
        fence_mbar_init();
    }
    if (tid < kRows) bars.buf_n[tid] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    auto q_stage = [&](int s) { return sm + (s < 2 ? kOffAhi : kOffBuf - 2 * kQStageBytes) + s * kQStageBytes; };
    auto sd_stage = [&](int s) { return sm + (s < 2 ? kOffKb + s * kSdStageBytes : kOffSeedB); };

    if (warp == 8) {
        // ------------------------------------------------------------------ TMA producer
        // First the tile's rows of the G query heads, one head per stage, for the group sum; then
        // the kbar tiles of the main pass.
        int hq = 0;  // heads issued
        if (lane == 0) {
            const uint32_t qbytes = (uint32_t)nrows * kD * 2;
            for (; hq < G; ++hq) {
                const int s = hq % kQStages, u = hq / kQStages;
                if (u >= 1 && !mbar_wait(&bars.q_empty[s], (u - 1) & 1, ctx)) { *abort = 1; break; }
                mbar_arrive_expect_tx(&bars.q_full[s], qbytes);
                bulk_load_g2s(q_stage(s), q + ((b * H + (int64_t)g * G + hq) * Nq + r0) * kD, qbytes,
                              &bars.q_full[s]);
            }
        }
        // Then the candidates' kbar rows for the pilot scores, piece by piece, and once the pieces
        // in the kbar tile stages have been read, the main pass's tiles.
        int ksd = 0;  // pieces issued
        if (lane == 0 && seeded) {
            bool ok = true;
            for (int cb = 0; cb < ncand_all && ok; cb += kNew) {
                const int nc = min(kNew, ncand_all - cb);
                for (int sc0 = 0; sc0 < nc; sc0 += kSdRows, ++ksd) {
                    const int s = ksd % kSdStages, u = ksd / kSdStages;
                    if (u >= 1 && !mbar_wait(&bars.sd_empty[s], (u - 1) & 1, ctx)) {
                        *abort = 1;
                        ok = false;
                        break;
                    }
                    // seed stage 2 is query stage 3: its last head must have been read
                    constexpr int kQ3 = kQStages - 1;
                    static_assert(kSdStages == 3 && kOffSeedB == kOffBuf + kQStageBytes, "stage overlap");
                    if (ksd == 2 && hq > kQ3 &&
                        !mbar_wait(&bars.q_empty[kQ3], ((kQ3 + kQStages * ((hq - 1 - kQ3) / kQStages)) / kQStages) & 1, ctx)) {
                        *abort = 1;
                        ok = false;
                        break;
                    }
                    const uint32_t bytes = (uint32_t)min(kSdRows, nc - sc0) * kD * 2;
                    mbar_arrive_expect_tx(&bars.sd_full[s], bytes);
                    bulk_load_g2s(sd_stage(s), kbar + (kv_plane * nb + lo + cb + sc0) * (int64_t)kD, bytes,
                                  &bars.sd_full[s]);
                }
            }
            for (int s = 0; s < min(ksd, 2); ++s)
                (void)mbar_wait(&bars.sd_empty[s], ((s + kSdStages * ((ksd - 1 - s) / kSdStages)) / kSdStages) & 1, ctx);
        }
        if (lane == 0 && n_tiles > 0) {
            int issued0 = -1, issued1 = -1;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t & 1, r = t >> 1;
                if (r >= 1 && !mbar_wait(&bars.kv_empty[s], (r - 1) & 1, ctx)) { *abort = 1; break; }
                uint8_t* st = sm + kOffKb + s * 2 * kSub;
                mbar_arrive_expect_tx(&bars.kv_full[s], 2 * kSub);
                const int y = lo + t * kCand;
                tma_load_3d(st, &tmKb, &bars.kv_full[s], 0, y, (int)kv_plane);
                tma_load_3d(st + kSub, &tmKb, &bars.kv_full[s], 64, y, (int)kv_plane);
                if (s == 0) issued0 = r; else issued1 = r;
            }
            if (issued0 >= 0) (void)mbar_wait(&bars.kv_full[0], issued0 & 1, ctx);
            if (issued1 >= 0) (void)mbar_wait(&bars.kv_full[1], issued1 & 1, ctx);
        }
        if (lane == 0) {  // drain: the last copy into each stage has landed
            for (int s = 0; s < min(hq, kQStages); ++s)
                (void)mbar_wait(&bars.q_full[s], ((s + kQStages * ((hq - 1 - s) / kQStages)) / kQStages) & 1, ctx);
            for (int s = 0; s < min(ksd, kSdStages); ++s)
                (void)mbar_wait(&bars.sd_full[s], ((s + kSdStages * ((ksd - 1 - s) / kSdStages)) / kSdStages) & 1, ctx);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            const uint32_t ahi = smem_u32(sm + kOffAhi), alo = smem_u32(sm + kOffAlo);
            bool ok = mbar_wait(&bars.a_ready, 0, ctx);
            // Seed scores: [128 rows] x [128 seeds], only when the floor is used.
            if (ok) ok = mbar_wait(&bars.seed_ready, 0, ctx);
            if (ok && bars.n_seeds == kSeeds) {
                tc_fence_after();
                const uint32_t sb = smem_u32(sm + kOffSeedB);
                const uint32_t idS = idesc_bf16_f32(128, kSeeds, false, false);
                for (int part = 0; part < 2; ++part) {
                    const uint32_t a = part ? alo : ahi;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_ss(tmem + kColSeed, sdesc_sw128(a + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024),
                               sdesc_sw128(sb + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024), idS,
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
        // (1) group-summed queries -> A (hi, lo), pilot partial sums.  The G heads' rows arrive
        // one head per stage; warp w sums rows 16w..16w+15, lane l columns 4l..4l+3, adding the
        // heads in order (rows past the tile stay 0).
        {
            float acc[16][4];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[rr][e] = 0.f;
            for (int h = 0; h < G; ++h) {
                const int s = h % kQStages, u = h / kQStages;
                const bool got = mbar_wait(&bars.q_full[s], u & 1, ctx);
                if (!__all_sync(0xffffffffu, got)) {
                    fail();
                    break;
                }
                const uint8_t* st = q_stage(s);
                uint2 v[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr)
                    v[rr] = *reinterpret_cast<const uint2*>(st + (warp * 16 + rr) * (kD * 2) + 8 * lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.q_empty[s]);
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    if (warp * 16 + rr >= nrows) continue;
                    acc[rr][0] += __uint_as_float(v[rr].x << 16);
                    acc[rr][1] += __uint_as_float(v[rr].x & 0xffff0000u);
                    acc[rr][2] += __uint_as_float(v[rr].y << 16);
                    acc[rr][3] += __uint_as_float(v[rr].y & 0xffff0000u);
                }
            }
            // A and the buffer area held the stages: every worker is done reading them
            sync_workers();
            float* ppart = reinterpret_cast<float*>(sm + kOffPPart);
            float pp[4] = {0.f, 0.f, 0.f, 0.f};
            const int sub = lane >> 4, chunk = (lane & 15) >> 1, within = (lane & 1) * 8;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int row = warp * 16 + rr;
                float a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) a[e] = G < kMaxG ? acc[rr][e] + 0.f : acc[rr][e];  // -0 -> +0 below 16 heads
                uint32_t hb[2], lb2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(a[2 * e]), h1 = __float2bfloat16_rn(a[2 * e + 1]);
                    const float d0 = a[2 * e] - __bfloat162float(h0), d1 = a[2 * e + 1] - __bfloat162float(h1);
                    hb[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    lb2[e] = pack_bf16x2(d0, d1);
                }
                const int off = sub * kSub + row * 128 + ((chunk ^ (row & 7)) << 4) + within;
                *reinterpret_cast<uint2*>(sm + kOffAhi + off) = make_uint2(hb[0], hb[1]);
                *reinterpret_cast<uint2*>(sm + kOffAlo + off) = make_uint2(lb2[0], lb2[1]);
#pragma unroll
                for (int e = 0; e < 4; ++e) pp[e] += a[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) ppart[warp * kD + 4 * lane + e] = pp[e];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.a_ready);
        }
        sync_workers();
        if (tid < kD) {
            const float* ppart = reinterpret_cast<const float*>(sm + kOffPPart);
            float p = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) p += ppart[w * kD + tid];
            bars.pilot[tid] = p;
        }
        sync_workers();
        // (2) seeds: the best kSeeds candidates of [lo, hi_all] by the pilot score (every row may
        // take them).  Pilot scores of a chunk of candidates, read from the staged kbar pieces (8
        // lanes per row, lane l: columns 8(l%8)..+7 and 64+8(l%8)..+7), plus the winners so far,
        // then a radix select.
        if (seeded) {
            uint64_t* pkeys = reinterpret_cast<uint64_t*>(sm + kOffPKeys);
            if (tid < kSeeds) bars.carry[tid] = 0ull;
            sync_workers();
            const int part = lane & 7;
            float pv[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                pv[e] = bars.pilot[part * 8 + e];
                pv[8 + e] = bars.pilot[64 + part * 8 + e];
            }
            int ksd = 0;  // pieces consumed
            for (int cb = 0; cb < ncand_all; cb += kNew) {
                const int nc = min(kNew, ncand_all - cb);
                for (int sc0 = 0; sc0 < nc; sc0 += kSdRows, ++ksd) {
                    const int s = ksd % kSdStages;
                    const bool got = !dead && mbar_wait(&bars.sd_full[s], (ksd / kSdStages) & 1, ctx);
                    if (!__all_sync(0xffffffffu, got)) {
                        if (!dead) fail();
                        continue;
                    }
                    const uint8_t* st = sd_stage(s);
                    uint4 raw[4][2];
#pragma unroll
                    for (int ps = 0; ps < 4; ++ps) {
                        const uint8_t* row = st + (ps * 32 + warp * 4 + (lane >> 3)) * (kD * 2) + part * 16;
                        raw[ps][0] = *reinterpret_cast<const uint4*>(row);
                        raw[ps][1] = *reinterpret_cast<const uint4*>(row + 128);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars.sd_empty[s]);
#pragma unroll
                    for (int ps = 0; ps < 4; ++ps) {
                        float d0 = 0.f, d1 = 0.f;
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const uint4 v = raw[ps][u];
                            const float* p8 = pv + 8 * u;
                            d0 = fmaf(p8[0], __uint_as_float(v.x << 16), d0);
                            d1 = fmaf(p8[1], __uint_as_float(v.x & 0xffff0000u), d1);
                            d0 = fmaf(p8[2], __uint_as_float(v.y << 16), d0);
                            d1 = fmaf(p8[3], __uint_as_float(v.y & 0xffff0000u), d1);
                            d0 = fmaf(p8[4], __uint_as_float(v.z << 16), d0);
                            d1 = fmaf(p8[5], __uint_as_float(v.z & 0xffff0000u), d1);
                            d0 = fmaf(p8[6], __uint_as_float(v.w << 16), d0);
                            d1 = fmaf(p8[7], __uint_as_float(v.w & 0xffff0000u), d1);
                        }
                        float d = d0 + d1;
                        d += __shfl_xor_sync(0xffffffffu, d, 1);
                        d += __shfl_xor_sync(0xffffffffu, d, 2);
                        d += __shfl_xor_sync(0xffffffffu, d, 4);
                        const int i = sc0 + ps * 32 + warp * 4 + (lane >> 3);
                        if (part == 0 && i < nc) pkeys[i] = sel_key(d, lo + cb + i);
                    }
                }
                for (int i = nc + tid; i < kNew; i += kWorkers) pkeys[i] = 0ull;
                if (tid < kSeeds) pkeys[kNew + tid] = bars.carry[tid];
                sync_workers();
                uint64_t key[kPilotChunk / kWorkers];
#pragma unroll
                for (int e = 0; e < kPilotChunk / kWorkers; ++e) key[e] = pkeys[e * kWorkers + tid];
                uint64_t prefix, mask;
                radix_kth<kPilotChunk / kWorkers>(key, kSeeds, bars.rs, prefix, mask, tid, sync_workers);
                if (tid == 0) bars.n_win = 0;
                sync_workers();
#pragma unroll
                for (int e = 0; e < kPilotChunk / kWorkers; ++e)
                    if (key[e] && (key[e] & mask) >= prefix) bars.carry[atomicAdd(&bars.n_win, 1)] = key[e];
                sync_workers();
            }
            if (tid < kSeeds) {
                const int sd = key_block(bars.carry[tid]);
                bars.seeds[tid] = in_bounds(ctx, sd >= lo && sd <= hi_all) ? sd : lo;
            }
            if (tid == 0) bars.n_seeds = kSeeds;
            sync_workers();
            // seed kbar rows -> B operand (K-major, 128-byte swizzle); all loads in flight first
            constexpr int kPer = kSeeds * 16 / kWorkers;
            uint4 sv[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int e = u * kWorkers + tid, j = e >> 4, cc = e & 15;
                sv[u] = reinterpret_cast<const uint4*>(kbar + (kv_plane * nb + bars.seeds[j]) * (int64_t)kD)[cc];
            }
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int e = u * kWorkers + tid, j = e >> 4, cc = e & 15;
                const int off = (cc >> 3) * kSub + j * 128 + (((cc & 7) ^ (j & 7)) << 4);
                *reinterpret_cast<uint4*>(sm + kOffSeedB + off) = sv[u];
            }
            fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.seed_ready);
        // (3) per-row floors: the k-th best of the row's own seed scores, to 16 bits of its
        // orderable form.  Warps 0-3, thread = row = TMEM lane: the row's seed scores come into
        // registers, and the bits of the k-th best are decided one at a time by counting, from the
        // highest bit in which the row's largest and smallest seed scores differ (the bits above
        // are common to all of them, hence to the k-th best).
        if (seeded && n_tiles > 0) {
            if (warp < 4) {
                if (!mbar_wait(&bars.seed_done, 0, ctx)) fail();
                tc_fence_after();
                float fl = -INFINITY;
                if (!__any_sync(0xffffffffu, dead)) {
                    const uint32_t lb = tmem_lane_base(warp);
                    uint32_t x[kSeeds];
#pragma unroll
                    for (int c = 0; c < kSeeds; c += 32)
                        tmem_ld32(tmem + lb + kColSeed + c, *reinterpret_cast<uint32_t(*)[32]>(x + c));
                    tmem_ld_wait();
                    uint32_t omax = 0u, omin = ~0u;
#pragma unroll
                    for (int j = 0; j < kSeeds; ++j) {
                        x[j] = orderable(__uint_as_float(x[j]));
                        omax = max(omax, x[j]);
                        omin = min(omin, x[j]);
                    }
                    const int p = __clz(omax ^ omin);  // 32 when all are equal
                    uint32_t t = p >= 32 ? omax : omax & ~(0xffffffffu >> p);
#pragma unroll 1
                    for (int bit = 31 - p; bit >= 16; --bit) {
                        const uint32_t c = t | (1u << bit);
                        int cnt = 0;
#pragma unroll
                        for (int j = 0; j < kSeeds; ++j) cnt += x[j] >= c ? 1 : 0;
                        t = cnt >= K ? c : t;
                    }
                    fl = from_orderable(t & 0xffff0000u);
                }
                bars.floor_s[tid] = fl;
            }
        } else if (tid < kRows) {
            bars.floor_s[tid] = -INFINITY;
        }
        sync_workers();
        if (stop_now()) dead = true;
        // (4) main pass, warps 0-3, thread = query row = TMEM lane: per 32-candidate chunk, the
        // candidates at or above the row's floor go to the row's buffer.  A row whose buffer would
        // overflow is first cut back to its best k by its whole warp (the floor rises).
        if (warp < 4 && n_tiles > 0) {
            const int row = tid;
            const int lim = row < nrows ? (r0 + row) / kBlk - n_local : -1;
            const bool act = lim - lo + 1 > topk;  // this row ranks its candidates
            float fl = bars.floor_s[row];
            int n = 0;
            uint64_t* bufs = reinterpret_cast<uint64_t*>(sm + kOffBuf);
            uint64_t* buf = bufs + row * kBufCap;
            const uint32_t lb = tmem_lane_base(warp);
            auto cut = [&](int src) {  // whole warp: row warp*32 + src back to its best K keys
                const int nsrc = __shfl_sync(0xffffffffu, n, src);
                uint64_t* b2 = bufs + (warp * 32 + src) * kBufCap;
                uint32_t v[1][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    v[0][u] = 4 * lane + u < nsrc ? (uint32_t)(b2[4 * lane + u] >> 32) : 0u;
                uint32_t t[1];
                kth_largest<1, 32>(v, K, t);
                const uint32_t s_k = t[0];
                keep_best(b2, nsrc, K, s_k, lane, [&](int pos, uint64_t key) { b2[pos] = key; });
                __syncwarp();
                if (lane == src) {
                    n = K;
                    fl = from_orderable(s_k);
                }
            };
            // One 32-candidate chunk of this row's scores (candidates jb .. jb + 31).
            // Whether any row of the warp has a visible candidate of the chunk at or above its floor.
            auto worth = [&](const uint32_t (&x)[32], int jb) {
                float m[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    m[k] = fmax3(__uint_as_float(x[4 * k]), __uint_as_float(x[4 * k + 1]),
                                 fmaxf(__uint_as_float(x[4 * k + 2]), __uint_as_float(x[4 * k + 3])));
                const float mx = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
                return __any_sync(0xffffffffu, act && lim >= jb && mx >= fl);
            };
            auto filter = [&](const uint32_t (&x)[32], int jb) {
                const int jmax = act ? min(32, lim - jb + 1) : 0;  // visible candidates
                auto passing = [&](uint32_t keep) {
                    uint32_t msk = 0;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        msk |= (j < jmax && __uint_as_float(x[j]) >= fl) ? (1u << j) : 0u;
                    return msk & keep;
                };
                auto append = [&](uint32_t msk) {
                    // A row passes ~1 candidate of 32: park the chunk in this thread's local memory
                    // (L1-resident) and visit only the set bits, in ascending order.
                    if (msk == 0u) return;
                    uint32_t xs[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) xs[j] = x[j];
                    do {
                        const int j = __ffs(msk) - 1;
                        msk &= msk - 1u;
                        if (in_bounds(ctx, n < kBufCap)) buf[n++] = sel_key(__uint_as_float(xs[j]), jb + j);
                    } while (msk);
                };
                const uint32_t pass = passing(~0u);
                if (__any_sync(0xffffffffu, n + __popc(pass) > kBufCap)) {
                    // rare: some row would overflow.  Append in two halves of 16, cutting the
                    // rows that would overflow before each half (a cut leaves k <= 64 keys, so a
                    // half always fits afterwards).
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t half = h ? 0xffff0000u : 0x0000ffffu;
                        unsigned need = __ballot_sync(0xffffffffu, n + __popc(passing(half)) > kBufCap);
                        while (need) {
                            const int src = __ffs(need) - 1;
                            need &= need - 1;
                            cut(src);
                        }
                        append(passing(half));
                    }
                } else {
                    append(pass);
                }
            };
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t & 1, r = t >> 1;
                if (!dead && !mbar_wait(&bars.s_full[s], r & 1, ctx)) fail();
                tc_fence_after();
                if (!__any_sync(0xffffffffu, dead)) {
                    const int j0 = lo + t * kCand;
#pragma unroll 1
                    for (int c = 0; c < kCand; c += 64) {
                        // 64 columns per TMEM round trip; most chunks have nothing at or above
                        // the floors.  The second chunk is loaded again after the first one's
                        // filter, so that it is not held across it.
                        const uint32_t col = tmem + lb + kColS0 + s * kCand + c;
                        uint32_t xa[32], xb[32];
                        tmem_ld32(col, xa);
                        tmem_ld32(col + 32, xb);
                        tmem_ld_wait();
                        const bool wa = worth(xa, j0 + c), wb = worth(xb, j0 + c + 32);
                        if (wa) {
                            filter(xa, j0 + c);
                            if (wb) {
                                tmem_ld32(col + 32, xb);
                                tmem_ld_wait();
                                filter(xb, j0 + c + 32);
                            }
                        } else if (wb) {
                            filter(xb, j0 + c + 32);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.s_free[s]);
            }
            bars.buf_n[row] = n;
        }
        sync_workers();
        // (5) output rows: init ids, the top-k ids in ascending order, local ids, -1 padding.
        // Warp w: rows 16w..16w+15.  A ranked row keeps the K largest keys of its buffer (score,
        // then the lower block), in buffer (= block) order.  The buffer holds n >= K keys, rarely
        // many more: the d = n - K smallest are dropped one at a time (two warp-wide minima
        // each); a row with more than kDrop extra keys takes the bitwise select of its K-th best
        // score instead.  Both keep the same keys.
        if (!stop_now() && !dead) {
            const uint64_t* bufs = reinterpret_cast<const uint64_t*>(sm + kOffBuf);
            constexpr int kDrop = 8;
            const unsigned below = (1u << lane) - 1u;
#pragma unroll 1
            for (int i = 0; i < 16; ++i) {
                const int row = warp * 16 + i;
                if (row >= nrows) break;
                const int rq = r0 + row;
                const int c = rq / kBlk;
                int32_t* out = idx + (bg * Nq + rq) * (int64_t)slots;
                if (c - n_local - n_init + 1 <= topk) {
                    for (int sl = lane; sl < slots; sl += 32) out[sl] = sl <= c ? sl : -1;
                    continue;
                }
                const int n = min(bars.buf_n[row], kBufCap);
                const uint64_t* b = bufs + row * kBufCap;
                int kept;
                if (n - K > kDrop) {
                    uint32_t v[1][4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[0][u] = 4 * lane + u < n ? (uint32_t)(b[4 * lane + u] >> 32) : 0u;
                    uint32_t t[1];
                    kth_largest<1, 32>(v, K, t);
                    kept = keep_best(b, n, K, t[0], lane,
                                     [&](int pos, uint64_t key) { out[n_init + pos] = key_block(key); });
                } else {
                    uint64_t key[3];
                    bool keep[3];
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        const int p = lane + 32 * j;
                        keep[j] = p < n;
                        key[j] = keep[j] ? b[p] : 0ull;
                    }
                    for (int it = K; it < n; ++it) {  // drop the smallest key still kept
                        uint64_t m = ~0ull;
#pragma unroll
                        for (int j = 0; j < 3; ++j) m = keep[j] && key[j] < m ? key[j] : m;
                        const uint32_t mh = __reduce_min_sync(0xffffffffu, (uint32_t)(m >> 32));
                        const uint32_t ml = __reduce_min_sync(0xffffffffu, (uint32_t)(m >> 32) == mh ? (uint32_t)m : ~0u);
                        const uint64_t mk = ((uint64_t)mh << 32) | ml;
#pragma unroll
                        for (int j = 0; j < 3; ++j) keep[j] = keep[j] && key[j] != mk;
                    }
                    kept = 0;
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        const unsigned ut = __ballot_sync(0xffffffffu, keep[j]);
                        if (keep[j]) out[n_init + kept + __popc(ut & below)] = key_block(key[j]);
                        kept += __popc(ut);
                    }
                }
                for (int u = kept + lane; u < K; u += 32) out[n_init + u] = -1;  // unreachable: >= k kept
                for (int sl = lane; sl < n_init; sl += 32) out[sl] = sl;
                for (int u = lane; u < n_local; u += 32) out[n_init + K + u] = c - n_local + 1 + u;
                for (int sl = n_init + K + n_local + lane; sl < slots; sl += 32) out[sl] = -1;
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
    (void)H; (void)Hkv; (void)nb;
    return d == kD && q_pos0 == 0 && Nq > 16 && topk >= 1 && topk <= kCap;
}

cudaError_t launch_block_topk_tc(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                 int Hkv, int Hs, int Nq, int nb, int topk, int n_init,
                                 int n_local, cudaStream_t st, DevCtx ctx) {
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
    dim3 grid((unsigned)(ceil_div(Nq, kRows) * B * Hs));
    topk_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        tm, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kbar), idx, H,
        Hkv, Hs, Nq, nb, topk, n_init, n_local, n_init + n_local + topk, ctx);
    return cudaGetLastError();
}

}  // namespace sala
