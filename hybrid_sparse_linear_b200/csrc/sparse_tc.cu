// Block-sparse softmax attention prefill on the 5th-generation tensor cores (sm_100a).
//
// Work unit ("tile"): 8 consecutive query tokens x the 16 query heads of one KV group = 128 rows,
// the M of one tcgen05 MMA.  Row r = head * 8 + token, so each head's 8 tokens are one 1024-byte
// swizzle atom and the Q tile arrives with a single 3-D TMA box per 64 columns.  The 8 tokens
// share their query block (8 divides 64), hence the forced blocks and the diagonal; their
// top-k choices differ, so the tile walks the UNION of the 8 selections (ascending) and each
// row masks the blocks its token did not choose.  Executed FLOPs exceed the algorithmic ones by
// the union overhead; the sum over each row's own selected keys is exact.
//
// The union is consumed two blocks at a time (a "pair", 128 keys):
//   S    = Q [K_a; K_b]^T        M=128 N=128 K=128  (one MMA; the two K tiles sit back to back
//                                                    in shared memory, so Q is read once)
//   P    = online softmax of S, masked per row by each block's selection bit and, on the
//          diagonal block, by causality                              (registers, fp32)
//   O   += P [V_a; V_b]          M=128 N=128 K=128  (A = P from TMEM, bf16, aliasing S)
// S is double-buffered in TMEM so the next pair's S runs on the tensor core while the softmax
// warps work on this one.  O is rescaled only when a row's running max grows by more than 8 in
// log2 units (the stale max keeps exp2 below 256 and cancels in O / l).
//
// Roles (192 threads, persistent: one CTA per SM walks tiles blockIdx.x, +gridDim.x, ...):
// warps 0-3 softmax + epilogue (thread = row = TMEM lane); warp 4 stages the next tile's
// selection rows in shared memory with coalesced loads, merges them into the union list and
// issues the TMA loads; warp 5 allocates TMEM and issues the MMAs (one thread).  Every wait is
// bounded; a timeout sets the status word, the roles wind down, and the kernel waits (bounded)
// for its own copies and MMAs before it frees TMEM and returns.
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
constexpr int kThreads = 192;

// Shared memory (offsets from a 1024-aligned base).
constexpr int kQBytes = 128 * kD * 2;                 // 2 sub-tiles [128 rows x 128 B]
constexpr int kHalfK = 8192;                          // one K box: [64 rows x 128 B]
constexpr int kPairBytes = 8 * kHalfK;                // K_a|K_b (d 0-63), K_a|K_b (d 64-127), V_a, V_b
constexpr int kOffQ = 0;
constexpr int kOffKV = kQBytes;
constexpr int kOffList = kOffKV + 2 * kPairBytes;
constexpr int kListBytes = kMaxList * 5;              // int32 ids + uint8 token masks
constexpr int kOffStage = kOffList + 2 * kListBytes;  // staged selection rows of one tile
constexpr int kSmemBytes = kOffStage + kTQ * kMaxSlots * 4 + 1024;

// TMEM columns: O [0,128), S buffers [128,256) and [256,384).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS0 = 128;

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t kv_full[2], kv_empty[2];
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t list_full[2], list_empty[2];
    uint64_t fin;
    uint32_t tmem_base;
    int list_n[2];
    int abort;
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
sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
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

    if (warp == 5) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.kv_full[b], 1);
            mbar_init(&bars.kv_empty[b], 1);
            mbar_init(&bars.s_full[b], 1);
            mbar_init(&bars.p_full[b], 4);
            mbar_init(&bars.pv_done[b], 1);
            mbar_init(&bars.list_full[b], 1);
            mbar_init(&bars.list_empty[b], 2);
        }
        mbar_init(&bars.fin, 1);
        bars.abort = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    int32_t* list_id[2] = {reinterpret_cast<int32_t*>(sm + kOffList),
                           reinterpret_cast<int32_t*>(sm + kOffList + kListBytes)};
    uint8_t* list_mask[2] = {sm + kOffList + kMaxList * 4, sm + kOffList + kListBytes + kMaxList * 4};

    if (warp == 4) {
        // ---------------------------------------------------------------- producer
        int32_t* stage = reinterpret_cast<int32_t*>(sm + kOffStage);
        int it = 0, gp = 0;
        uint32_t q_issued = 0;
        int last_phase[2] = {-1, -1};
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
                        list_mask[lb][n - 1] |= (uint8_t)msk;
                    } else if (n < kMaxList) {
                        list_id[lb][n] = m;
                        list_mask[lb][n] = (uint8_t)msk;
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
            if (lane == 0 && it >= 1 && !wait_or_abort(&bars.q_empty, (it - 1) & 1, ctx, abort)) stop = 1;
            if (lane == 0 && !stop) {
                mbar_arrive_expect_tx(&bars.q_full, kQBytes);
                const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
                tma_load_3d(sm + kOffQ, &tmQ, &bars.q_full, 0, i0, z);
                tma_load_3d(sm + kOffQ + kQBytes / 2, &tmQ, &bars.q_full, 64, i0, z);
                q_issued = it + 1;
                for (int u = 0; u < n; u += 2, ++gp) {
                    const int s = gp & 1, r = gp >> 1;
                    if (r >= 1 && !wait_or_abort(&bars.kv_empty[s], (r - 1) & 1, ctx, abort)) break;
                    const int nb = min(2, n - u);
                    uint8_t* st = sm + kOffKV + s * kPairBytes;
                    mbar_arrive_expect_tx(&bars.kv_full[s], nb * 4 * kHalfK);
                    for (int e = 0; e < nb; ++e) {
                        const int y = list_id[lb][u + e] * kBlk;
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
        if (lane == 0) {
            if (q_issued) (void)mbar_wait(&bars.q_full, (q_issued - 1) & 1, ctx);
            for (int s = 0; s < 2; ++s)
                if (last_phase[s] >= 0) (void)mbar_wait(&bars.kv_full[s], last_phase[s] & 1, ctx);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS2 = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idS1 = idesc_bf16_f32(128, 64, false, false);
            const uint32_t idPV = idesc_bf16_f32(128, kD, false, true);
            const uint32_t q0 = smem_u32(sm + kOffQ);
            int it = 0, gp = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++it) {
                const int lb = it & 1;
                ok = wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort);
                if (!ok) break;
                const int n = bars.list_n[lb];
                const int np = (n + 1) >> 1;
                mbar_arrive(&bars.list_empty[lb]);
                ok = wait_or_abort(&bars.q_full, it & 1, ctx, abort);
                if (!ok) break;
                tc_fence_after();
                auto issue_s = [&](int j, int g) -> bool {
                    const int s = g & 1;
                    if (!wait_or_abort(&bars.kv_full[s], (g >> 1) & 1, ctx, abort)) return false;
                    tc_fence_after();
                    const uint32_t kb = smem_u32(sm + kOffKV + s * kPairBytes);
                    const uint32_t dS = tmem + kColS0 + s * 128;
                    const uint32_t id = (2 * j + 1 < n) ? idS2 : idS1;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint64_t a = sdesc_sw128(q0 + (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32, 16, 1024);
                        const uint64_t b = sdesc_sw128(kb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 32, 16, 1024);
                        mma_ss(dS, a, b, id, ks > 0);
                    }
                    mma_commit(&bars.s_full[s]);
                    return true;
                };
                if (np > 0) ok = issue_s(0, gp);
                for (int j = 0; j < np && ok; ++j) {
                    const int g = gp + j;
                    if (j + 1 < np) {
                        ok = issue_s(j + 1, g + 1);
                        if (!ok) break;
                    } else {
                        mma_commit(&bars.q_empty);  // every S MMA of the tile has been issued
                    }
                    ok = wait_or_abort(&bars.p_full[g & 1], (g >> 1) & 1, ctx, abort);
                    if (!ok) break;
                    tc_fence_after();
                    const int s = g & 1;
                    const uint32_t vb = smem_u32(sm + kOffKV + s * kPairBytes + 4 * kHalfK);
                    const uint32_t aP = tmem + kColS0 + s * 128;
                    const int ksteps = (2 * j + 1 < n) ? 8 : 4;
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const uint64_t b = sdesc_sw128(vb + (ks >> 2) * 2 * kHalfK + (ks & 3) * 16 * 128, kHalfK, 1024);
                        mma_ts(tmem + kColO, aP + ks * 8, b, idPV, (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars.kv_empty[s]);
                    mma_commit(&bars.pv_done[s]);
                }
                if (np == 0) mma_commit(&bars.q_empty);
                gp += np;
            }
            mma_commit(&bars.fin);
            (void)mbar_wait(&bars.fin, 0, ctx);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int r = tid;
        const int t = r % kTQ, hh = r / kTQ;
        const uint32_t lane_base = tmem_lane_base(warp);
        int it = 0, gp = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort)) break;
            const int n = bars.list_n[lb];
            const int np = (n + 1) >> 1;
            const int64_t bg = tile / tiles_per_seq;
            const int i0 = (tile % tiles_per_seq) * kTQ;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            float m_run = -INFINITY, l = 0.f;  // m_run in scaled log2 units
            bool ok = true;
            for (int j = 0; j < np; ++j) {
                const int g = gp + j, s = g & 1;
                const bool two = 2 * j + 1 < n;
                const int blk_a = list_id[lb][2 * j];
                const int blk_b = two ? list_id[lb][2 * j + 1] : -1;
                const bool sel_a = (list_mask[lb][2 * j] >> t) & 1;
                const bool sel_b = two && ((list_mask[lb][2 * j + 1] >> t) & 1);
                // last visible key of each half (-1: none)
                const int lim_a = !sel_a ? -1 : (blk_a == c ? i - blk_a * kBlk : kBlk - 1);
                const int lim_b = !sel_b ? -1 : (blk_b == c ? i - blk_b * kBlk : kBlk - 1);
                if (!wait_or_abort(&bars.s_full[s], (g >> 1) & 1, ctx, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t colS = tmem + lane_base + kColS0 + s * 128;
                uint32_t xa[64], xb[64];
                tmem_ld32(colS, *reinterpret_cast<uint32_t(*)[32]>(&xa[0]));
                tmem_ld32(colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&xa[32]));
                if (two) {
                    tmem_ld32(colS + 64, *reinterpret_cast<uint32_t(*)[32]>(&xb[0]));
                    tmem_ld32(colS + 96, *reinterpret_cast<uint32_t(*)[32]>(&xb[32]));
                }
                tmem_ld_wait();
                // Row max in raw units over the visible keys (diagonal block: masked first).
                if (lim_a >= 0 && lim_a < kBlk - 1)
#pragma unroll
                    for (int jj = 0; jj < 64; ++jj) xa[jj] = jj <= lim_a ? xa[jj] : __float_as_uint(-INFINITY);
                if (lim_b >= 0 && lim_b < kBlk - 1)
#pragma unroll
                    for (int jj = 0; jj < 64; ++jj) xb[jj] = jj <= lim_b ? xb[jj] : __float_as_uint(-INFINITY);
                float mx = -INFINITY;
                if (lim_a >= 0) mx = max64(xa);
                if (lim_b >= 0) mx = fmaxf(mx, max64(xb));
                mx *= sl2;
                const bool grow = mx > m_run + 8.f;
                const bool need_rescale = grow && l > 0.f;
                if (__any_sync(0xffffffffu, need_rescale)) {
                    if (j >= 1) {
                        const int gq = g - 1;
                        if (!wait_or_abort(&bars.pv_done[gq & 1], (gq >> 1) & 1, ctx, abort)) { ok = false; break; }
                    }
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
                if (grow) {
                    l = (m_run == -INFINITY) ? 0.f : l * ex2(m_run - mx);
                    m_run = mx;
                }
                uint32_t pk[64];
                float ps = 0.f;
                if (lim_a >= 0) {
                    ps += exp_half(xa, sl2, -m_run, lim_a, pk);
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) pk[q] = 0u;
                }
                if (two) {
                    if (lim_b >= 0) {
                        ps += exp_half(xb, sl2, -m_run, lim_b, pk + 32);
                    } else {
#pragma unroll
                        for (int q = 32; q < 64; ++q) pk[q] = 0u;
                    }
                }
                l += ps;
                tmem_st16(colS, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                tmem_st16(colS + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                if (two) {
                    tmem_st16(colS + 32, *reinterpret_cast<uint32_t(*)[16]>(&pk[32]));
                    tmem_st16(colS + 48, *reinterpret_cast<uint32_t(*)[16]>(&pk[48]));
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[s]);
            }
            if (!ok) break;
            const int64_t orow = (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
            if (np > 0) {
                const int gl = gp + np - 1;
                if (!wait_or_abort(&bars.pv_done[gl & 1], (gl >> 1) & 1, ctx, abort)) break;
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < kD; c0 += 32) {
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
            } else if (i < N) {
                uint4* d4 = reinterpret_cast<uint4*>(out + orow);
                for (int q = 0; q < kD / 8; ++q) d4[q] = make_uint4(0, 0, 0, 0);
            }
            gp += np;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (tid == 0) mbar_arrive(&bars.list_empty[lb]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
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
    const int tiles_per_seq = (N + kTQ - 1) / kTQ;
    const int n_tiles = tiles_per_seq * B * Hkv;
    const int grid = n_tiles < num_sms ? n_tiles : num_sms;
    const float sl2 = scale * 1.4426950408889634f;
    sparse_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), H, Hkv, N, slots, sl2, n_tiles, ctx);
    return cudaGetLastError();
}

}  // namespace sala
