// Block-sparse softmax attention prefill on the 5th-generation tensor cores (sm_100a).
//
// Work unit: 16 consecutive query tokens of one KV group, split into two tiles A (tokens 0-7) and
// B (tokens 8-15) of 128 rows each (row = head * 8 + token, the 16 query heads of the group), the
// M of one tcgen05 MMA.  The 16 tokens share their query block (16 divides 64), hence the forced
// blocks and the diagonal; their top-k choices differ, so the unit walks the UNION of the 16
// selections (ascending).  K and V of each union block are loaded once for both tiles; a tile none
// of whose 8 tokens chose the block skips it, and each row masks the blocks its own token did not
// choose, so a row's sum runs over exactly its selected keys.
//
// Per block b and active tile X:
//   S_X  = Q_X K_b^T      M=128 N=64 K=128   (Q_X and K_b from shared memory)
//   P_X  = online softmax of S_X (selection mask per row, causal mask on the diagonal block)
//   O_X += P_X V_b        M=128 N=128 K=64   (A = P_X from TMEM, aliasing S_X; B = V_b)
// Each tile's MMAs come from its own issuing thread, and each tile has two S buffers in TMEM, so
// the S of the tile's next block runs while its softmax works on this one: per tile the chain is
// softmax -> PV, and the two tiles' chains overlap each other's MMAs (the ping-pong
// FlashAttention-4 uses on this architecture).  O_X is rescaled only when a row's running max
// grows by more than 8 in log2 units (the stale max keeps exp2 below 256 and cancels in O / l).
//
// Shared memory holds the unit's two Q tiles and a ring of four 32 KiB stages, each the K and V
// of one block, loaded by TMA up to four blocks ahead.
//
// Roles (384 threads, persistent: one CTA per SM walks units blockIdx.x, +gridDim.x, ...):
// warps 0-3 softmax + epilogue of tile A, warps 4-7 of tile B (thread = row = TMEM lane); warp 11
// stages the next unit's 16 selection rows and merges them into its union list (double-buffered,
// one unit ahead); warp 8 issues the TMA loads (Q tiles, then the ring); warp 9 allocates TMEM and
// issues the MMAs of tile A, warp 10 those of tile B (one elected lane of each converged warp).
// Every wait is bounded; a timeout sets the status word, the roles wind down, and the kernel waits
// (bounded) for its own copies and MMAs before it frees TMEM.
//
// Per-head selections (kPerHead: idx is [B, H, N, slots], one row per query head and token): the
// unit's union is over its 16 heads x 16 tokens.  The list warp sets one bit per chosen block in
// two bitmaps (tile A's rows, tile B's rows), and every role walks the set bits of their OR in
// ascending order; a tile skips the blocks its bitmap lacks, and each softmax thread decides its
// row's mask by walking its own (ascending) selection row alongside the union.
#include <climits>

#include "fastexp.cuh"
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
constexpr int kStages = 4;

// Shared memory (offsets from a 1024-aligned base): Q_A, Q_B (two [128 x 128 B] halves each,
// d 0-63 and d 64-127), then the ring; a stage holds K_b (two [64 x 128 B] halves) then V_b.
constexpr int kQBytes = 32768;
constexpr int kHalfQ = 16384;                         // one [128 rows x 128 B] box
constexpr int kStageBytes = 32768;
constexpr int kHalfBlk = 8192;                        // one [64 rows x 128 B] box
constexpr int kOffRing = 2 * kQBytes;
constexpr int kOffList = kOffRing + kStages * kStageBytes;
constexpr int kListBytes = kMaxList * 6;              // int32 ids + uint16 token masks
constexpr int kOffStage = kOffList + 2 * kListBytes;  // staged selection rows of one unit
constexpr int kSmemBytes = kOffStage + kUT * kMaxSlots * 4 + 1024;
// Per-head mode keeps, in the list area, two bitmaps (tiles A, B) per list buffer over the
// candidate blocks 0 .. c of the unit: up to 2^14 blocks, i.e. N <= 2^20.
constexpr int kMaxBmWords = 512;
static_assert(4 * kMaxBmWords * 4 <= 2 * kListBytes, "bitmaps exceed the list area");

// TMEM columns: O_A [0,128), O_B [128,256), S_A two buffers [256,384), S_B two buffers [384,512).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;

struct Bars {
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2][2], p_full[2][2], pv_done[2][2];  // per tile and S buffer
    uint64_t q_full, q_empty;
    uint64_t list_full[2], list_empty[2];
    uint64_t fin[2];
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
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (!mbar_wait(bar, parity, ctx)) {
        *abort = 1;
        return false;
    }
    return true;
}

__device__ __forceinline__ uint32_t (&sub32(uint32_t (&a)[64], int k))[32] {
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

// Which key pairs take the FMA-pipe exp2 instead of the multi-function unit (ex2.approx): one pair
// in kPolyEvery, outside the diagonal block.  Per block both tiles' softmax warps on a scheduler
// need 16384 exponentials, 1024 cycles of the multi-function unit at 16 per cycle, as long as the
// block's MMAs; moving a quarter to the FMA pipe takes that unit off the critical path.
constexpr int kPolyEvery = 4;

// p = 2^(s * sl2 + nb) for 64 keys, packed to 32 bf16 pairs and stored to TMEM columns
// taddr .. taddr+31 in two pieces of 16; sums added to a0..a3.  kMasked zeroes the keys past lim
// (the causal edge) and uses ex2.approx throughout, so masked keys give exact zeros.  kTrain (the
// training forward) takes every key through ex2.approx, as the backward recomputes P, and stores
// the bf16 rounding residual p - bf16(p) to columns taddr+32 .. taddr+63 (the S values there are
// already in registers), so P V can be taken as P_hi V + P_lo V.
template <bool kMasked, bool kTrain>
__device__ __forceinline__ void exp_block(const uint32_t* s, float sl2, float nb, int lim,
                                          uint32_t taddr, float& a0, float& a1, float& a2,
                                          float& a3) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t pk[16], lo[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int k = 32 * h + 2 * q;
            float y0, y1;
            fma2_bcast(y0, y1, __uint_as_float(s[k]), __uint_as_float(s[k + 1]), sl2, nb);
            float p0, p1;
            if (!kMasked && !kTrain && q % kPolyEvery == kPolyEvery - 1) {
                p0 = y0;
                p1 = y1;
                exp2_poly2(p0, p1);
            } else {
                p0 = ex2(y0);
                p1 = ex2(y1);
            }
            if (kMasked) {
                p0 = k <= lim ? p0 : 0.f;
                p1 = k + 1 <= lim ? p1 : 0.f;
            }
            if (q & 1) add2(a2, a3, p0, p1);
            else add2(a0, a1, p0, p1);
            pk[q] = pack_bf16x2(p0, p1);
            if (kTrain)
                lo[q] = pack_bf16x2(p0 - __uint_as_float(pk[q] << 16),
                                    p1 - __uint_as_float(pk[q] & 0xffff0000u));
        }
        tmem_st16(taddr + 16 * h, pk);
        if (kTrain) tmem_st16(taddr + 32 + 16 * h, lo);
    }
}

// A unit's union in ascending block order.  Group selections: the list of (block, 16-bit token
// mask) entries.  Per-head selections: the set bits of bitmap A | bitmap B over words 0 .. nw-1,
// with m = bit 0 (a row of tile A chose the block) | bit 1 (a row of tile B did).
template <bool kPerHead>
struct UnionWalk {
    const int32_t* ids;
    const uint16_t* msks;
    const uint32_t* bm_a;
    const uint32_t* bm_b;
    int pos, w, nw;
    uint32_t bits;
    __device__ __forceinline__ void next(int& blk, uint32_t& m) {
        if constexpr (!kPerHead) {
            blk = ids[pos];
            m = msks[pos];
            ++pos;
        } else {
            while (bits == 0u && w + 1 < nw) {
                ++w;
                bits = bm_a[w] | bm_b[w];
            }
            const int bit = __ffs((int)bits) - 1;  // callers take exactly the counted entries
            bits &= bits - 1u;
            blk = w * 32 + bit;
            m = ((bm_a[w] >> bit) & 1u) | (((bm_b[w] >> bit) & 1u) << 1);
        }
    }
    // Whether some row of tile x chose the block.
    __device__ __forceinline__ static bool tile_active(uint32_t m, int x) {
        if constexpr (kPerHead) return (m >> x) & 1u;
        else return ((m >> (8 * x)) & 0xffu) != 0u;
    }
};

template <bool kTrain, bool kPerHead>
__global__ void __launch_bounds__(kThreads, 1)
sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out,
                         float* __restrict__ lse, __nv_bfloat16* __restrict__ out_lo, int H,
                         int Hkv, int N, int slots, float sl2,
                         int n_units, DevCtx ctx) {
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
            mbar_init(&bars.kv_empty[s], 2);  // released by both MMA issuers
        }
        for (int b = 0; b < 2; ++b) {
            for (int j = 0; j < 2; ++j) {
                mbar_init(&bars.s_full[b][j], 1);
                mbar_init(&bars.p_full[b][j], 4);
                mbar_init(&bars.pv_done[b][j], 1);
            }
            mbar_init(&bars.list_full[b], 1);
            mbar_init(&bars.list_empty[b], 4);  // producer, both issuers, softmax
            mbar_init(&bars.fin[b], 1);
        }
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_empty, 2);  // both MMA issuers
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
    auto bitmap = [&](int lb, int x) {
        return reinterpret_cast<uint32_t*>(sm + kOffList + (lb * 2 + x) * kMaxBmWords * 4);
    };
    // The union of list buffer lb for a unit whose tokens lie in query block c.
    auto walk = [&](int lb, int c) {
        UnionWalk<kPerHead> u;
        u.ids = list_id(lb);
        u.msks = list_mask(lb);
        u.bm_a = bitmap(lb, 0);
        u.bm_b = bitmap(lb, 1);
        u.pos = 0;
        u.w = -1;
        u.nw = c / 32 + 1;
        u.bits = 0u;
        return u;
    };
    // Ring entry e lives in stage e % kStages and is that stage's use number e / kStages.
    auto stage_ptr = [&](uint32_t e) { return sm + kOffRing + (e % kStages) * kStageBytes; };
    auto full_bar = [&](uint32_t e) { return &bars.kv_full[e % kStages]; };
    auto empty_bar = [&](uint32_t e) { return &bars.kv_empty[e % kStages]; };
    auto round_of = [](uint32_t e) { return (e / kStages) & 1u; };

    if (warp == 11) {
        // ---------------------------------------------------------------- union lists
        // Builds unit u+1's union list (double-buffered) while unit u is being consumed, so the
        // producer never stalls the ring on it: the unit's 16 selection rows (contiguous in
        // memory) are staged with all loads in flight, then merged.
        int it = 0;
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            if (it >= 2 && !wait_or_abort(&bars.list_empty[lb], ((it - 2) >> 1) & 1, ctx, abort)) break;
            const int64_t bg = unit / units_per_seq;
            const int i0 = (unit % units_per_seq) * kUT;
            const int c = i0 / kBlk;
            const int n_act = min(kUT, N - i0);
            const int total = n_act * slots;
            int n = 0;
            if constexpr (!kPerHead) {
                int32_t* stage = reinterpret_cast<int32_t*>(sm + kOffStage);
                const int32_t* src = idx + (bg * N + i0) * (int64_t)slots;
                {
                    constexpr int kPer = kMaxList / 32;  // entries per lane at most
                    int32_t v[kPer];
#pragma unroll
                    for (int j = 0; j < kPer; ++j) {
                        const int e = lane + 32 * j;
                        v[j] = e < total ? __ldg(src + e) : -1;
                    }
#pragma unroll
                    for (int j = 0; j < kPer; ++j) {
                        const int e = lane + 32 * j;
                        if (e < total && in_bounds(ctx, e < kUT * kMaxSlots)) stage[e] = v[j];
                    }
                }
                __syncwarp();
                // 16-way merge of the ascending rows, one lane per token.
                const int32_t* row = stage + lane * slots;
                const bool active = lane < n_act;
                int p = 0, prev = -1;
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
                            if (in_bounds(ctx, n >= 1 && n <= kMaxList)) list_mask(lb)[n - 1] |= (uint16_t)msk;
                        } else if (n < kMaxList) {
                            list_id(lb)[n] = m;
                            list_mask(lb)[n] = (uint16_t)msk;
                            ++n;
                        }
                    }
                    n = __shfl_sync(0xffffffffu, n, 0);
                    prev = m;
                }
            } else {
                // Per-head rows: the unit's 16 heads, each a run of n_act rows of slots entries;
                // entries of the first 8 tokens go to tile A's bitmap, the rest to tile B's.
                uint32_t* bm_a = bitmap(lb, 0);
                uint32_t* bm_b = bitmap(lb, 1);
                const int nw = c / 32 + 1;
                for (int w = lane; w < nw; w += 32) {
                    bm_a[w] = 0u;
                    bm_b[w] = 0u;
                }
                __syncwarp();
                const int split = kTQ * slots;
                bool bad = false;
                constexpr int kPer = kMaxList / 32;
                for (int h0 = 0; h0 < kG; h0 += 2) {
                    int32_t v[2][kPer];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int64_t head = (bg / Hkv) * H + (bg % Hkv) * kG + h0 + u;
                        const int32_t* src = idx + (head * N + i0) * (int64_t)slots;
#pragma unroll
                        for (int j = 0; j < kPer; ++j) {
                            const int e = lane + 32 * j;
                            v[u][j] = e < total ? __ldg(src + e) : -1;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int j = 0; j < kPer; ++j) {
                            const int m = v[u][j];
                            if (m > c) {  // in the future of every token of the unit
                                bad = true;
                            } else if (m >= 0 && in_bounds(ctx, (m >> 5) < nw && nw <= kMaxBmWords)) {
                                const int e = lane + 32 * j;
                                atomicOr((e < split ? bm_a : bm_b) + (m >> 5), 1u << (m & 31));
                            }
                        }
                }
                if (__any_sync(0xffffffffu, bad) && lane == 0) flag(ctx, kStatusBounds);
                __syncwarp();
                for (int w = lane; w < nw; w += 32) n += __popc(bm_a[w] | bm_b[w]);
                n = __reduce_add_sync(0xffffffffu, n);
                __threadfence_block();  // every lane's bitmap words before lane 0 publishes them
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
        // A unit with a non-empty union loads its Q tiles, then one ring entry per union block;
        // its list buffer goes back to the list warp once the last entry is issued.
        int it = 0;
        uint32_t rc = 0, kq = 0;  // ring entries issued, Q tile pairs issued
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            int stop = 0;
            if (lane == 0) {
                if (!wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort)) stop = 1;
                const int n = stop ? 0 : bars.list_n[lb];
                const int64_t bg = unit / units_per_seq;
                const int i0 = (unit % units_per_seq) * kUT;
                UnionWalk<kPerHead> uw = walk(lb, i0 / kBlk);
                if (n > 0) {
                    // Q_A, Q_B: 16 heads x 8 tokens x 128 columns each, once both issuers are
                    // done with the previous unit's S MMAs.
                    if (kq >= 1 && !wait_or_abort(&bars.q_empty, (kq - 1) & 1, ctx, abort)) stop = 1;
                    if (!stop) {
                        const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
                        mbar_arrive_expect_tx(&bars.q_full, 2 * kQBytes);
                        for (int q = 0; q < 2; ++q) {
                            tma_load_3d(sm + q * kQBytes, &tmQ, &bars.q_full, 0, i0 + q * kTQ, z);
                            tma_load_3d(sm + q * kQBytes + kHalfQ, &tmQ, &bars.q_full, 64, i0 + q * kTQ, z);
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
                        mbar_arrive_expect_tx(fb, kStageBytes);
                        int blk;
                        uint32_t m;
                        uw.next(blk, m);
                        if (!in_bounds(ctx, blk >= 0 && blk <= i0 / kBlk)) blk = 0;  // load a real block
                        const int y = blk * kBlk;
                        tma_load_3d(st, &tmK, fb, 0, y, (int)bg);
                        tma_load_3d(st + kHalfBlk, &tmK, fb, 64, y, (int)bg);
                        tma_load_3d(st + 2 * kHalfBlk, &tmV, fb, 0, y, (int)bg);
                        tma_load_3d(st + 3 * kHalfBlk, &tmV, fb, 64, y, (int)bg);
                    }
                }
                if (!stop) mbar_arrive(&bars.list_empty[lb]);  // done reading the list
            }
            rc = __shfl_sync(0xffffffffu, rc, 0);
            kq = __shfl_sync(0xffffffffu, kq, 0);
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop || *abort) break;
        }
        if (lane == 0) {  // drain: every copy this warp started has landed before the block exits
            if (kq > 0) (void)mbar_wait(&bars.q_full, (kq - 1) & 1, ctx);
            for (uint32_t e = rc > kStages ? rc - kStages : 0; e < rc; ++e)
                (void)mbar_wait(full_bar(e), round_of(e), ctx);
        }
    } else if (warp == 9 || warp == 10) {
        // ---------------------------------------------------------------- MMA issuers
        // Warp 9 issues the MMAs of tile A, warp 10 those of tile B.  The whole warp runs the loop
        // converged with warp-uniform operands and one elected lane issues each instruction (a
        // single-lane branch ran the same loop ~3 % slower).  Two issuers keep the tensor pipe
        // fed and the tiles' chains never wait on each other.
        // Order per tile: S of round k+1 is issued before PV of round k (two S buffers), so the
        // tensor core computes the next S while the softmax works on this one.  Each issuer
        // observes every ring entry in order (so its parity waits never run two uses ahead of a
        // stage) and returns each entry once: after the tile's PV for a block it used, right away
        // for a block it did not.  Before it waits for an entry whose stage still holds a block of
        // its own, it issues that block's PV, so it never holds a stage the producer needs.
        const int x = warp - 9;
        auto wait_w = [&](uint64_t* bar, uint32_t parity) -> bool {  // warp-uniform outcome
            const bool r = wait_or_abort(bar, parity, ctx, abort);
            return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
        };
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        const uint32_t idS = idesc_bf16_f32(128, kBlk, false, false);
        const uint32_t idPV = idesc_bf16_f32(128, kD, false, true);
        const uint32_t dO = tm + kColO + x * 128;
        // Shared-memory descriptors: one high half for every operand here (stride 1024 B, 128-byte
        // swizzle); low halves = address | leading offset, plus the K step.
        const uint64_t dhi = (uint64_t)sdesc_sw128_hi(1024) << 32;
        const uint64_t q_d = dhi | sdesc_sw128_lo(smem_u32(sm + x * kQBytes), 16);
        const uint64_t ring_d = dhi | sdesc_sw128_lo(smem_u32(sm + kOffRing), 16);
        const uint64_t ring_v_d = dhi | sdesc_sw128_lo(smem_u32(sm + kOffRing + 2 * kHalfBlk), kHalfBlk);
        int it = 0;
        uint32_t rc = 0, kq = 0, a = 0;  // ring entries seen, Q tile pairs used, S rounds issued
        bool ok = true;
        for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            ok = wait_w(&bars.list_full[lb], (it >> 1) & 1);
            if (!ok) break;
            const int n = bars.list_n[lb];
            UnionWalk<kPerHead> uw = walk(lb, ((unit % units_per_seq) * kUT) / kBlk);
            if (n > 0) {
                ok = wait_w(&bars.q_full, kq & 1);
                ++kq;
                tc_fence_after();
                // Rounds whose S is issued and whose PV is not: at most two, oldest first.
                int np = 0;
                uint32_t pe0 = 0, pk0 = 0, pe1 = 0, pk1 = 0;  // ring entry, round
                bool accum = false;
                auto flush_pv = [&]() -> bool {
                    const uint32_t e = pe0, k = pk0;
                    pe0 = pe1;
                    pk0 = pk1;
                    --np;
                    if (!wait_w(&bars.p_full[x][k & 1], (k >> 1) & 1)) return false;
                    tc_fence_after();
                    const uint32_t aP = tm + kColS + x * 128 + (k & 1) * 64;
                    const uint64_t v_d = ring_v_d + (e % kStages) * (kStageBytes >> 4);
#pragma unroll
                    for (int ks = 0; ks < kBlk / 16; ++ks)
                        mma_ts_elect(dO, aP + ks * 8, v_d + ((ks * 16 * 128) >> 4), idPV,
                                     (accum || ks > 0) ? 1u : 0u);
                    if constexpr (kTrain) {  // + P_lo V: the residual columns of the same buffer
#pragma unroll
                        for (int ks = 0; ks < kBlk / 16; ++ks)
                            mma_ts_elect(dO, aP + 32 + ks * 8, v_d + ((ks * 16 * 128) >> 4), idPV, 1u);
                    }
                    mma_commit_elect(&bars.pv_done[x][k & 1]);
                    mma_commit_elect(empty_bar(e));
                    accum = true;
                    return true;
                };
                for (int b = 0; b < n && ok; ++b) {
                    const uint32_t e = rc + b;
                    int blk;
                    uint32_t m;
                    uw.next(blk, m);
                    const bool act = UnionWalk<kPerHead>::tile_active(m, x);
                    while (ok && np > 0 && pe0 + kStages <= e) ok = flush_pv();
                    if (ok && np == 2) ok = flush_pv();
                    if (!ok) break;
                    if (!(ok = wait_w(full_bar(e), round_of(e)))) break;
                    if (!act) {  // no token of this tile chose the block
                        mbar_arrive_elect(empty_bar(e));
                        continue;
                    }
                    tc_fence_after();
                    const uint32_t dS = tm + kColS + x * 128 + (a & 1) * 64;
                    const uint64_t k_d = ring_d + (e % kStages) * (kStageBytes >> 4);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_ss_elect(dS, q_d + (((ks >> 2) * kHalfQ + (ks & 3) * 32) >> 4),
                                     k_d + (((ks >> 2) * kHalfBlk + (ks & 3) * 32) >> 4), idS,
                                     ks > 0 ? 1u : 0u);
                    mma_commit_elect(&bars.s_full[x][a & 1]);
                    if (np == 0) {
                        pe0 = e;
                        pk0 = a;
                    } else {
                        pe1 = e;
                        pk1 = a;
                    }
                    ++np;
                    ++a;
                    if (np == 2) ok = flush_pv();
                }
                mma_commit_elect(&bars.q_empty);  // every S MMA reading this unit's Q is issued
                while (ok && np > 0) ok = flush_pv();
                rc += n;
            }
            mbar_arrive_elect(&bars.list_empty[lb]);
        }
        mma_commit_elect(&bars.fin[x]);
        (void)mbar_wait(&bars.fin[x], 0, ctx);
        __syncwarp();
    } else {
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
        const uint32_t colS0 = tmem + lane_base + kColS + x * 128;  // + 64 for the second buffer
        volatile int* sm_stop = &bars.sm_stop;
        int nbar = 0;
        bool dead = false;
        auto fail = [&]() {
            dead = true;
            atomicCAS(&bars.sm_stop, 0, nbar + 1);
            *abort = 1;
        };
        int it = 0;
        uint32_t a = 0;  // rounds of this tile (one per active block), in the issuer's numbering
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!dead && !mbar_wait(&bars.list_full[lb], (it >> 1) & 1, ctx)) fail();
            const int n = dead ? 0 : bars.list_n[lb];
            const int64_t bg = unit / units_per_seq;
            const int i0 = (unit % units_per_seq) * kUT;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            UnionWalk<kPerHead> uw = walk(lb, c);
            // Per-head: this row's own selection, read four entries ahead (own0 is the first entry
            // not below the blocks walked so far; INT_MAX past the row's end).
            const int32_t* own = nullptr;
            int own0 = INT_MAX, own1 = INT_MAX, own2 = INT_MAX, own3 = INT_MAX, own_p = 0;
            if constexpr (kPerHead) {
                if (i < N) {
                    own = idx + (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * slots;
                    own0 = __ldg(own);
                    own1 = slots > 1 ? __ldg(own + 1) : INT_MAX;
                    own2 = slots > 2 ? __ldg(own + 2) : INT_MAX;
                    own3 = slots > 3 ? __ldg(own + 3) : INT_MAX;
                    own_p = 4;
                }
            }
            float m_run = -INFINITY, l = 0.f;  // running max (scaled log2 units), row sum
            int last = -1;
            for (int b = 0; b < n; ++b) {
                int blk;
                uint32_t msk;
                uw.next(blk, msk);
                if (!UnionWalk<kPerHead>::tile_active(msk, x)) continue;  // no row of the tile chose it
                const bool diag = blk == c;                      // uniform over the warpgroup
                bool sel;
                if constexpr (kPerHead) {
                    while (own0 < blk) {  // padding (-1) and blocks the walk has passed
                        own0 = own1;
                        own1 = own2;
                        own2 = own3;
                        own3 = own_p < slots ? __ldg(own + own_p) : INT_MAX;
                        ++own_p;
                    }
                    sel = own0 == blk;
                } else {
                    sel = (msk >> t) & 1u;
                }
                const int lim = !sel ? -1 : (diag ? i - blk * kBlk : kBlk - 1);  // last visible key
                const uint32_t j = a & 1u, colS = colS0 + j * 64;
                if (!dead && !mbar_wait(&bars.s_full[x][j], (a >> 1) & 1u, ctx)) fail();
                tc_fence_after();
                const bool go = !__any_sync(0xffffffffu, dead);
                uint32_t sr[64];
                float mx = -INFINITY;
                if (go) {
                    tmem_ld32(colS, sub32(sr, 0));
                    tmem_ld32(colS + 32, sub32(sr, 1));
                    tmem_ld_wait();
                    mx = diag ? max64_masked(sr, lim) : (lim >= 0 ? max64(sr) : -INFINITY);
                }
                mx *= sl2;
                const bool grow = mx > m_run + 8.f;
                const bool need_rescale = grow && m_run != -INFINITY;
                const float alpha = need_rescale ? ex2(m_run - mx) : 1.f;
                if (grow) {
                    l = (m_run == -INFINITY) ? 0.f : l * alpha;
                    m_run = mx;
                }
                // p = 2^(s * sl2 - m) as bf16 pairs over the first 32 columns of S (already read).
                if (go) {
                    const float nb = lim >= 0 ? -m_run : -INFINITY;
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                    if (diag) exp_block<true, kTrain>(sr, sl2, nb, lim, colS, a0, a1, a2, a3);
                    else exp_block<false, kTrain>(sr, sl2, nb, lim, colS, a0, a1, a2, a3);
                    l += (a0 + a1) + (a2 + a3);
                }
                // Rescale O_x by 2^(m_old - m_new) where the max grew past the threshold (before
                // this thread releases P, so before this block's PV can add into O_x).
                if (go && __any_sync(0xffffffffu, need_rescale)) {
                    if (last >= 0) {  // the tile's previous PV into O_x must be complete
                        if (!dead && !mbar_wait(&bars.pv_done[x][last & 1], ((uint32_t)last >> 1) & 1u, ctx)) fail();
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
                if (lane == 0) mbar_arrive(&bars.p_full[x][j]);
                last = (int)a;
                ++a;
            }
            // Epilogue: O_x / l -> bf16 -> global (zeros when the tile saw no block); with lse,
            // the row's natural log-sum-exp ln(sum_j e^(scale s_j)) = (m_run + log2 l) ln 2; with
            // out_lo, the bf16 rounding residual of each output element.
            const int64_t orow = (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
            if (kTrain && lse != nullptr && i < N && !dead)
                lse[orow / kD] = (last >= 0 && m_run != -INFINITY && l > 0.f)
                                     ? (m_run + log2f(l)) * 0.69314718055994531f
                                     : -INFINITY;
            if (last >= 0) {
                if (!dead && !mbar_wait(&bars.pv_done[x][last & 1], ((uint32_t)last >> 1) & 1u, ctx)) fail();
                if (!__any_sync(0xffffffffu, dead)) {
                    tc_fence_after();
                    // No visible key (m_run = -inf): zeros (masked keys may have added 2^-125 terms).
                    const float inv = (m_run != -INFINITY && l > 0.f) ? 1.f / l : 0.f;
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
                            if (kTrain && out_lo != nullptr) {
#pragma unroll
                                for (int q = 0; q < 16; ++q) {
                                    const float x0 = __uint_as_float(orr[2 * q]) * inv;
                                    const float x1 = __uint_as_float(orr[2 * q + 1]) * inv;
                                    wp[q] = pack_bf16x2(x0 - __uint_as_float(wp[q] << 16),
                                                        x1 - __uint_as_float(wp[q] & 0xffff0000u));
                                }
                                uint4* l4 = reinterpret_cast<uint4*>(out_lo + orow + c0);
#pragma unroll
                                for (int q = 0; q < 4; ++q) l4[q] = w[q];
                            }
                        }
                    }
                    tc_fence_before();
                }
            } else if (i < N && !dead) {
                uint4* d4 = reinterpret_cast<uint4*>(out + orow);
                for (int q = 0; q < kD / 8; ++q) d4[q] = make_uint4(0, 0, 0, 0);
                if (kTrain && out_lo != nullptr) {
                    uint4* l4 = reinterpret_cast<uint4*>(out_lo + orow);
                    for (int q = 0; q < kD / 8; ++q) l4[q] = make_uint4(0, 0, 0, 0);
                }
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

}  // namespace

bool sparse_prefill_tc_supported(int H, int Hkv, int d) {
    return d == kD && Hkv > 0 && H == Hkv * kG;
}

cudaError_t launch_sparse_prefill_tc(const void* q, const void* k, const void* v,
                                     const int32_t* idx, void* o, float* lse, void* o_lo, int B,
                                     int H, int Hkv, int N, int d, int slots, float scale,
                                     bool per_head, cudaStream_t st, DevCtx ctx) {
    if (d != kD || H != Hkv * kG || slots > kMaxSlots) return cudaErrorNotSupported;
    if (per_head && (lse != nullptr || o_lo != nullptr || (N + kBlk - 1) / kBlk > 32 * kMaxBmWords))
        return cudaErrorNotSupported;
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
    const int num_sms = device_sm_count();
    const bool train = lse != nullptr;
    cudaError_t e = train      ? ensure_smem<sparse_prefill_tc_kernel<true, false>>(kSmemBytes)
                    : per_head ? ensure_smem<sparse_prefill_tc_kernel<false, true>>(kSmemBytes)
                               : ensure_smem<sparse_prefill_tc_kernel<false, false>>(kSmemBytes);
    if (e != cudaSuccess) return e;
    const int units_per_seq = (N + kUT - 1) / kUT;
    const int n_units = units_per_seq * B * Hkv;
    const int grid = n_units < num_sms ? n_units : num_sms;
    const float sl2 = scale * 1.4426950408889634f;
    if (train)
        sparse_prefill_tc_kernel<true, false><<<grid, kThreads, kSmemBytes, st>>>(
            tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), lse,
            static_cast<__nv_bfloat16*>(o_lo), H, Hkv, N, slots, sl2, n_units, ctx);
    else if (per_head)
        sparse_prefill_tc_kernel<false, true><<<grid, kThreads, kSmemBytes, st>>>(
            tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), nullptr, nullptr, H, Hkv, N, slots,
            sl2, n_units, ctx);
    else
        sparse_prefill_tc_kernel<false, false><<<grid, kThreads, kSmemBytes, st>>>(
            tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), nullptr, nullptr, H, Hkv, N, slots,
            sl2, n_units, ctx);
    return cudaGetLastError();
}

}  // namespace sala
