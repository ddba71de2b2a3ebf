// Block-sparse softmax attention prefill on the 5th-generation tensor cores (sm_100a).
//
// Work unit ("tile"): 8 consecutive query tokens x the 16 query heads of one KV group = 128 rows,
// the M of one tcgen05 MMA.  Row r = head * 8 + token, so each head's 8 tokens are one 1024-byte
// swizzle atom and the Q tile arrives with a single 3-D TMA box per 64 columns.  The 8 tokens
// share their query block (8 divides 64), hence the forced blocks and the diagonal; their
// top-k choices differ, so the tile walks the UNION of the 8 selections (ascending) and each
// row masks the blocks its token did not choose.  Executed FLOPs exceed the algorithmic ones by
// the union overhead; the sum over the selected keys of each row is exact.
//
// Per union block u (64 keys of the group's K/V, one TMA box per 64 columns):
//   S_u  = Q K_u^T            M=128 N=64  K=128, A and B from shared memory -> TMEM (fp32)
//   P_u  = online softmax of S_u, rows masked by selection and causality      (registers)
//   O   += P_u V_u            M=128 N=128 K=64,  A = P_u from TMEM (bf16, aliasing S_u), B = V
// S is double-buffered in TMEM so S_{u+1} runs on the tensor core while the softmax warps
// process S_u.  O is rescaled only when a row's running max grows by more than 2^8 (the stale
// max keeps exp2 below 256, far from overflow, and cancels in O / l).
//
// Roles (192 threads, persistent: one CTA per SM walks tiles blockIdx.x, +gridDim.x, ...):
// warps 0-3 softmax + epilogue (thread = row = TMEM lane); warp 4 builds the next tile's union
// list and issues the TMA loads; warp 5 allocates TMEM and issues the MMAs (one thread).
// Every wait is bounded; a timeout sets the status word, the roles wind down, and the kernel
// waits (bounded) for its own copies and MMAs before it frees TMEM and returns.
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
constexpr int kStages = 3;       // K/V pipeline depth
constexpr int kMaxList = 1024;   // union capacity (8 x slots, slots <= 128)
constexpr int kThreads = 192;

// Shared memory layout (offsets from a 1024-aligned base).
constexpr int kQBytes = 128 * kD * 2;                 // 32 KiB: 2 sub-tiles [128 x 128 B]
constexpr int kKBytes = kBlk * kD * 2;                // 16 KiB: 2 sub-tiles [64 x 128 B]
constexpr int kVBytes = kBlk * kD * 2;                // 16 KiB: 2 sub-tiles [64 x 128 B]
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kStageBytes = kKBytes + kVBytes;
constexpr int kOffList = kOffKV + kStages * kStageBytes;   // 2 x kMaxList int32 + 2 x kMaxList u8
constexpr int kListBytes = kMaxList * 5;
constexpr int kSmemBytes = kOffList + 2 * kListBytes + 1024;

// TMEM columns: O [0,128), S buffers [128,192) and [192,256).
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0, kColS0 = 128;

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t kv_full[kStages], kv_empty[kStages];
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

__global__ void __launch_bounds__(kThreads, 1)
sparse_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out, int H,
                         int Hkv, int N, int slots, float scale_log2, int n_tiles, DevCtx ctx) {
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
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
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
        int it = 0;     // tile iteration of this CTA
        int gblk = 0;   // global block counter (pipeline position)
        uint32_t q_issued = 0;
        int last_phase[kStages];
        for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            const int lb = it & 1;
            if (it >= 2 && !wait_or_abort(&bars.list_empty[lb], ((it - 2) >> 1) & 1, ctx, abort)) break;
            const int64_t bg = tile / tiles_per_seq;
            const int i0 = (tile % tiles_per_seq) * kTQ;
            const int c = i0 / kBlk;
            // Union of the (up to) 8 tokens' ascending selections: 8-way merge, one lane per token.
            const int32_t* row = idx + (bg * N + i0 + lane) * (int64_t)slots;
            const bool active = lane < kTQ && i0 + lane < N;
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
                if (m > c) {  // a block in the future of every token of the tile
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
                mbar_arrive(&bars.list_full[lb]);  // release: list writes precede the arrive
            }
            __syncwarp();
            if (lane == 0) {
                // Q tile: 16 heads x 8 tokens x 128 columns (two boxes of 64 columns).
                if (it >= 1 && !wait_or_abort(&bars.q_empty, (it - 1) & 1, ctx, abort)) break;
                mbar_arrive_expect_tx(&bars.q_full, kQBytes);
                const int z = (int)((bg / Hkv) * H + (bg % Hkv) * kG);
                tma_load_3d(sm + kOffQ, &tmQ, &bars.q_full, 0, i0, z);
                tma_load_3d(sm + kOffQ + kQBytes / 2, &tmQ, &bars.q_full, 64, i0, z);
                q_issued = it + 1;
                for (int u = 0; u < n; ++u, ++gblk) {
                    const int s = gblk % kStages;
                    const int r = gblk / kStages;
                    if (r >= 1 && !wait_or_abort(&bars.kv_empty[s], (r - 1) & 1, ctx, abort)) break;
                    const int blk = list_id[lb][u];
                    uint8_t* st = sm + kOffKV + s * kStageBytes;
                    mbar_arrive_expect_tx(&bars.kv_full[s], kStageBytes);
                    tma_load_3d(st, &tmK, &bars.kv_full[s], 0, blk * kBlk, (int)bg);
                    tma_load_3d(st + kKBytes / 2, &tmK, &bars.kv_full[s], 64, blk * kBlk, (int)bg);
                    tma_load_3d(st + kKBytes, &tmV, &bars.kv_full[s], 0, blk * kBlk, (int)bg);
                    tma_load_3d(st + kKBytes + kVBytes / 2, &tmV, &bars.kv_full[s], 64, blk * kBlk, (int)bg);
                    last_phase[s] = r;
                }
            }
            gblk = __shfl_sync(0xffffffffu, gblk, 0);
            if (*abort) break;
        }
        // Wind down: wait (bounded) for every copy this warp issued.
        if (lane == 0) {
            if (q_issued) (void)mbar_wait(&bars.q_full, (q_issued - 1) & 1, ctx);
            for (int s = 0; s < kStages; ++s)
                if (last_phase[s] >= 0) (void)mbar_wait(&bars.kv_full[s], last_phase[s] & 1, ctx);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, kBlk, false, false);
            const uint32_t idPV = idesc_bf16_f32(128, kD, false, true);
            const uint32_t q0 = smem_u32(sm + kOffQ);
            int it = 0, gblk = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++it) {
                const int lb = it & 1;
                ok = wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort);
                if (!ok) break;
                const int n = bars.list_n[lb];
                mbar_arrive(&bars.list_empty[lb]);
                ok = wait_or_abort(&bars.q_full, it & 1, ctx, abort);
                if (!ok) break;
                tc_fence_after();
                auto issue_s = [&](int g) -> bool {
                    const int s = g % kStages;
                    if (!wait_or_abort(&bars.kv_full[s], (g / kStages) & 1, ctx, abort)) return false;
                    tc_fence_after();
                    const uint32_t kb = smem_u32(sm + kOffKV + s * kStageBytes);
                    const uint32_t dS = tmem + kColS0 + (g & 1) * 64;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint64_t a = sdesc_sw128(q0 + (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32, 16, 1024);
                        const uint64_t b = sdesc_sw128(kb + (ks >> 2) * (kKBytes / 2) + (ks & 3) * 32, 16, 1024);
                        mma_ss(dS, a, b, idS, ks > 0);
                    }
                    mma_commit(&bars.s_full[g & 1]);
                    return true;
                };
                if (n > 0) ok = issue_s(gblk);
                for (int u = 0; u < n && ok; ++u) {
                    const int g = gblk + u;
                    if (u + 1 < n) {
                        ok = issue_s(g + 1);
                        if (!ok) break;
                    } else {
                        mma_commit(&bars.q_empty);  // every S MMA of the tile has been issued
                    }
                    ok = wait_or_abort(&bars.p_full[g & 1], (g >> 1) & 1, ctx, abort);
                    if (!ok) break;
                    tc_fence_after();
                    const int s = g % kStages;
                    const uint32_t vb = smem_u32(sm + kOffKV + s * kStageBytes + kKBytes);
                    const uint32_t aP = tmem + kColS0 + (g & 1) * 64;
#pragma unroll
                    for (int ks = 0; ks < kBlk / 16; ++ks) {
                        const uint64_t b = sdesc_sw128(vb + ks * 16 * 128, kVBytes / 2, 1024);
                        mma_ts(tmem + kColO, aP + ks * 8, b, idPV, (u > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars.kv_empty[s]);
                    mma_commit(&bars.pv_done[g & 1]);
                }
                if (n == 0) mma_commit(&bars.q_empty);
                gblk += n;
            }
            // Drain: every MMA this thread issued has completed before TMEM is released.
            mma_commit(&bars.fin);
            (void)mbar_wait(&bars.fin, 0, ctx);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int r = tid;                  // row = TMEM lane
        const int t = r % kTQ, hh = r / kTQ;
        const uint32_t lane_base = tmem_lane_base(warp);
        int it = 0, gblk = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            const int lb = it & 1;
            if (!wait_or_abort(&bars.list_full[lb], (it >> 1) & 1, ctx, abort)) break;
            const int n = bars.list_n[lb];
            const int64_t bg = tile / tiles_per_seq;
            const int i0 = (tile % tiles_per_seq) * kTQ;
            const int c = i0 / kBlk;
            const int i = i0 + t;
            float m_run = -INFINITY, l = 0.f;
            bool o_live = false;  // O holds an accumulated value for this tile
            bool ok = true;
            for (int u = 0; u < n; ++u) {
                const int g = gblk + u;
                const int blk = list_id[lb][u];
                const bool sel = (list_mask[lb][u] >> t) & 1;
                if (!wait_or_abort(&bars.s_full[g & 1], (g >> 1) & 1, ctx, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t colS = tmem + lane_base + kColS0 + (g & 1) * 64;
                uint32_t sr[64];
                tmem_ld32(colS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_ld_wait();
                const int lim = (blk == c) ? (i - blk * kBlk) : (kBlk - 1);  // last visible key
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    float x = __uint_as_float(sr[j]) * scale_log2;
                    x = (sel && j <= lim) ? x : -INFINITY;
                    sr[j] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
                // Stale-max online softmax: rescale only when the max grows by more than 8.
                const bool grow = mx > m_run + 8.f;
                const bool need_rescale = grow && o_live && l > 0.f;
                if (__any_sync(0xffffffffu, need_rescale)) {
                    if (u >= 1) {
                        const int gp = g - 1;
                        if (!wait_or_abort(&bars.pv_done[gp & 1], (gp >> 1) & 1, ctx, abort)) { ok = false; break; }
                    }
                    tc_fence_after();
                    const float alpha = need_rescale ? ex2(m_run - mx) : 1.f;
#pragma unroll 1
                    for (int c0 = 0; c0 < kD; c0 += 32) {
                        uint32_t orr[32];
                        tmem_ld32(tmem + lane_base + kColO + c0, orr);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
                        tmem_st16(tmem + lane_base + kColO + c0, *reinterpret_cast<uint32_t(*)[16]>(&orr[0]));
                        tmem_st16(tmem + lane_base + kColO + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&orr[16]));
                    }
                    tmem_st_wait();
                }
                if (grow) {
                    l = (m_run == -INFINITY) ? 0.f : l * ex2(m_run - mx);
                    m_run = mx;
                }
                uint32_t pk[32];
                float ps = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x0 = __uint_as_float(sr[2 * j]), x1 = __uint_as_float(sr[2 * j + 1]);
                    const float p0 = (x0 == -INFINITY) ? 0.f : ex2(x0 - m_run);
                    const float p1 = (x1 == -INFINITY) ? 0.f : ex2(x1 - m_run);
                    ps += p0 + p1;
                    pk[j] = pack_bf16x2(p0, p1);
                }
                l += ps;
                o_live = true;
                tmem_st16(colS, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                tmem_st16(colS + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[g & 1]);
            }
            if (!ok) break;
            // Epilogue: O / l -> bf16 -> global.
            if (n > 0) {
                const int gl = gblk + n - 1;
                if (!wait_or_abort(&bars.pv_done[gl & 1], (gl >> 1) & 1, ctx, abort)) break;
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                __nv_bfloat16* dst = out + (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
#pragma unroll 1
                for (int c0 = 0; c0 < kD; c0 += 32) {
                    uint32_t orr[32];
                    tmem_ld32(tmem + lane_base + kColO + c0, orr);
                    tmem_ld_wait();
                    if (i < N) {
                        uint4 w[4];
                        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            wp[j] = pack_bf16x2(__uint_as_float(orr[2 * j]) * inv,
                                                __uint_as_float(orr[2 * j + 1]) * inv);
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
                        for (int j = 0; j < 4; ++j) d4[j] = w[j];
                    }
                }
                tc_fence_before();
            } else if (i < N) {
                __nv_bfloat16* dst = out + (((bg / Hkv) * H + (bg % Hkv) * kG + hh) * (int64_t)N + i) * kD;
                for (int j = 0; j < kD; ++j) dst[j] = __float2bfloat16_rn(0.f);
            }
            gblk += n;
            // All four softmax warps are done with this list and with O.
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
    if (d != kD || H != Hkv * kG || slots > kMaxList / kTQ) return cudaErrorNotSupported;
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
    cudaError_t e = cudaFuncSetAttribute(sparse_prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles_per_seq = (N + kTQ - 1) / kTQ;
    const int n_tiles = tiles_per_seq * B * Hkv;
    const int grid = n_tiles < num_sms ? n_tiles : num_sms;
    const float scale_log2 = scale * 1.4426950408889634f;
    sparse_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(
        tmQ, tmK, tmV, idx, static_cast<__nv_bfloat16*>(o), H, Hkv, N, slots, scale_log2, n_tiles,
        ctx);
    return cudaGetLastError();
}

}  // namespace sala
