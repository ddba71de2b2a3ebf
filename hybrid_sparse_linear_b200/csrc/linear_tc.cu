// Linear (Lightning-style) attention prefill on the 5th-generation tensor cores (sm_100a).
//
//   o_i = sum_{j<=i} lambda^{i-j} (q_i . k_j) v_j + lambda^{i+1} q_i S_in
//
// One CTA owns one (batch, head, 64-wide slice of the value columns): S[:, slice] and
// o[:, slice] depend on no other slice, so the 2 slices of a head run on different SMs and only
// re-read Q and K (which the sibling CTA pulls through L2 at the same time).  The CTA walks the
// sequence in tiles of 128 rows; each tile is two 64-row chunks of the chunked form, with the
// chunk-to-chunk term inside the tile computed directly instead of through the state (the same
// sum, associated differently).  Per tile c (rows t, s in [0, 128), len valid):
//   MMA1  A    = Q_c K_c^T                    M=128 N=128 K=128   (SMEM x SMEM -> TMEM)
//   EPI-A A'   = A * lambda^{t-s} [s <= t]    bf16, written back over A in TMEM
//   MMA2  O1   = A' V_c[:, slice]             M=128 N=64  K=128   (TMEM x SMEM)
//   MMA3  O2   = Q_c Sb                       M=128 N=64  K=128   (Sb = bf16 copy of S_{c-1})
//   EPI-A o_t  = O1_t + lambda^{t+1} O2_t     -> bf16 -> global
//   EPI-S V~   = diag(lambda^{len-1-s}) V_c   bf16 in SMEM (double-buffered)
//   MMA4  dS   = K_c^T V~                     M=128 N=64  K=128   (A read transposed)
//   EPI-S S    = lambda^len S + dS            fp32, one row of S per thread, in registers
// The only serial dependency between tiles is the state: S(c) = lambda^len S(c-1) + dS(c), where
// dS(c) needs no state at all.  The MMA issuer therefore computes dS one tile ahead (into a second
// TMEM buffer): per tile, one thread issues MMA2(c) then MMA1(c+1) and the other MMA3(c) then
// MMA4(c+1); after MMA2(c) and MMA3(c), the last readers of stage c, the stage goes back to the
// producer a full tile before it is needed again, the state warps find dS(c) already done and the
// tensor core always has independent work queued.
// The bf16 state copy is double-buffered: Sb(c) lives in buffer (c+1)&1, MMA3(c) reads Sb(c-1)
// from buffer c&1 and releases it through sb_free[c&1]; with one barrier per buffer no barrier
// can run two phases ahead of its waiter.
// Roles (512 threads): warps 0-3 "EPI-A" (mask + output, thread = row = TMEM lane), warps 4-7
// "EPI-S" (V~ + state, thread = row of S), warp 8 TMA producer (2-stage ring of Q/K/V tiles),
// warp 9 TMEM owner and issuer of MMA1/MMA2, warp 10 issuer of MMA3/MMA4 (one issuing thread
// cannot keep four products per tile in flight), warp 11 idle, warps 12-15 RoPE (with a rotary
// embedding: each stage's Q and K rotated in place, thread = row, before the stage's MMAs).
// Every wait is bounded (see ptx::mbar_wait).
#include "kernels.h"
#include "ptx.cuh"
#include "rope.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

using namespace ptx;

constexpr int kD = 128, kC = 128, kDv = 64, kSlices = kD / kDv;
constexpr int kThreads = 512;
// Register split (setmaxnreg): the mask/output and V~/state warpgroups hold wide TMEM rows; the
// producer/issuer warpgroup and the RoPE warpgroup need little.  256 * 168 + 256 * 88 = 512 * 128,
// the per-thread count the block is launched with.
constexpr int kRegsLaunch = 128, kRegsEpi = 168, kRegsOther = 88;
static_assert(256 * kRegsEpi + 256 * kRegsOther == kThreads * kRegsLaunch, "register split");
constexpr int kSub = kC * 128;                    // one [128 rows x 128 B] sub-tile: 16 KiB
constexpr int kOffQ = 0, kOffK = 2 * kSub, kOffV = 4 * kSub;
constexpr int kStageBytes = 5 * kSub;             // Q (2) + K (2) + V slice (1)
constexpr int kOffVt = 2 * kStageBytes;           // V~ (decay-weighted V slice)
constexpr int kOffSb = kOffVt + kSub;             // bf16 copies of the state slice, 2 buffers
constexpr int kOffOst = kOffSb + 2 * kSub;        // output tile staged for its TMA store
constexpr int kSmemBytes = kOffOst + kSub + 1024;
static_assert(kSmemBytes <= 227 * 1024, "descriptor address fields (14 bits of 16-byte units) must not carry");

constexpr uint32_t kColA0 = 0, kColO1 = 256, kColO2 = 320, kColDS = 384, kTmemCols = 512;  // dS: 2 x 64

struct Bars {
    uint64_t full[2], empty[2];
    uint64_t qk_done[2], a_ready[2], v_ready[2], ds_done[2], s_ready[2], sb_free[2];
    uint64_t rot_ready[2];  // RoPE: Q and K of the stage rotated in place
    uint64_t o_done, o_free, fin;
    uint32_t tmem_base;
    int abort;
    float pw[kC + 1];  // lambda^n, n = 0..128
    double turn[kD / 2];  // RoPE: theta_i / 2pi
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                              volatile int* abort) {
    if (*abort) return false;
    if (!mbar_wait(bar, parity, ctx)) {
        *abort = 1;
        return false;
    }
    return true;
}

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// RoPE of row t (lane = t % 32) of NT [128 x 128] bf16 tiles in place, each held as two
// 128-byte-swizzled sub-tiles kSub apart (d 0-63, d 64-127), so the pair (i, i + 64) sits at the
// same offset in both halves.  The tile's rows sit at positions p0 + t and share frequencies: each
// lane reduces p0 * theta_j / 2pi to a fraction of a turn in double precision for j = lane and
// j = lane + 32, the warp shares them by shuffles, and row t adds t * theta_j / 2pi (at most ~21
// turns, exact to ~2e-6 turns) in single precision before the final reduction and sine/cosine.
template <int NT>
__device__ __forceinline__ void rope_rows(uint8_t* const (&tiles)[NT], int t, int lane,
                                          const double* turn, int64_t p0) {
    float fa, fb, ta, tb;
    {
        double x = (double)p0 * turn[lane];
        double y = (double)p0 * turn[lane + 32];
        fa = (float)(x - rint(x));
        fb = (float)(y - rint(y));
        ta = (float)turn[lane];
        tb = (float)turn[lane + 32];
    }
    const float tr = (float)t;
#pragma unroll 1
    for (int cj = 0; cj < 8; ++cj) {
        const int off = t * 128 + ((cj ^ (t & 7)) << 4);
        float cs[8], sn[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int j = 8 * cj + e;  // frequency index
            const float f0 = __shfl_sync(0xffffffffu, j < 32 ? fa : fb, j & 31);
            const float tj = __shfl_sync(0xffffffffu, j < 32 ? ta : tb, j & 31);
            float x = fmaf(tr, tj, f0);
            x -= rintf(x);
            __sincosf(x * 6.28318530717958647f, &sn[e], &cs[e]);
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const uint4 a = *reinterpret_cast<const uint4*>(tiles[n] + off);
            const uint4 b = *reinterpret_cast<const uint4*>(tiles[n] + kSub + off);
            uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                float x0 = bf_lo(av[w]), x1 = bf_hi(av[w]), y0 = bf_lo(bv[w]), y1 = bf_hi(bv[w]);
                rope_rot(x0, y0, cs[2 * w], sn[2 * w]);
                rope_rot(x1, y1, cs[2 * w + 1], sn[2 * w + 1]);
                av[w] = pack_bf16x2(x0, x1);
                bv[w] = pack_bf16x2(y0, y1);
            }
            *reinterpret_cast<uint4*>(tiles[n] + off) = make_uint4(av[0], av[1], av[2], av[3]);
            *reinterpret_cast<uint4*>(tiles[n] + kSub + off) = make_uint4(bv[0], bv[1], bv[2], bv[3]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
linear_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmO, const float* __restrict__ decay,
                         const float* s_in, float* s_out, int H,
                         int N, int seg_len, int n_seg, int64_t s_in_seg_stride, Rope rope,
                         DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ Bars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA = (batch*head, segment of the sequence, value slice); the segment's incoming state is
    // s_in + seg * s_in_seg_stride (one segment: the whole sequence, stride 0).
    const int slice = blockIdx.x % kSlices;
    const int seg = (blockIdx.x / kSlices) % n_seg;
    const int64_t bh = blockIdx.x / kSlices / n_seg;
    const int row0 = seg * seg_len;
    const int Ns = min(seg_len, N - row0);  // rows of this segment
    const int n_tiles = (Ns + kC - 1) / kC;
    if (s_in) s_in += seg * s_in_seg_stride;
    volatile int* abort = &bars.abort;

    if (warp == 9) {
        tmem_alloc(&bars.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.full[b], 1);
            mbar_init(&bars.empty[b], 2);   // one commit per issuer
            mbar_init(&bars.qk_done[b], 1);
            mbar_init(&bars.a_ready[b], 4);
            mbar_init(&bars.v_ready[b], 4);
            mbar_init(&bars.ds_done[b], 1);
            mbar_init(&bars.s_ready[b], 4);
            mbar_init(&bars.sb_free[b], 1);
            mbar_init(&bars.rot_ready[b], 4);
        }
        mbar_init(&bars.o_done, 2);  // O1 (warp 9) and O2 (warp 10)
        mbar_init(&bars.o_free, 4);
        mbar_init(&bars.fin, 2);
        bars.abort = 0;
        fence_mbar_init();
    }
    {
        const double lam = (double)decay[bh % H];
        for (int n = tid; n <= kC; n += kThreads) bars.pw[n] = (float)pow(lam, (double)n);
        if (rope.base > 0.0)
            for (int i = tid; i < kD / 2; i += kThreads) bars.turn[i] = rope_turn(rope.base, i, kD);
    }
    const bool use_rope = rope.base > 0.0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    // Each warpgroup changes its register count at the top of its own role branch (ptxas then
    // allocates the branch within the new count).
    if (warp >= 8 && warp < 12) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (warp == 8) {
            // ------------------------------------------------------------------ TMA producer
            if (lane == 0) {
                int issued[2] = {-1, -1};
                for (int c = 0; c < n_tiles; ++c) {
                    const int s = c & 1, r = c >> 1;
                    if (r >= 1 && !wait_or_abort(&bars.empty[s], (r - 1) & 1, ctx, abort)) break;
                    uint8_t* st = sm + s * kStageBytes;
                    mbar_arrive_expect_tx(&bars.full[s], kStageBytes);
                    const int y = row0 + c * kC, z = (int)bh;
                    tma_load_3d(st + kOffQ, &tmQ, &bars.full[s], 0, y, z);
                    tma_load_3d(st + kOffQ + kSub, &tmQ, &bars.full[s], 64, y, z);
                    tma_load_3d(st + kOffK, &tmK, &bars.full[s], 0, y, z);
                    tma_load_3d(st + kOffK + kSub, &tmK, &bars.full[s], 64, y, z);
                    tma_load_3d(st + kOffV, &tmV, &bars.full[s], slice * kDv, y, z);
                    issued[s] = r;
                }
                for (int s = 0; s < 2; ++s)
                    if (issued[s] >= 0) (void)mbar_wait(&bars.full[s], issued[s] & 1, ctx);
            }
            __syncwarp();
        } else if (warp == 9 || warp == 10) {
            // ------------------------------------------------------------------ MMA issuers
            // Two issuing threads, so that one thread's issue latency does not serialise the four
            // products: warp 9 issues the attention path (MMA1, MMA2), warp 10 the state path (MMA3,
            // MMA4).  Each commits its own share of the stage release, of o_done and of fin.  The
            // shared-memory descriptors are kept as 32-bit halves; a K-step adds to the low half.
            if (lane == 0) {
                const uint32_t hi = sdesc_sw128_hi(1024);
                // Low halves for stage 0; stage st adds st * kStageBytes / 16 to the address field.
                const uint32_t base = smem_u32(sm);
                const uint32_t q_lo0 = sdesc_sw128_lo(base + kOffQ, 16);
                const uint32_t k_lo0 = sdesc_sw128_lo(base + kOffK, 16);
                const uint32_t kt_lo0 = sdesc_sw128_lo(base + kOffK, kSub);  // K read transposed (MMA4)
                const uint32_t v_lo0 = sdesc_sw128_lo(base + kOffV, 8192);
                auto at_stage = [](uint32_t lo, int st) -> uint32_t { return lo + (uint32_t)(st * (kStageBytes >> 4)); };
                // K-major operand [128 x 128] in two 64-column sub-tiles: K-step ks starts at
                // sub-tile ks / 4, byte 32 (ks % 4) of its rows.
                auto kstep = [](int ks) -> uint32_t { return (uint32_t)(((ks >> 2) * kSub + (ks & 3) * 32) >> 4); };
                if (warp == 9) {
                    const uint32_t idQK = idesc_bf16_f32(128, 128, false, false);
                    const uint32_t idO = idesc_bf16_f32(128, kDv, false, true);
                    auto issue_qk = [&](int c) -> bool {  // MMA1: A = Q K^T
                        const int st = c & 1;
                        if (!wait_or_abort(&bars.full[st], (c >> 1) & 1, ctx, abort)) return false;
                        // with RoPE, Q and K of the stage are rotated in place first
                        if (use_rope && !wait_or_abort(&bars.rot_ready[st], (c >> 1) & 1, ctx, abort)) return false;
                        tc_fence_after();
    #pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks)
                            mma_ss_lohi(tmem + kColA0 + st * 128, at_stage(q_lo0, st) + kstep(ks), at_stage(k_lo0, st) + kstep(ks), hi,
                                        idQK, ks > 0);
                        mma_commit(&bars.qk_done[st]);
                        return true;
                    };
                    bool ok = n_tiles > 0 ? issue_qk(0) : true;
                    for (int c = 0; c < n_tiles && ok; ++c) {
                        const int st = c & 1;
                        // MMA2: O1 = A' V (A' from TMEM) once the mask is done and O1 is free.
                        if (!wait_or_abort(&bars.a_ready[st], (c >> 1) & 1, ctx, abort)) break;
                        if (c >= 1 && !wait_or_abort(&bars.o_free, (c - 1) & 1, ctx, abort)) break;
                        tc_fence_after();
    #pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            mma_ts_lohi(tmem + kColO1, tmem + kColA0 + st * 128 + ks * 8,
                                        at_stage(v_lo0, st) + (uint32_t)((ks * 16 * 128) >> 4), hi, idO, ks > 0);
                        mma_commit(&bars.o_done);
                        mma_commit(&bars.empty[st]);  // this thread's last read of stage c
                        if (c + 1 < n_tiles) ok = issue_qk(c + 1);
                    }
                } else {
                    const uint32_t idO = idesc_bf16_f32(128, kDv, false, true);
                    const uint32_t idDS = idesc_bf16_f32(128, kDv, true, true);
                    const uint32_t sb_lo0 = sdesc_sw128_lo(smem_u32(sm + kOffSb), 8192);
                    const uint32_t vt_lo0 = sdesc_sw128_lo(smem_u32(sm + kOffVt), 8192);
                    auto issue_ds = [&](int c) -> bool {  // MMA4: dS(c) = K^T V~ (A read transposed)
                        const int st = c & 1;
                        if (!wait_or_abort(&bars.full[st], (c >> 1) & 1, ctx, abort)) return false;
                        if (!wait_or_abort(&bars.v_ready[st], (c >> 1) & 1, ctx, abort)) return false;
                        // with RoPE, Q (MMA3) and K (MMA4) of the stage rotated in place first
                        if (use_rope && !wait_or_abort(&bars.rot_ready[st], (c >> 1) & 1, ctx, abort)) return false;
                        tc_fence_after();
                        const uint32_t vt_lo = vt_lo0;
    #pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            mma_ss_lohi(tmem + kColDS + st * kDv, at_stage(kt_lo0, st) + (uint32_t)((ks * 16 * 128) >> 4),
                                        vt_lo + (uint32_t)((ks * 16 * 128) >> 4), hi, idDS, ks > 0);
                        mma_commit(&bars.ds_done[st]);
                        return true;
                    };
                    bool ok = n_tiles > 0 ? issue_ds(0) : true;
                    for (int c = 0; c < n_tiles && ok; ++c) {
                        const int st = c & 1;
                        // MMA3: O2 = Q Sb(c-1), read from buffer c&1.  Sb(c-1) published also means
                        // dS(c-1) has been consumed, so its TMEM buffer is free for dS(c+1) below.
                        if (!wait_or_abort(&bars.s_ready[st], (c >> 1) & 1, ctx, abort)) break;
                        if (c >= 1 && !wait_or_abort(&bars.o_free, (c - 1) & 1, ctx, abort)) break;
                        tc_fence_after();
                        const uint32_t sb_lo = sb_lo0 + (uint32_t)((st * kSub) >> 4);
    #pragma unroll
                        for (int ks = 0; ks < kD / 16; ++ks)
                            mma_ss_lohi(tmem + kColO2, at_stage(q_lo0, st) + kstep(ks), sb_lo + (uint32_t)((ks * 16 * 128) >> 4),
                                        hi, idO, ks > 0);
                        mma_commit(&bars.sb_free[st]);
                        mma_commit(&bars.o_done);
                        mma_commit(&bars.empty[st]);  // MMA4(c) came earlier: this thread is done with c
                        if (c + 1 < n_tiles) ok = issue_ds(c + 1);  // dS one tile ahead
                    }
                }
                mma_commit(&bars.fin);
                (void)mbar_wait(&bars.fin, 0, ctx);
            }
            __syncwarp();
        }  // warp 11: idle
    } else if (warp >= 12) {
        // ------------------------------------------------------------------ RoPE of Q and K
        // thread = row of the tile; each stage's Q and K rotated in place before its MMAs
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (use_rope) {
            const int t = tid - 384;
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c & 1;
                if (!wait_or_abort(&bars.full[s], (c >> 1) & 1, ctx, abort)) break;
                uint8_t* const qk[2] = {sm + s * kStageBytes + kOffQ, sm + s * kStageBytes + kOffK};
                rope_rows<2>(qk, t, lane, bars.turn, rope.pos0 + row0 + (int64_t)c * kC);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.rot_ready[s]);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------------ EPI-A: mask, output
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
        const int t = tid;
        const uint32_t lb = tmem_lane_base(warp);
        const float wq = bars.pw[t + 1];
        // Per tile the warp group reads O(c), masks tile c+1, then stores o(c): reading O before
        // the mask frees O1 and O2 early, so MMA2(c+1) and MMA3(c+1) -- the last readers of the
        // stage of tile c+1 -- issue right after the mask (with the mask first they waited for
        // the whole output step, and the ring's refill with them).
        auto mask = [&](int c) -> bool {  // A' = A * lambda^{t-s} [s <= t], bf16, over A in TMEM
            const int s = c & 1;
            if (!wait_or_abort(&bars.qk_done[s], (c >> 1) & 1, ctx, abort)) return false;
            tc_fence_after();
            const uint32_t colA = tmem + lb + kColA0 + s * 128;
            // s > t is masked; tiles never reach s >= 128, and rows/keys past len are zero.
            const int kmax = (t >> 5) + 1;  // 32-column chunks holding some s <= t
#pragma unroll 1
            for (int kc = 0; kc < 4; ++kc) {
                const int k0 = kc * 32;
                uint32_t pk[16];
                if (__any_sync(0xffffffffu, kc < kmax)) {
                    uint32_t x[32];
                    tmem_ld32(colA + k0, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int s0 = k0 + 2 * j, s1 = s0 + 1;
                        const float w0 = s0 <= t ? bars.pw[t - s0] : 0.f;
                        const float w1 = s1 <= t ? bars.pw[t - s1] : 0.f;
                        pk[j] = pack_bf16x2(__uint_as_float(x[2 * j]) * w0, __uint_as_float(x[2 * j + 1]) * w1);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) pk[j] = 0u;
                }
                tmem_st16(colA + k0 / 2, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.a_ready[s]);
            return true;
        };
        // o_t = O1 + lambda^{t+1} O2 in two steps.  read_out takes O1 and O2 of tile c out of TMEM
        // and frees them at once (MMA2(c+1) and MMA3(c+1) wait for that), keeping the packed bf16
        // row; store_out writes it once the next tile's mask is done.
        auto read_out = [&](int c, uint32_t (&wp)[32]) -> bool {
            if (!wait_or_abort(&bars.o_done, c & 1, ctx, abort)) return false;
            tc_fence_after();
            uint32_t o1[64], o2[64];
            tmem_ld32(tmem + lb + kColO1, *reinterpret_cast<uint32_t(*)[32]>(&o1[0]));
            tmem_ld32(tmem + lb + kColO1 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o1[32]));
            tmem_ld32(tmem + lb + kColO2, *reinterpret_cast<uint32_t(*)[32]>(&o2[0]));
            tmem_ld32(tmem + lb + kColO2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o2[32]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.o_free);
#pragma unroll
            for (int j = 0; j < 32; ++j)
                wp[j] = pack_bf16x2(fmaf(wq, __uint_as_float(o2[2 * j]), __uint_as_float(o1[2 * j])),
                                    fmaf(wq, __uint_as_float(o2[2 * j + 1]), __uint_as_float(o1[2 * j + 1])));
            return true;
        };
        auto store_out = [&](int c, const uint32_t (&wp)[32]) {
            // The warp's 32 rows go out as one TMA store from its own 4 KiB of the staging tile
            // (128-byte swizzle, as the tensor map reads it): the previous tile's store from the
            // same rows must have read them first.  Rows past the sequence end are clipped by the
            // tensor map; within a sequence every tile but the last is full.
            uint8_t* stg = sm + kOffOst + warp * 32 * 128;
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int cj = 0; cj < 8; ++cj)
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((cj ^ (lane & 7)) << 4)) =
                    make_uint4(wp[4 * cj], wp[4 * cj + 1], wp[4 * cj + 2], wp[4 * cj + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && c * kC + warp * 32 < Ns) {  // no store starts past the end
                tma_store_3d(&tmO, stg, slice * kDv, row0 + c * kC + warp * 32, (int)bh);
                bulk_commit();
            }
        };
        // Per tile c: O(c) out of TMEM, then the mask of tile c+1 (MMA2(c+1) and MMA3(c+1) can
        // issue as soon as it is done, and the stage of tile c+1 goes back to the producer right
        // after them), then the store of o(c).
        bool ok = n_tiles > 0 ? mask(0) : true;
        for (int c = 0; c < n_tiles && ok; ++c) {
            uint32_t wp[32];
            if (!read_out(c, wp)) break;
            if (c + 1 < n_tiles && !mask(c + 1)) break;
            store_out(c, wp);
        }
        if (lane == 0) bulk_wait0();  // this warp's stores complete before the CTA retires
    } else if (warp < 8) {
        // ------------------------------------------------------------------ EPI-S: V~, state
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
        const int t = tid - 128;  // row of the V tile / of the state slice
        const uint32_t lb = tmem_lane_base(warp);
        float S[kDv];
        const float* sin_row = s_in ? s_in + (bh * kD + t) * kD + slice * kDv : nullptr;
#pragma unroll
        for (int j = 0; j < kDv; j += 4) {
            float4 x = sin_row ? *reinterpret_cast<const float4*>(sin_row + j) : make_float4(0, 0, 0, 0);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        // bf16 copy Sb(c) of this thread's state row (128-byte swizzle) into buffer (c+1)&1.
        auto write_sb = [&](int c) {
            const int b = (c + 1) & 1;
            uint8_t* sbrow = sm + kOffSb + b * kSub + t * 128;
#pragma unroll
            for (int cj = 0; cj < 8; ++cj) {
                uint4 w;
                w.x = pack_bf16x2(S[cj * 8 + 0], S[cj * 8 + 1]);
                w.y = pack_bf16x2(S[cj * 8 + 2], S[cj * 8 + 3]);
                w.z = pack_bf16x2(S[cj * 8 + 4], S[cj * 8 + 5]);
                w.w = pack_bf16x2(S[cj * 8 + 6], S[cj * 8 + 7]);
                *reinterpret_cast<uint4*>(sbrow + ((cj ^ (t & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_ready[b]);
        };
        // V~(c) = lambda^{len-1-s} V (row t of the V tile), same swizzled layout; the 16-byte
        // chunks are visited in their physical order so a warp's 32 rows hit distinct banks.
        auto make_vt = [&](int c) -> bool {
            const int s = c & 1;
            const int len = min(kC, Ns - c * kC);
            if (!wait_or_abort(&bars.full[s], (c >> 1) & 1, ctx, abort)) return false;
            const float w = t < len ? bars.pw[len - 1 - t] : 0.f;
            const uint8_t* vrow = sm + s * kStageBytes + kOffV + t * 128;
            uint8_t* vtrow = sm + kOffVt + t * 128;
#pragma unroll
            for (int cj = 0; cj < 8; ++cj) {
                const int p = (cj ^ (t & 7)) << 4;
                uint4 a = *reinterpret_cast<const uint4*>(vrow + p);
                uint4 b;
                b.x = pack_bf16x2(bf_lo(a.x) * w, bf_hi(a.x) * w);
                b.y = pack_bf16x2(bf_lo(a.y) * w, bf_hi(a.y) * w);
                b.z = pack_bf16x2(bf_lo(a.z) * w, bf_hi(a.z) * w);
                b.w = pack_bf16x2(bf_lo(a.w) * w, bf_hi(a.w) * w);
                *reinterpret_cast<uint4*>(vtrow + p) = b;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.v_ready[s]);
            return true;
        };
        write_sb(-1);
        bool ok = n_tiles > 0 ? make_vt(0) : true;
        for (int c = 0; c < n_tiles && ok; ++c) {
            const int s = c & 1;
            const int len = min(kC, Ns - c * kC);
            // S <- lambda^len S + dS(c), then its bf16 copy for the next tile; then V~(c+1) into
            // the one V~ buffer, which MMA4(c) (done with dS(c)) has finished reading.
            if (!wait_or_abort(&bars.ds_done[s], (c >> 1) & 1, ctx, abort)) { ok = false; break; }
            tc_fence_after();
            uint32_t d0[32], d1[32];
            tmem_ld32(tmem + lb + kColDS + s * kDv, d0);
            tmem_ld32(tmem + lb + kColDS + s * kDv + 32, d1);
            tmem_ld_wait();
            const float decay_len = bars.pw[len];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                S[j] = fmaf(decay_len, S[j], __uint_as_float(d0[j]));
                S[32 + j] = fmaf(decay_len, S[32 + j], __uint_as_float(d1[j]));
            }
            tc_fence_before();
            // Buffer (c+1)&1 last held Sb(c-2), read by MMA3(c-1): wait until that MMA is done.
            if (c >= 1 && !wait_or_abort(&bars.sb_free[(c - 1) & 1], ((c - 1) >> 1) & 1, ctx, abort)) {
                ok = false;
                break;
            }
            write_sb(c);
            if (c + 1 < n_tiles && !make_vt(c + 1)) { ok = false; break; }
        }
        if (ok && s_out) {
            float* row = s_out + (bh * kD + t) * kD + slice * kDv;
#pragma unroll
            for (int j = 0; j < kDv; j += 4)
                *reinterpret_cast<float4*>(row + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------------------
// Sequence-parallel prefill.  The state recursion S(c) = lambda^len S(c-1) + dS(c) is the only
// serial dependency, and dS needs no state: so a sequence split into segments can first compute
// each segment's own contribution S_seg (from a zero state, K and V only), then chain the segments'
// incoming states in a tiny pass (S_in(p+1) = lambda^len(p) S_in(p) + S_seg(p)), then run the
// output pass above on every segment at once.  K and V are read twice, but every SM has work.
//
// State pass, per CTA = (batch*head, segment, value slice): warp 4 streams K and the V slice
// through a 3-stage ring, warp 5 issues dS = K^T V~ per tile into one of two TMEM buffers,
// warps 0-3 (thread = row of S) write V~ and fold dS into the fp32 state held in registers, and
// with RoPE warps 6-9 rotate each stage's K in place (thread = row of the tile).
constexpr int kStStages = 3;
constexpr int kStStage = 3 * kSub;                     // K (2 sub-tiles) + V slice (1)
constexpr int kStOffVt = kStStages * kStStage;         // V~, 2 buffers
constexpr int kStSmem = kStOffVt + 2 * kSub + 1024;
constexpr int kStThreads = 320;  // warps 6-9 rotate K when RoPE is on (idle otherwise)

struct StBars {
    uint64_t full[kStStages], empty[kStStages], rot_ready[kStStages];
    uint64_t v_ready[2], ds_done[2], ds_free[2];
    uint64_t fin;
    uint32_t tmem_base;
    int abort;
    float pw[kC + 1];
    double turn[kD / 2];  // RoPE: theta_i / 2pi
};

__global__ void __launch_bounds__(kStThreads, 1)
linear_state_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const float* __restrict__ decay, float* __restrict__ s_seg, int H, int N,
                       int seg_len, int n_seg, int64_t seg_stride, Rope rope, DevCtx ctx) {
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
    __shared__ StBars bars;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % kSlices;
    const int seg = (blockIdx.x / kSlices) % n_seg;
    const int64_t bh = blockIdx.x / kSlices / n_seg;
    const int row0 = seg * seg_len;
    const int Ns = min(seg_len, N - row0);
    const int n_tiles = (Ns + kC - 1) / kC;
    volatile int* abort = &bars.abort;
    if (warp == 5) {
        tmem_alloc(&bars.tmem_base, 128);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < kStStages; ++s) {
            mbar_init(&bars.full[s], 1);
            mbar_init(&bars.empty[s], 1);
            mbar_init(&bars.rot_ready[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.v_ready[b], 4);
            mbar_init(&bars.ds_done[b], 1);
            mbar_init(&bars.ds_free[b], 4);
        }
        mbar_init(&bars.fin, 1);
        bars.abort = 0;
        fence_mbar_init();
    }
    {
        const double lam = (double)decay[bh % H];
        for (int n = tid; n <= kC; n += kStThreads) bars.pw[n] = (float)pow(lam, (double)n);
        if (rope.base > 0.0)
            for (int i = tid; i < kD / 2; i += kStThreads) bars.turn[i] = rope_turn(rope.base, i, kD);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int last = -1;
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c % kStStages, r = c / kStStages;
                if (r >= 1 && !wait_or_abort(&bars.empty[s], (r - 1) & 1, ctx, abort)) break;
                uint8_t* st = sm + s * kStStage;
                mbar_arrive_expect_tx(&bars.full[s], kStStage);
                const int y = row0 + c * kC, z = (int)bh;
                tma_load_3d(st, &tmK, &bars.full[s], 0, y, z);
                tma_load_3d(st + kSub, &tmK, &bars.full[s], 64, y, z);
                tma_load_3d(st + 2 * kSub, &tmV, &bars.full[s], slice * kDv, y, z);
                last = c;
            }
            for (int c = last - kStStages + 1; c <= last; ++c)  // drain: copies in flight land
                if (c >= 0) (void)mbar_wait(&bars.full[c % kStStages], (c / kStStages) & 1, ctx);
        }
        __syncwarp();
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idDS = idesc_bf16_f32(128, kDv, true, true);
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c % kStStages, b = c & 1;
                if (!wait_or_abort(&bars.full[s], (c / kStStages) & 1, ctx, abort)) break;
                if (!wait_or_abort(&bars.v_ready[b], (c >> 1) & 1, ctx, abort)) break;
                if (rope.base > 0.0 && !wait_or_abort(&bars.rot_ready[s], (c / kStStages) & 1, ctx, abort)) break;
                if (c >= 2 && !wait_or_abort(&bars.ds_free[b], ((c - 2) >> 1) & 1, ctx, abort)) break;
                tc_fence_after();
                const uint32_t k = smem_u32(sm + s * kStStage);
                const uint32_t vt = smem_u32(sm + kStOffVt + b * kSub);
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_ss(tmem + b * kDv, sdesc_sw128(k + ks * 16 * 128, kSub, 1024),
                           sdesc_sw128(vt + ks * 16 * 128, 8192, 1024), idDS, ks > 0);
                mma_commit(&bars.ds_done[b]);
                mma_commit(&bars.empty[s]);
            }
            mma_commit(&bars.fin);
            (void)mbar_wait(&bars.fin, 0, ctx);
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- RoPE of K
        // thread = row of the K tile; each stage's K rotated in place before its MMA
        if (rope.base > 0.0) {
            const int t = tid - 192;
            for (int c = 0; c < n_tiles; ++c) {
                const int s = c % kStStages;
                if (!wait_or_abort(&bars.full[s], (c / kStStages) & 1, ctx, abort)) break;
                uint8_t* const kt[1] = {sm + s * kStStage};
                rope_rows<1>(kt, t, lane, bars.turn, rope.pos0 + row0 + (int64_t)c * kC);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.rot_ready[s]);
            }
        }
    } else {
        // ---------------------------------------------------------------- V~ and the state
        const int t = tid;  // row of the V tile / of the state slice
        const uint32_t lb = tmem_lane_base(warp);
        float S[kDv];
#pragma unroll
        for (int j = 0; j < kDv; ++j) S[j] = 0.f;
        auto make_vt = [&](int c) -> bool {
            const int s = c % kStStages;
            const int len = min(kC, Ns - c * kC);
            if (!wait_or_abort(&bars.full[s], (c / kStStages) & 1, ctx, abort)) return false;
            const float w = t < len ? bars.pw[len - 1 - t] : 0.f;
            const uint8_t* vrow = sm + s * kStStage + 2 * kSub + t * 128;
            uint8_t* vtrow = sm + kStOffVt + (c & 1) * kSub + t * 128;
#pragma unroll
            for (int cj = 0; cj < 8; ++cj) {
                const int p = (cj ^ (t & 7)) << 4;
                const uint4 a = *reinterpret_cast<const uint4*>(vrow + p);
                uint4 o;
                o.x = pack_bf16x2(bf_lo(a.x) * w, bf_hi(a.x) * w);
                o.y = pack_bf16x2(bf_lo(a.y) * w, bf_hi(a.y) * w);
                o.z = pack_bf16x2(bf_lo(a.z) * w, bf_hi(a.z) * w);
                o.w = pack_bf16x2(bf_lo(a.w) * w, bf_hi(a.w) * w);
                *reinterpret_cast<uint4*>(vtrow + p) = o;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.v_ready[c & 1]);
            return true;
        };
        bool ok = n_tiles > 0 ? make_vt(0) : true;
        for (int c = 0; c < n_tiles && ok; ++c) {
            const int b = c & 1;
            const int len = min(kC, Ns - c * kC);
            if (c + 1 < n_tiles && !(ok = make_vt(c + 1))) break;
            if (!(ok = wait_or_abort(&bars.ds_done[b], (c >> 1) & 1, ctx, abort))) break;
            tc_fence_after();
            uint32_t d0[32], d1[32];
            tmem_ld32(tmem + lb + b * kDv, d0);
            tmem_ld32(tmem + lb + b * kDv + 32, d1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.ds_free[b]);
            const float decay_len = bars.pw[len];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                S[j] = fmaf(decay_len, S[j], __uint_as_float(d0[j]));
                S[32 + j] = fmaf(decay_len, S[32 + j], __uint_as_float(d1[j]));
            }
        }
        if (ok) {
            float* row = s_seg + seg * seg_stride + (bh * kD + t) * kD + slice * kDv;
#pragma unroll
            for (int j = 0; j < kDv; j += 4)
                *reinterpret_cast<float4*>(row + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// Chains the segments' states, in place: on entry s_seg[p] holds segment p's own contribution, on
// exit its incoming state S_in(p); S_in(0) = state_in (or 0), S_in(p+1) = lambda^len(p) S_in(p)
// + S_seg(p).  state_out (if given) receives the state after the last segment.  Thread = one
// state element of one head.
constexpr int kMaxSeg = 64;
__global__ void __launch_bounds__(256)
linear_state_chain_kernel(float* __restrict__ s_seg, const float* __restrict__ state_in,
                          float* __restrict__ state_out, const float* __restrict__ decay, int BH,
                          int H, int N, int seg_len, int n_seg) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over BH * d * d
    if (e >= (int64_t)BH * kD * kD) return;
    const int64_t bh = e / (kD * kD);
    const int64_t seg_stride = (int64_t)BH * kD * kD;
    const double lam = (double)decay[bh % H];
    const float w_full = (float)pow(lam, (double)seg_len);
    const float w_last = (float)pow(lam, (double)(N - (n_seg - 1) * seg_len));
    float s = state_in ? state_in[e] : 0.f;
    for (int p0 = 0; p0 < n_seg; p0 += 8) {  // 8 segments' loads in flight, then their updates
        float contrib[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) contrib[i] = p0 + i < n_seg ? s_seg[(p0 + i) * seg_stride + e] : 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int p = p0 + i;
            if (p < n_seg) {
                s_seg[p * seg_stride + e] = s;
                s = fmaf(p + 1 < n_seg ? w_full : w_last, s, contrib[i]);
            }
        }
    }
    if (state_out) state_out[e] = s;
}

}  // namespace

bool linear_prefill_tc_supported(int d) { return d == kD; }

namespace {

int sm_count() { return device_sm_count(); }

// Segments for the sequence-parallel form: the count that minimises (waves of output-pass CTAs) x
// (rows per segment) plus a per-segment cost for the state chaining (a segment boundary costs about
// as much as 64 rows of output work).  Short sequences, or ones whose heads already fill the GPU,
// stay in one segment.
void pick_segments(int B, int H, int N, int* n_seg, int* seg_len) {
    *n_seg = 1;
    *seg_len = N;
    const int64_t ctas1 = (int64_t)B * H * kSlices;
    const int nsm = sm_count();
    if (N < 8 * kC || ctas1 >= 2 * nsm) return;
    double best = (double)((ctas1 + nsm - 1) / nsm) * N;
    for (int n = 2; n <= kMaxSeg; ++n) {
        const int len = ((N + n - 1) / n + kC - 1) / kC * kC;
        const int ne = (N + len - 1) / len;
        if (ne != n) continue;
        const double waves = (double)((ctas1 * ne + nsm - 1) / nsm);
        const double cost = waves * len + 64.0 * ne;
        if (cost < best) {
            best = cost;
            *n_seg = ne;
            *seg_len = len;
        }
    }
}

}  // namespace

size_t linear_prefill_tc_workspace(int B, int H, int N, int d) {
    if (d != kD || B <= 0 || H <= 0 || N <= 0) return 0;
    int n_seg, seg_len;
    pick_segments(B, H, N, &n_seg, &seg_len);
    return n_seg > 1 ? (size_t)n_seg * B * H * kD * kD * sizeof(float) : 0;
}

cudaError_t launch_linear_prefill_tc(const void* q, const void* k, const void* v,
                                     const float* decay, void* o, const float* s_in,
                                     float* s_out, int B, int H, int N, int d, void* ws,
                                     size_t ws_bytes, Rope rope, cudaStream_t st, DevCtx ctx) {
    if (d != kD) return cudaErrorNotSupported;
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return cudaErrorNotSupported;
    auto make3 = [&](CUtensorMap* m, const void* base, uint32_t box_rows) -> bool {
        cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)N, (cuuint64_t)B * H};
        cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kD * 2 * N};
        cuuint32_t box[3] = {64, box_rows, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    CUtensorMap tmQ, tmK, tmV, tmO;  // O: one warp's 32 rows per store
    if (!make3(&tmQ, q, kC) || !make3(&tmK, k, kC) || !make3(&tmV, v, kC) || !make3(&tmO, o, 32))
        return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem<linear_prefill_tc_kernel>(kSmemBytes);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits until the block's pool holds the registers: launch only when the
    // compiled per-thread count (the pool is that count times the threads) covers the split.
    static int regs_ok = -1;
    if (regs_ok < 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, linear_prefill_tc_kernel);
        if (e != cudaSuccess) return e;
        regs_ok = fa.numRegs * kThreads >= 256 * kRegsEpi + 256 * kRegsOther ? 1 : 0;
    }
    if (!regs_ok) return cudaErrorNotSupported;
    int n_seg, seg_len;
    pick_segments(B, H, N, &n_seg, &seg_len);
    const int64_t seg_stride = (int64_t)B * H * kD * kD;
    if (n_seg > 1 && ws && ws_bytes >= (size_t)n_seg * seg_stride * sizeof(float)) {
        float* s_seg = static_cast<float*>(ws);
        e = ensure_smem<linear_state_tc_kernel>(kStSmem);
        if (e != cudaSuccess) return e;
        linear_state_tc_kernel<<<B * H * n_seg * kSlices, kStThreads, kStSmem, st>>>(
            tmK, tmV, decay, s_seg, H, N, seg_len, n_seg, seg_stride, rope, ctx);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int64_t elems = seg_stride;
        linear_state_chain_kernel<<<(unsigned)((elems + 255) / 256), 256, 0, st>>>(
            s_seg, s_in, s_out, decay, B * H, H, N, seg_len, n_seg);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        linear_prefill_tc_kernel<<<B * H * n_seg * kSlices, kThreads, kSmemBytes, st>>>(
            tmQ, tmK, tmV, tmO, decay, s_seg, nullptr, H, N, seg_len, n_seg, seg_stride, rope, ctx);
        return cudaGetLastError();
    }
    // One segment.  If state_out aliases state_in, every CTA reads its slice before it writes it
    // back, and no two CTAs share a slice, so in-place update is safe.
    linear_prefill_tc_kernel<<<B * H * kSlices, kThreads, kSmemBytes, st>>>(
        tmQ, tmK, tmV, tmO, decay, s_in, s_out, H, N, N, 1, 0, rope, ctx);
    return cudaGetLastError();
}

}  // namespace sala
