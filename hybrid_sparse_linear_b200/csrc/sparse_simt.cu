// Block-sparse softmax attention on CUDA cores: the fp32 prefill and the decode step.
//
// Prefill: one CTA per (batch, KV group, query row).  The G query heads of the group share the
// row's selected blocks, so each selected K/V block is staged in shared memory once and read by
// every head (one warp per head); each warp keeps an online softmax (running max m, running sum
// l, running output o) over the blocks.  Keys after the query position, or past N, are masked.
//
// Decode: flash-decoding style.  Kernel 1 gives every selected block its own CTA and writes a
// partial (m, l, o) per head; kernel 2 combines the partials of each head.
#include <float.h>

#include "kernels.h"

namespace sala {
namespace {

constexpr int kBlk = 64;
constexpr int kWarps = 8;

template <int D>
struct BlockSmem {
    static constexpr size_t bytes = sizeof(float) * (D * (kBlk + 1) + kBlk * D);
};

// Stage block `blk` of one KV head into shared memory: Kt[D][65] (transposed), Vs[64][D].
template <typename T, int D>
__device__ __forceinline__ void stage_block(const T* __restrict__ kh, const T* __restrict__ vh,
                                            int blk, int nrows, float* Kt, float* Vs) {
    for (int e = threadIdx.x; e < kBlk * D; e += blockDim.x) {
        const int t = e / D, a = e % D;
        const int64_t j = (int64_t)blk * kBlk + t;
        const bool ok = j < nrows;
        Kt[a * (kBlk + 1) + t] = ok ? to_f(kh[j * D + a]) : 0.f;
        Vs[t * D + a] = ok ? to_f(vh[j * D + a]) : 0.f;
    }
}

// One warp folds one staged block into its head's online softmax.  Keys j with j > last are
// masked.  qv: this lane's view of q is read from shared memory qrow[D].
template <int D>
__device__ __forceinline__ void fold_block(const float* Kt, const float* Vs, const float* qrow,
                                           int64_t j0, int64_t last, float scale, float& m,
                                           float& l, float (&o)[D / 32], int lane) {
    float s[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int t = hf * 32 + lane;
        float acc = 0.f;
#pragma unroll 8
        for (int a = 0; a < D; ++a) acc = fmaf(qrow[a], Kt[a * (kBlk + 1) + t], acc);
        s[hf] = (j0 + t <= last) ? acc * scale : -INFINITY;
    }
    float mx = fmaxf(s[0], s[1]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) return;  // nothing attended yet
    const float corr = expf(m - m_new);
    const float p0 = expf(s[0] - m_new), p1 = expf(s[1] - m_new);
    float ps = p0 + p1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * corr + ps;
    m = m_new;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) o[j] *= corr;
    for (int t = 0; t < kBlk; ++t) {
        const float p = __shfl_sync(0xffffffffu, t < 32 ? p0 : p1, t & 31);
        if (p == 0.f) continue;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) o[j] = fmaf(p, Vs[t * D + j * 32 + lane], o[j]);
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
sparse_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                           const T* __restrict__ v, const int32_t* __restrict__ idx,
                           T* __restrict__ o, int H, int Hkv, int Hs, int N, int slots,
                           float scale, DevCtx ctx) {
    extern __shared__ float sms[];
    float* Kt = sms;
    float* Vs = Kt + D * (kBlk + 1);
    float* Qs = Vs + kBlk * D;  // [G][D]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // Selection group (b, g) of Hs per batch: heads g*G .. g*G+G-1 share idx row (b, g, i) and
    // read the K/V of their KV head.
    const int G = H / Hs;
    const int64_t i = blockIdx.x;
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hs;
    const int g = (int)(bg % Hs);
    const int64_t kv_plane = b * Hkv + g / (Hs / Hkv);
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int hh = e / D, a = e % D;
        Qs[e] = to_f(q[((b * H + (int64_t)g * G + hh) * N + i) * D + a]);
    }
    const T* kh = k + kv_plane * (int64_t)N * D;
    const T* vh = v + kv_plane * (int64_t)N * D;
    const int32_t* sel = idx + (bg * N + i) * (int64_t)slots;
    const int max_blk = (int)(i / kBlk);

    constexpr int kHeadsPerWarp = 2;  // G <= 16 with 8 warps
    float m[kHeadsPerWarp], l[kHeadsPerWarp], acc[kHeadsPerWarp][D / 32];
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
        m[u] = -INFINITY;
        l[u] = 0.f;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) acc[u][j] = 0.f;
    }
    for (int s = 0; s < slots; ++s) {
        const int blk = sel[s];
        if (blk < 0) continue;
        if (blk > max_blk) {
            if (threadIdx.x == 0) flag(ctx, kStatusBounds);
            continue;
        }
        __syncthreads();
        stage_block<T, D>(kh, vh, blk, N, Kt, Vs);
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kHeadsPerWarp; ++u) {
            const int hh = warp + u * kWarps;
            if (hh < G)
                fold_block<D>(Kt, Vs, Qs + hh * D, (int64_t)blk * kBlk, i, scale, m[u], l[u],
                              acc[u], lane);
        }
    }
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
        const int hh = warp + u * kWarps;
        if (hh >= G) continue;
        const float inv = l[u] > 0.f ? 1.f / l[u] : 0.f;
        T* out = o + ((b * H + (int64_t)g * G + hh) * N + i) * D;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) out[j * 32 + lane] = from_f<T>(acc[u][j] * inv);
    }
}

template <typename T, int D>
cudaError_t prefill(const void* q, const void* k, const void* v, const int32_t* idx, void* o, int B,
                    int H, int Hkv, int Hs, int N, int slots, float scale, cudaStream_t st,
                    DevCtx ctx) {
    auto kern = sparse_prefill_simt_kernel<T, D>;
    const int G = H / Hs;
    const size_t smem = BlockSmem<D>::bytes + sizeof(float) * G * D;
    cudaError_t e = ensure_smem<sparse_prefill_simt_kernel<T, D>>((int)(BlockSmem<D>::bytes + sizeof(float) * 2 * kWarps * D));
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)N, (unsigned)(B * Hs));
    kern<<<grid, kWarps * 32, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                          static_cast<const T*>(v), idx, static_cast<T*>(o), H,
                                          Hkv, Hs, N, slots, scale, ctx);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Decode.  Partial record per (batch*group, slot, head): [m, l, o[0..D)].
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
sparse_decode_partial_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                             const T* __restrict__ vc, const int32_t* __restrict__ idx,
                             float* __restrict__ part, int H, int Hkv, int pos, int Tmax,
                             int slots, float scale, DevCtx ctx) {
    extern __shared__ float sms[];
    float* Kt = sms;
    float* Vs = Kt + D * (kBlk + 1);
    float* Qs = Vs + kBlk * D;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = H / Hkv;
    const int s = blockIdx.x;
    const int64_t bg = blockIdx.y;
    const int64_t b = bg / Hkv;
    const int g = (int)(bg % Hkv);
    int blk = idx[bg * slots + s];
    if (blk > pos / kBlk) {
        if (threadIdx.x == 0) flag(ctx, kStatusBounds);
        blk = -1;
    }
    float* rec = part + (bg * slots + s) * (int64_t)G * (D + 2);
    if (blk < 0) {
        for (int e = threadIdx.x; e < G; e += blockDim.x) {
            rec[e * (D + 2)] = -INFINITY;
            rec[e * (D + 2) + 1] = 0.f;
        }
        return;
    }
    for (int e = threadIdx.x; e < G * D; e += blockDim.x)
        Qs[e] = to_f(q[(b * H + (int64_t)g * G) * D + e]);
    stage_block<T, D>(kc + bg * (int64_t)Tmax * D, vc + bg * (int64_t)Tmax * D, blk, pos + 1, Kt, Vs);
    __syncthreads();
    for (int hh = warp; hh < G; hh += kWarps) {
        float m = -INFINITY, l = 0.f, acc[D / 32];
#pragma unroll
        for (int j = 0; j < D / 32; ++j) acc[j] = 0.f;
        fold_block<D>(Kt, Vs, Qs + hh * D, (int64_t)blk * kBlk, pos, scale, m, l, acc, lane);
        float* r = rec + hh * (D + 2);
        if (lane == 0) { r[0] = m; r[1] = l; }
#pragma unroll
        for (int j = 0; j < D / 32; ++j) r[2 + j * 32 + lane] = acc[j];
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(32)
sparse_decode_combine_kernel(const float* __restrict__ part, T* __restrict__ o, int H, int Hkv,
                             int slots) {
    const int lane = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / H;
    const int h = (int)(bh % H);
    const int G = H / Hkv;
    const int g = h / G, hh = h % G;
    const int64_t bg = b * Hkv + g;
    float M = -INFINITY;
    for (int s = 0; s < slots; ++s) M = fmaxf(M, part[((bg * slots + s) * G + hh) * (D + 2)]);
    float L = 0.f, acc[D / 32];
#pragma unroll
    for (int j = 0; j < D / 32; ++j) acc[j] = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < slots; ++s) {
            const float* r = part + ((bg * slots + s) * G + hh) * (D + 2);
            if (r[0] == -INFINITY) continue;
            const float w = expf(r[0] - M);
            L += w * r[1];
#pragma unroll
            for (int j = 0; j < D / 32; ++j) acc[j] = fmaf(w, r[2 + j * 32 + lane], acc[j]);
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) o[bh * D + j * 32 + lane] = from_f<T>(acc[j] * inv);
}

template <typename T, int D>
cudaError_t decode(const void* q, const void* kc, const void* vc, const int32_t* idx, void* o,
                   int B, int H, int Hkv, int pos, int Tmax, int slots, float scale, void* ws,
                   cudaStream_t st, DevCtx ctx) {
    auto kern = sparse_decode_partial_kernel<T, D>;
    const int G = H / Hkv;
    const size_t smem = BlockSmem<D>::bytes + sizeof(float) * G * D;
    cudaError_t e = ensure_smem<sparse_decode_partial_kernel<T, D>>((int)(BlockSmem<D>::bytes + sizeof(float) * 2 * kWarps * D));
    if (e != cudaSuccess) return e;
    float* part = static_cast<float*>(ws);
    kern<<<dim3(slots, B * Hkv), kWarps * 32, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(kc), static_cast<const T*>(vc), idx, part,
        H, Hkv, pos, Tmax, slots, scale, ctx);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sparse_decode_combine_kernel<T, D><<<B * H, 32, 0, st>>>(part, static_cast<T*>(o), H, Hkv, slots);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_prefill_simt(DType dt, const void* q, const void* k, const void* v,
                                       const int32_t* idx, void* o, int B, int H, int Hkv, int Hs,
                                       int N, int d, int slots, float scale, cudaStream_t st,
                                       DevCtx ctx) {
    if (H / Hs > 2 * kWarps) return cudaErrorNotSupported;
    if (dt == DType::F32)
        return d == 64 ? prefill<float, 64>(q, k, v, idx, o, B, H, Hkv, Hs, N, slots, scale, st, ctx)
                       : prefill<float, 128>(q, k, v, idx, o, B, H, Hkv, Hs, N, slots, scale, st, ctx);
    return d == 64 ? prefill<__nv_bfloat16, 64>(q, k, v, idx, o, B, H, Hkv, Hs, N, slots, scale, st, ctx)
                   : prefill<__nv_bfloat16, 128>(q, k, v, idx, o, B, H, Hkv, Hs, N, slots, scale, st, ctx);
}

size_t sparse_decode_attn_workspace(int B, int H, int Hkv, int slots, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0) return 0;
    return (size_t)B * Hkv * slots * (H / Hkv) * (d + 2) * sizeof(float);
}

cudaError_t launch_sparse_decode_attn(DType dt, const void* q, const void* kc, const void* vc,
                                      const int32_t* idx, void* o, int B, int H, int Hkv, int pos,
                                      int Tmax, int d, int slots, float scale, void* ws,
                                      cudaStream_t st, DevCtx ctx) {
    if (dt == DType::F32)
        return d == 64 ? decode<float, 64>(q, kc, vc, idx, o, B, H, Hkv, pos, Tmax, slots, scale, ws, st, ctx)
                       : decode<float, 128>(q, kc, vc, idx, o, B, H, Hkv, pos, Tmax, slots, scale, ws, st, ctx);
    return d == 64 ? decode<__nv_bfloat16, 64>(q, kc, vc, idx, o, B, H, Hkv, pos, Tmax, slots, scale, ws, st, ctx)
                   : decode<__nv_bfloat16, 128>(q, kc, vc, idx, o, B, H, Hkv, pos, Tmax, slots, scale, ws, st, ctx);
}

}  // namespace sala
