// Linear (Lightning-style) attention on CUDA cores: the fp32 prefill and the decode step.
//
// Prefill is the chunked form of o_i = sum_{j<=i} lambda^{i-j} (q_i.k_j) v_j: per chunk of C
// rows, an intra-chunk decay-masked product plus the carried d x d state.  One CTA owns one
// (batch, head, slice of DV value columns) and walks the chunks in order; S[:, slice] evolves
// independently of the other slices, so slices run in parallel with no communication.
#include "kernels.h"
#include "rope.cuh"

namespace sala {
namespace {

constexpr int kC = 64;        // chunk rows
constexpr int kThreads = 256;

template <int D, int DV>
struct PrefillSmem {
    static constexpr int kQK = kC * (D + 1);
    static constexpr size_t bytes = sizeof(double) * (D / 2) +  // RoPE turns per frequency
        sizeof(float) * (2 * kQK + kC * DV + kC * (kC + 1) + D * DV + (kC + 1));
};

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads)
linear_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                           const T* __restrict__ v, const float* __restrict__ decay,
                           T* __restrict__ o, const float* s_in, float* s_out, int H, int N,
                           Rope rope) {
    extern __shared__ double smd[];
    double* turn = smd;                     // [D/2]  theta_i / 2pi (RoPE)
    float* sm = reinterpret_cast<float*>(smd + D / 2);
    float* Qs = sm;                         // [C][D+1]
    float* Ks = Qs + kC * (D + 1);          // [C][D+1]
    float* Vs = Ks + kC * (D + 1);          // [C][DV]
    float* As = Vs + kC * DV;               // [C][C+1]
    float* Ss = As + kC * (kC + 1);         // [D][DV]  state slice
    float* pw = Ss + D * DV;                // [C+1]    lambda^n

    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * DV;         // first value column of this slice
    const int64_t bh = blockIdx.y;
    const int h = (int)(bh % H);
    const float lam = decay[h];
    for (int n = tid; n <= kC; n += kThreads) pw[n] = (float)pow((double)lam, (double)n);
    const bool use_rope = rope.base > 0.0;
    if (use_rope)
        for (int i = tid; i < D / 2; i += kThreads) turn[i] = rope_turn(rope.base, i, D);
    for (int e = tid; e < D * DV; e += kThreads) {
        const int a = e / DV, c = e % DV;
        Ss[e] = s_in ? s_in[(bh * D + a) * D + c0 + c] : 0.f;
    }
    const T* qb = q + bh * (int64_t)N * D;
    const T* kb = k + bh * (int64_t)N * D;
    const T* vb = v + bh * (int64_t)N * D;
    T* ob = o + bh * (int64_t)N * D;

    for (int r0 = 0; r0 < N; r0 += kC) {
        const int len = min(kC, N - r0);
        __syncthreads();
        if (use_rope) {  // rotate-half pairs (i, i + D/2) of q and k at position pos0 + row
            for (int e = tid; e < kC * (D / 2); e += kThreads) {
                const int t = e / (D / 2), i = e % (D / 2);
                const bool ok = t < len;
                const int64_t base = (int64_t)(r0 + t) * D;
                float q0 = ok ? to_f(qb[base + i]) : 0.f, q1 = ok ? to_f(qb[base + i + D / 2]) : 0.f;
                float k0 = ok ? to_f(kb[base + i]) : 0.f, k1 = ok ? to_f(kb[base + i + D / 2]) : 0.f;
                float c, s;
                rope_cs(turn[i], rope.pos0 + r0 + t, c, s);
                rope_rot(q0, q1, c, s);
                rope_rot(k0, k1, c, s);
                Qs[t * (D + 1) + i] = q0;
                Qs[t * (D + 1) + i + D / 2] = q1;
                Ks[t * (D + 1) + i] = k0;
                Ks[t * (D + 1) + i + D / 2] = k1;
            }
        } else {
            for (int e = tid; e < kC * D; e += kThreads) {
                const int t = e / D, a = e % D;
                const bool ok = t < len;
                Qs[t * (D + 1) + a] = ok ? to_f(qb[(int64_t)(r0 + t) * D + a]) : 0.f;
                Ks[t * (D + 1) + a] = ok ? to_f(kb[(int64_t)(r0 + t) * D + a]) : 0.f;
            }
        }
        for (int e = tid; e < kC * DV; e += kThreads) {
            const int t = e / DV, c = e % DV;
            Vs[e] = t < len ? to_f(vb[(int64_t)(r0 + t) * D + c0 + c]) : 0.f;
        }
        __syncthreads();
        // Intra-chunk scores, decay-masked: A[t][s] = lambda^{t-s} q_t.k_s for s <= t.
        {
            const int t = tid >> 2;
            for (int m = 0; m < kC / 4; ++m) {
                const int s = (tid & 3) + 4 * m;
                float acc = 0.f;
                if (s <= t) {
                    const float* qr = Qs + t * (D + 1);
                    const float* kr = Ks + s * (D + 1);
#pragma unroll 8
                    for (int a = 0; a < D; ++a) acc = fmaf(qr[a], kr[a], acc);
                    acc *= pw[t - s];
                }
                As[t * (kC + 1) + s] = acc;
            }
        }
        __syncthreads();
        // o_t = A[t,:] V + lambda^{t+1} q_t S.
        {
            const int t = tid >> 2;
            if (t < len) {
                for (int m = 0; m < DV / 4; ++m) {
                    const int c = (tid & 3) + 4 * m;
                    float intra = 0.f, inter = 0.f;
                    for (int s = 0; s <= t; ++s) intra = fmaf(As[t * (kC + 1) + s], Vs[s * DV + c], intra);
                    const float* qr = Qs + t * (D + 1);
#pragma unroll 8
                    for (int a = 0; a < D; ++a) inter = fmaf(qr[a], Ss[a * DV + c], inter);
                    ob[(int64_t)(r0 + t) * D + c0 + c] = from_f<T>(intra + pw[t + 1] * inter);
                }
            }
        }
        __syncthreads();
        // S <- lambda^len S + sum_s lambda^{len-1-s} k_s^T v_s.
        {
            constexpr int kPer = D * DV / kThreads;
            const int a = (tid * kPer) / DV;
            const int cb = (tid * kPer) % DV;
            float acc[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) acc[j] = pw[len] * Ss[a * DV + cb + j];
            for (int s = 0; s < len; ++s) {
                const float w = pw[len - 1 - s] * Ks[s * (D + 1) + a];
#pragma unroll
                for (int j = 0; j < kPer; ++j) acc[j] = fmaf(w, Vs[s * DV + cb + j], acc[j]);
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) Ss[a * DV + cb + j] = acc[j];
        }
    }
    __syncthreads();
    if (s_out)
        for (int e = tid; e < D * DV; e += kThreads) {
            const int a = e / DV, c = e % DV;
            s_out[(bh * D + a) * D + c0 + c] = Ss[e];
        }
}

template <typename T, int D>
cudaError_t prefill_simt(const void* q, const void* k, const void* v, const float* decay, void* o,
                         const float* s_in, float* s_out, int B, int H, int N, Rope rope,
                         cudaStream_t st) {
    constexpr int DV = 32;
    auto kern = linear_prefill_simt_kernel<T, D, DV>;
    const size_t smem = PrefillSmem<D, DV>::bytes;
    cudaError_t e = ensure_smem<linear_prefill_simt_kernel<T, D, DV>>((int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(D / DV, (unsigned)(B * H));
    kern<<<grid, kThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                       static_cast<const T*>(v), decay, static_cast<T*>(o), s_in,
                                       s_out, H, N, rope);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Decode: S <- lambda S + k^T v ; o = q S.  One CTA per (batch*head, 16-column slice); thread
// (a, half) owns row a of the slice, 8 columns, loaded and stored as two float4.
// kPdl: launched as a programmatic dependent of the previous kernel in the stream.  The state
// row is requested first, while that kernel may still run (the caller guarantees it does not
// write this state); q, k, v and the decays are read after griddepcontrol.wait, i.e. after it
// has completed and its writes are visible.  Before the wait their lines are only pulled into
// L2: L2 is where every SM's writes land, so a line fetched there early is updated by any later
// write of the previous kernel, and nothing is held in this SM's L1 or registers.  Only after the
// wait may the next kernel launch, so a dependent's early reads overlap this kernel alone, never
// the one before it.
template <typename T, int D, bool kRope, bool kPdl>
__global__ void __launch_bounds__(2 * D)
linear_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ decay, float* __restrict__ state,
                     T* __restrict__ o, int H, Rope rope) {
    constexpr int kCols = 16;
    constexpr int kWarps = 2 * D / 32;
    __shared__ float red[kWarps][kCols];
    const int tid = threadIdx.x;
    const int a = tid >> 1, half = tid & 1;
    const int64_t bh = blockIdx.y;
    const int c0 = blockIdx.x * kCols + half * 8;
    float4* row = reinterpret_cast<float4*>(state + (bh * D + a) * D + c0);
    float4 s0 = row[0], s1 = row[1];
    if constexpr (kPdl) {
        constexpr int kLines = D * (int)sizeof(T) / 128;  // 128-byte lines of a q or k row
        const void* line = nullptr;
        if (tid < kLines) line = reinterpret_cast<const char*>(q + bh * D) + 128 * tid;
        else if (tid < 2 * kLines) line = reinterpret_cast<const char*>(k + bh * D) + 128 * (tid - kLines);
        else if (tid == 2 * kLines) line = v + bh * D + blockIdx.x * kCols;
        else if (tid == 2 * kLines + 1) line = decay + bh % H;
        if (line != nullptr) asm volatile("prefetch.global.L2 [%0];" ::"l"(line));
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    const float lam = decay[bh % H];
    float ka = to_f(k[bh * D + a]);
    float qa = to_f(q[bh * D + a]);
    if constexpr (kRope) {  // rotate-half pair (a, a +- D/2) at position pos0
        const int i = a % (D / 2), partner = a < D / 2 ? a + D / 2 : a - D / 2;
        const float kp = to_f(k[bh * D + partner]), qp = to_f(q[bh * D + partner]);
        float c, s;
        rope_cs(rope_turn(rope.base, i, D), rope.pos0, c, s);
        if (a >= D / 2) s = -s;  // x'_hi = x_hi c + x_lo s;  x'_lo = x_lo c - x_hi s
        ka = ka * c - kp * s;
        qa = qa * c - qp * s;
    }
    float vv[8];
    if constexpr (sizeof(T) == 2) {  // the 8 values as one 16-byte load (c0 is a multiple of 8)
        const uint4 raw = *reinterpret_cast<const uint4*>(v + bh * D + c0);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            vv[2 * j] = __uint_as_float(w[j] << 16);
            vv[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) vv[j] = to_f(v[bh * D + c0 + j]);
    }
    float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    float part[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sv[j] = fmaf(lam, sv[j], ka * vv[j]);
        part[j] = qa * sv[j];
    }
    row[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
    row[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
    // Sum part[] over the 16 rows of this warp that share `half`, then over warps.
#pragma unroll
    for (int j = 0; j < 8; ++j)
        for (int off = 2; off < 32; off <<= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
    const int lane = tid & 31, w = tid >> 5;
    if (lane < 2)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[w][lane * 8 + j] = part[j];
    __syncthreads();
    if (tid < kCols) {
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) acc += red[ww][tid];
        o[bh * D + blockIdx.x * kCols + tid] = from_f<T>(acc);
    }
}

template <typename T, int D, bool kRope>
cudaError_t decode_launch_pdl(const void* q, const void* k, const void* v, const float* decay,
                              float* state, void* o, int H, Rope rope, dim3 grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(2 * D);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, linear_decode_kernel<T, D, kRope, true>,
                              static_cast<const T*>(q), static_cast<const T*>(k),
                              static_cast<const T*>(v), decay, state, static_cast<T*>(o), H, rope);
}

template <typename T, int D>
cudaError_t decode_launch(const void* q, const void* k, const void* v, const float* decay,
                          float* state, void* o, int B, int H, Rope rope, bool pdl,
                          cudaStream_t st) {
    dim3 grid(D / 16, (unsigned)(B * H));
    if (pdl)
        return rope.base > 0.0 ? decode_launch_pdl<T, D, true>(q, k, v, decay, state, o, H, rope, grid, st)
                               : decode_launch_pdl<T, D, false>(q, k, v, decay, state, o, H, rope, grid, st);
    if (rope.base > 0.0)
        linear_decode_kernel<T, D, true, false><<<grid, 2 * D, 0, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), decay,
            state, static_cast<T*>(o), H, rope);
    else
        linear_decode_kernel<T, D, false, false><<<grid, 2 * D, 0, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), decay,
            state, static_cast<T*>(o), H, rope);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_linear_prefill_simt(DType dt, const void* q, const void* k, const void* v,
                                       const float* decay, void* o, const float* s_in,
                                       float* s_out, int B, int H, int N, int d, Rope rope,
                                       cudaStream_t st, DevCtx) {
    if (N == 0) {
        // Nothing to attend to: the state passes through unchanged (or stays zero).
        if (!s_out) return cudaSuccess;
        const size_t bytes = (size_t)B * H * d * d * sizeof(float);
        if (s_in) return s_in == s_out ? cudaSuccess
                                       : cudaMemcpyAsync(s_out, s_in, bytes, cudaMemcpyDeviceToDevice, st);
        return cudaMemsetAsync(s_out, 0, bytes, st);
    }
    if (dt == DType::F32)
        return d == 64 ? prefill_simt<float, 64>(q, k, v, decay, o, s_in, s_out, B, H, N, rope, st)
                       : prefill_simt<float, 128>(q, k, v, decay, o, s_in, s_out, B, H, N, rope, st);
    return d == 64 ? prefill_simt<__nv_bfloat16, 64>(q, k, v, decay, o, s_in, s_out, B, H, N, rope, st)
                   : prefill_simt<__nv_bfloat16, 128>(q, k, v, decay, o, s_in, s_out, B, H, N, rope, st);
}

cudaError_t launch_linear_decode(DType dt, const void* q, const void* k, const void* v,
                                 const float* decay, float* state, void* o, int B, int H, int d,
                                 Rope rope, bool pdl, cudaStream_t st, DevCtx) {
    if (dt == DType::F32)
        return d == 64 ? decode_launch<float, 64>(q, k, v, decay, state, o, B, H, rope, pdl, st)
                       : decode_launch<float, 128>(q, k, v, decay, state, o, B, H, rope, pdl, st);
    return d == 64 ? decode_launch<__nv_bfloat16, 64>(q, k, v, decay, state, o, B, H, rope, pdl, st)
                   : decode_launch<__nv_bfloat16, 128>(q, k, v, decay, state, o, B, H, rope, pdl, st);
}

}  // namespace sala
