// Test-only library (libsala_selftest.so): one tcgen05 MMA tile through the same TMA, shared
// memory descriptor and TMEM paths the kernels use, so the tests can check each operand layout
// in isolation against a host product.
//
//   sala_selftest_mma(A, B, D, N, K, b_mn_major, a_mode, status, stream)
//     A : a_mode 0/1 -> [128, K] bf16, K contiguous; a_mode 2 -> [K, 128] bf16, M contiguous
//         (the MMA reads A transposed, "MN-major").
//     B : b_mn_major == 0 -> [N, K] bf16, K contiguous, and D = A B^T
//         b_mn_major == 1 -> [K, N] bf16, N contiguous, and D = A B
//     D : [128, N] fp32.   N in {64, 128, 256}, K in {64, 128}.
//     a_mode 1: A is first copied into TMEM (bf16 pairs packed per 32-bit column) and the
//     MMA reads it from there instead of shared memory.
//   Returns 0 on success, a negative value for bad arguments, or a CUDA error code.
//
//   sala_selftest_exp2_poly(y, out, n, stream)
//     out[i] = 2^y[i] through the FMA-pipe polynomial the softmax kernels use (fastexp.cuh), so
//     the tests can check it against an exact 2^y.  y, out: n fp32 values on the device.
#include "fastexp.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace sala {
namespace {

constexpr int kM = 128;

__global__ void __launch_bounds__(128)
selftest_mma_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                    const __nv_bfloat16* __restrict__ A, float* __restrict__ D, int N, int K,
                    int b_mn_major, int a_mode, DevCtx ctx) {
    const int a_tmem = a_mode == 1, a_mn = a_mode == 2;
    extern __shared__ uint8_t smraw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = sm;                  // K/64 sub-tiles of [128 rows x 128 B]
    uint8_t* sB = sm + 32768;          // K-major: K/64 x [N x 128 B]; MN-major: N/64 x [K x 128 B]
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (warp == 0) {
        ptx::tmem_alloc(&tmem_base, 512);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(&bar_tma, 1);
        ptx::mbar_init(&bar_mma, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tm = tmem_base;
    const uint32_t tD = tm;          // columns [0, N)
    const uint32_t tA_cols = tm + 256;  // columns [256, 256 + K/2)

    if (tid == 0) {
        const uint32_t bytes = (uint32_t)(kM * K * 2 + N * K * 2);
        ptx::mbar_arrive_expect_tx(&bar_tma, bytes);
        if (!a_mn) {
            for (int kb = 0; kb < K / 64; ++kb) ptx::tma_load_2d(sA + kb * kM * 128, &tA, &bar_tma, kb * 64, 0);
        } else {
            for (int mb = 0; mb < kM / 64; ++mb) ptx::tma_load_2d(sA + mb * K * 128, &tA, &bar_tma, mb * 64, 0);
        }
        if (!b_mn_major) {
            for (int kb = 0; kb < K / 64; ++kb) ptx::tma_load_2d(sB + kb * N * 128, &tB, &bar_tma, kb * 64, 0);
        } else {
            for (int nb = 0; nb < N / 64; ++nb) ptx::tma_load_2d(sB + nb * K * 128, &tB, &bar_tma, nb * 64, 0);
        }
    }
    if (a_tmem) {
        // Row `tid` of A into TMEM lane `tid`: column c holds elements (2c, 2c+1).
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
            for (int j = 0; j < 16; ++j) {
                const float lo = __bfloat162float(A[(int64_t)tid * K + 2 * (c0 + j)]);
                const float hi = __bfloat162float(A[(int64_t)tid * K + 2 * (c0 + j) + 1]);
                r[j] = ptx::pack_bf16x2(lo, hi);
            }
            ptx::tmem_st16(tA_cols + ptx::tmem_lane_base(warp) + c0, r);
        }
        ptx::tmem_st_wait();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    bool ok = ptx::mbar_wait(&bar_tma, 0, ctx);
    if (tid == 0 && ok) {
        const uint32_t idesc = ptx::idesc_bf16_f32(kM, N, a_mn != 0, b_mn_major != 0);
        const uint32_t a0 = ptx::smem_u32(sA), b0 = ptx::smem_u32(sB);
        for (int ks = 0; ks < K / 16; ++ks) {
            uint64_t bdesc;
            if (!b_mn_major)
                bdesc = ptx::sdesc_sw128(b0 + (ks / 4) * N * 128 + (ks % 4) * 32, 16, 1024);
            else
                bdesc = ptx::sdesc_sw128(b0 + ks * 16 * 128, (uint32_t)K * 128, 1024);
            if (a_tmem) {
                ptx::mma_ts(tD, tA_cols + ks * 8, bdesc, idesc, ks > 0);
            } else if (a_mn) {
                const uint64_t adesc = ptx::sdesc_sw128(a0 + ks * 16 * 128, (uint32_t)K * 128, 1024);
                ptx::mma_ss(tD, adesc, bdesc, idesc, ks > 0);
            } else {
                const uint64_t adesc = ptx::sdesc_sw128(a0 + (ks / 4) * kM * 128 + (ks % 4) * 32, 16, 1024);
                ptx::mma_ss(tD, adesc, bdesc, idesc, ks > 0);
            }
        }
        ptx::mma_commit(&bar_mma);
    }
    __syncthreads();
    if (ok) ok = ptx::mbar_wait(&bar_mma, 0, ctx);
    ptx::tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            ptx::tmem_ld16(tD + ptx::tmem_lane_base(warp) + c0, r);
            ptx::tmem_ld_wait();
            for (int j = 0; j < 16; ++j) D[(int64_t)tid * N + c0 + j] = __uint_as_float(r[j]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) ptx::tmem_dealloc(tm, 512);
}

}  // namespace
}  // namespace sala

extern "C" int sala_selftest_mma(const void* A, const void* B, float* D, int N, int K,
                                 int b_mn_major, int a_mode, unsigned* status, void* stream) {
    using namespace sala;
    if (!(N == 64 || N == 128 || N == 256) || !(K == 64 || K == 128) || !A || !B || !D || !status)
        return -1;
    CUtensorMap tA, tB;
    if (a_mode < 0 || a_mode > 2) return -1;
    cudaError_t e = a_mode == 2 ? make_tmap_bf16_2d(&tA, A, kM, K, kM, 64, K)
                                : make_tmap_bf16_2d(&tA, A, K, kM, K, 64, kM);
    if (e != cudaSuccess) return -2;
    if (!b_mn_major)
        e = make_tmap_bf16_2d(&tB, B, K, N, K, 64, N);
    else
        e = make_tmap_bf16_2d(&tB, B, N, K, N, 64, K);
    if (e != cudaSuccess) return -3;
    const size_t smem = 1024 + 32768 + 65536;
    e = cudaFuncSetAttribute(selftest_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    DevCtx ctx{status, 1000000000ull};
    selftest_mma_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        tA, tB, static_cast<const __nv_bfloat16*>(A), D, N, K, b_mn_major, a_mode, ctx);
    return (int)cudaGetLastError();
}

namespace {
__global__ void exp2_poly_kernel(const float* __restrict__ y, float* __restrict__ out, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    float a = y[i], b = i + 1 < n ? y[i + 1] : 0.f;
    sala::exp2_poly2(a, b);
    out[i] = a;
    if (i + 1 < n) out[i + 1] = b;
}
}  // namespace

extern "C" int sala_selftest_exp2_poly(const float* y, float* out, int n, void* stream) {
    if (n < 0 || (n > 0 && (!y || !out))) return -1;
    if (n == 0) return 0;
    const int threads = 256, pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(y, out, n);
    return (int)cudaGetLastError();
}
