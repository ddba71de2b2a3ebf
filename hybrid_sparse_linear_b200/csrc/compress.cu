// Block compression: kbar[b, g, j] = mean of the 64 keys of block j, rounded once.
//
// One warp per (batch*KV head, block).  Each lane owns d/32 adjacent columns; the warp reads the
// block row by row (one coalesced d-wide row per step) and accumulates in fp64, which is exact
// for sums of 64 bf16 values, so the single final rounding matches the definition bit for bit.
#include "kernels.h"

namespace sala {
namespace {

constexpr int kBlock = 64;

template <typename T, int D>
__global__ void __launch_bounds__(256)
block_compress_kernel(const T* __restrict__ k, T* __restrict__ kbar, int N, int first_block,
                      int n_blocks, int nb_cap, DevCtx ctx) {
    constexpr int kPer = D / 32;
    const int lane = threadIdx.x & 31;
    const int nbi = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (nbi >= n_blocks) return;
    const int64_t bg = blockIdx.y;
    const int blk = first_block + nbi;
    if (!in_bounds(ctx, blk < nb_cap && ((int64_t)blk + 1) * kBlock <= N)) return;
    const T* src = k + (bg * N + (int64_t)blk * kBlock) * D + lane * kPer;
    double acc[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[j] = 0.0;
#pragma unroll 4
    for (int t = 0; t < kBlock; ++t) {
#pragma unroll
        for (int j = 0; j < kPer; ++j) acc[j] += (double)to_f(src[(int64_t)t * D + j]);
    }
    T* dst = kbar + (bg * nb_cap + blk) * D + lane * kPer;
#pragma unroll
    for (int j = 0; j < kPer; ++j) dst[j] = round_from_double<T>(acc[j] * (1.0 / kBlock));
}

template <typename T, int D>
cudaError_t launch(const void* k, void* kbar, int B, int Hkv, int N, int first_block, int n_blocks,
                   int nb_cap, cudaStream_t st, DevCtx ctx) {
    dim3 grid(ceil_div(n_blocks, 8), (unsigned)(B * Hkv));
    block_compress_kernel<T, D><<<grid, 256, 0, st>>>(static_cast<const T*>(k), static_cast<T*>(kbar),
                                                      N, first_block, n_blocks, nb_cap, ctx);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_compress(DType dt, const void* k, void* kbar, int B, int Hkv, int N, int d,
                                  int first_block, int n_blocks, int nb_cap, cudaStream_t st,
                                  DevCtx ctx) {
    if (dt == DType::F32)
        return d == 64 ? launch<float, 64>(k, kbar, B, Hkv, N, first_block, n_blocks, nb_cap, st, ctx)
                       : launch<float, 128>(k, kbar, B, Hkv, N, first_block, n_blocks, nb_cap, st, ctx);
    return d == 64 ? launch<__nv_bfloat16, 64>(k, kbar, B, Hkv, N, first_block, n_blocks, nb_cap, st, ctx)
                   : launch<__nv_bfloat16, 128>(k, kbar, B, Hkv, N, first_block, n_blocks, nb_cap, st, ctx);
}

}  // namespace sala
