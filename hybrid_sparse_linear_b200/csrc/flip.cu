// Reversal of the row order of [BH][N][d] tensors: out[bh][N - 1 - i] = in[bh][i].  The backward
// pass of the linear attention runs the anti-causal sums (dk, dv) as forward linear attentions of
// the reversed sequence.  One thread per 16 bytes; rows are 128 (fp32 d 64 / bf16 d 128) to 512
// bytes, so a warp moves whole rows and the access stays coalesced.
#include <algorithm>

#include "kernels.h"

namespace sala {
namespace {

__global__ void flip_rows_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t BH,
                                 int N, int vec_per_row) {
    const int64_t total = BH * (int64_t)N * vec_per_row;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / vec_per_row;
        const int c = (int)(e % vec_per_row);
        const int64_t bh = row / N;
        const int i = (int)(row % N);
        out[(bh * N + (N - 1 - i)) * vec_per_row + c] = in[e];
    }
}

}  // namespace

cudaError_t launch_flip_rows(DType dt, const void* in, void* out, int64_t BH, int N, int d,
                             cudaStream_t st) {
    const int esize = dt == DType::F32 ? 4 : 2;
    const int vec_per_row = d * esize / 16;
    const int64_t total = BH * (int64_t)N * vec_per_row;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((total + threads - 1) / threads, 148 * 16);
    flip_rows_kernel<<<(unsigned)blocks, threads, 0, st>>>(static_cast<const uint4*>(in),
                                                          static_cast<uint4*>(out), BH, N,
                                                          vec_per_row);
    return cudaGetLastError();
}

}  // namespace sala
