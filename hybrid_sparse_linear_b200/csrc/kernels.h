// Internal launchers of libsala.  Each returns the CUDA error of its launch(es).  Arguments are
// validated by api.cu before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sala.h"
#include "common.cuh"

namespace sala {

enum class DType { F32 = 0, BF16 = 1 };

// Linear attention.  rope: rotary position embedding of q and k (off when base <= 0); row r of
// a prefill sits at position pos0 + r, a decode step at pos0.
struct Rope {
    double base;
    int64_t pos0;
};
cudaError_t launch_linear_prefill_simt(DType dt, const void* q, const void* k, const void* v,
                                       const float* decay, void* o, const float* s_in,
                                       float* s_out, int B, int H, int N, int d, Rope rope,
                                       cudaStream_t st, DevCtx ctx);
// bf16, d = 128.  With a workspace of linear_prefill_tc_workspace(...) bytes (0 = not needed) the
// sequence is split into segments processed in parallel (state pass, chaining, output pass);
// without it, or when one segment is best, a single pass over the whole sequence.
size_t linear_prefill_tc_workspace(int B, int H, int N, int d);
cudaError_t launch_linear_prefill_tc(const void* q, const void* k, const void* v,
                                     const float* decay, void* o, const float* s_in,
                                     float* s_out, int B, int H, int N, int d, void* ws,
                                     size_t ws_bytes, Rope rope, cudaStream_t st, DevCtx ctx);
bool linear_prefill_tc_supported(int d);
// pdl: launched as a programmatic dependent of the previous kernel in the stream (the state is
// read before that kernel completes; it must not write this state).
cudaError_t launch_linear_decode(DType dt, const void* q, const void* k, const void* v,
                                 const float* decay, float* state, void* o, int B, int H, int d,
                                 Rope rope, bool pdl, cudaStream_t st, DevCtx ctx);

// Sparse attention.
cudaError_t launch_block_compress(DType dt, const void* k, void* kbar, int B, int Hkv, int N,
                                  int d, int first_block, int n_blocks, int nb_cap,
                                  cudaStream_t st, DevCtx ctx);
// Query-block-granular selection: one row per (batch, KV group, 64-token query block), written
// to every token row of the block.
cudaError_t launch_block_topk_qblock(DType dt, const void* q, const void* kbar, int32_t* idx, int B,
                                     int H, int Hkv, int Nq, int nb, int d, int topk, int n_init,
                                     int n_local, cudaStream_t st, DevCtx ctx);
// The same granularity scored by softmax-probability group aggregation (G <= 16).
cudaError_t launch_block_topk_qblock_softmax(DType dt, const void* q, const void* kbar, int32_t* idx,
                                             int B, int H, int Hkv, int Nq, int nb, int d, int topk,
                                             int n_init, int n_local, float scale, cudaStream_t st,
                                             DevCtx ctx);
// Hs = selection groups per batch: Hkv (the group-summed query of each KV group) or H (one
// selection per query head, each scored with its KV head's kbar); idx is [B, Hs, Nq, slots].
cudaError_t launch_block_topk_tiled(DType dt, const void* q, const void* kbar, int32_t* idx,
                                    int B, int H, int Hkv, int Hs, int Nq, int q_pos0, int nb,
                                    int d, int topk, int n_init, int n_local, cudaStream_t st,
                                    DevCtx ctx);
// Tensor-core selection (bf16, d 128, prefill rows from position 0, topk <= 64).
bool block_topk_tc_supported(int H, int Hkv, int Nq, int q_pos0, int nb, int d, int topk);
cudaError_t launch_block_topk_tc(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                 int Hkv, int Hs, int Nq, int nb, int topk, int n_init,
                                 int n_local, cudaStream_t st, DevCtx ctx);
// Row-wise selection for few query rows and many blocks: candidates split across CTAs, then a
// merge.  Workspace = rowwise_topk_workspace(...) bytes.
size_t rowwise_topk_workspace(int B, int Hkv, int Nq, int q_pos0, int topk);
cudaError_t launch_block_topk_rowwise(DType dt, const void* q, const void* kbar, int32_t* idx,
                                      int B, int H, int Hkv, int Nq, int q_pos0, int nb, int d,
                                      int topk, int n_init, int n_local, void* ws,
                                      cudaStream_t st, DevCtx ctx);
// Hs as in the selection: idx [B, Hs, N, slots] is shared by the H / Hs heads of a selection
// group (Hs = Hkv: the KV group; Hs = H: a selection per query head).
cudaError_t launch_sparse_prefill_simt(DType dt, const void* q, const void* k, const void* v,
                                       const int32_t* idx, void* o, int B, int H, int Hkv, int Hs,
                                       int N, int d, int slots, float scale, cudaStream_t st,
                                       DevCtx ctx);
// lse (may be null): the training forward -- per query row the natural log-sum-exp of its
// visible scaled logits, P V taken as P_hi V + P_lo V, and (o_lo, may be null) the bf16 rounding
// residual of o.
// per_head: idx is [B, H, N, slots], a selection per query head (forward only: lse and o_lo
// null); N <= 2^20.
cudaError_t launch_sparse_prefill_tc(const void* q, const void* k, const void* v,
                                     const int32_t* idx, void* o, float* lse, void* o_lo, int B,
                                     int H, int Hkv, int N, int d, int slots, float scale,
                                     bool per_head, cudaStream_t st, DevCtx ctx);

// Sparse attention backward (bf16, G = 16, d = 128), selection held fixed.
// The transposed selection: for key k = ((b * Hkv + g) * n_chunks + chunk) * nb + j,
// list[off[k] .. off[k+1]) holds the query tokens of the chunk (kChunkTok tokens) whose selection
// row holds block j; off[n_keys] is the total.  item_key[it] is the list holding position
// it * kItem (the key side's unit of work).
constexpr int kChunkTok = 8192;
constexpr int kItem = 512;
struct SparseBwdCsr {
    int nb, n_chunks, n_keys, n_items;
    int *cnt, *cur, *off, *list, *item_key, *bsum;
    size_t bytes;  // workspace bytes the arrays take
};
SparseBwdCsr sparse_bwd_csr_layout(void* ws, int B, int Hkv, int N, int slots);
cudaError_t launch_sparse_bwd_csr(const int32_t* idx, int B, int Hkv, int N, int slots,
                                  const SparseBwdCsr& c, cudaStream_t st, DevCtx ctx);
// delta[row] = sum_c (o + o_lo)[row, c] * dout[row, c] in fp32, rows of 128 bf16 (o_lo may be
// null).
cudaError_t launch_sparse_bwd_delta(const void* o, const void* o_lo, const void* dout,
                                    float* delta, int64_t rows, cudaStream_t st);
// dq (bf16) from the query side: the forward's units walking the union of their selections.
cudaError_t launch_sparse_dq_tc(const void* q, const void* k, const void* v, const void* dout,
                                const int32_t* idx, const float* lse, const float* delta, void* dq,
                                int B, int H, int Hkv, int N, int slots, float scale,
                                cudaStream_t st, DevCtx ctx);
// dk_acc, dv_acc (fp32, zeroed by the caller) += the key side: key blocks walking their
// transposed lists; unscaled (dk_acc holds sum_i dS_ij q_i).
cudaError_t launch_sparse_dkv_tc(const void* q, const void* k, const void* v, const void* dout,
                                 const float* lse, const float* delta, const SparseBwdCsr& c,
                                 float* dk_acc, float* dv_acc, int B, int H, int Hkv, int N,
                                 float scale, cudaStream_t st, DevCtx ctx);
// dk = bf16(scale * dk_acc), dv = bf16(dv_acc); n elements, a multiple of 4.
cudaError_t launch_sparse_bwd_finish(const float* dk_acc, const float* dv_acc, void* dk, void* dv,
                                     int64_t n, float scale, cudaStream_t st);
bool sparse_prefill_tc_supported(int H, int Hkv, int d);
size_t sparse_decode_attn_workspace(int B, int H, int Hkv, int slots, int d);
// Sparse decode in one cooperative launch (scoring, top-k, attention, combine).  Returns
// cudaErrorNotSupported, launching nothing, when the problem does not fit it (k > 64, more than
// 80 slots, more than 16 heads per group, more than 8192 span-list keys, a grid that cannot be
// resident at once, or a smaller workspace); the caller then uses the multi-kernel path.
// Workspace: [0, 256) barrier words (zero before the first call, left zero), then its data.
size_t sparse_decode_fused_workspace(int B, int H, int Hkv, int pos, int topk, int n_init,
                                     int n_local, int d);
// Paged KV cache and per-sequence positions for the one-launch decode (all null / 0: the dense
// cache [B * Hkv][Tmax][d] and the launch's pos for every sequence).  pos_b: [B] device positions,
// each at most the launch's pos; pages: [B][max_pages] device page ids, page p holding the 64 rows
// of one block for every KV head, [n_pages][Hkv][64][d].
struct DecodePaging {
    const int32_t* pos_b;
    const int32_t* pages;
    int max_pages;
    int n_pages;
};
cudaError_t launch_sparse_decode_fused(DType dt, const void* q, const void* kc, const void* vc,
                                       const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                       void* o, int B, int H, int Hkv, int pos, int Tmax,
                                       int nb_cap, int d, int topk, int n_init, int n_local,
                                       float scale, void* ws, size_t ws_bytes, DecodePaging pg, cudaStream_t st,
                                       DevCtx ctx);
// Sparse decode in two launches (bf16, d 64 or 128, dense cache, one position): a score kernel over
// every SM (k_bar prefetched into shared memory, each CTA's best keys stored) and an attend kernel of
// one 16-CTA cluster per (batch, KV group) that ranks the stored keys, attends the winners and
// combines the partials in distributed shared memory.  pdl: the first launch is a programmatic
// dependent of the previous kernel (k_bar is read before that kernel completes).  Returns
// cudaErrorNotSupported, launching nothing, when the problem does not fit (k > 64, more than 80
// slots, more than 16 heads per group, more than 16 groups or more than the GPU holds clusters, a
// scoring CTA's share of k_bar above its shared memory, or a smaller workspace).  ws: the path's own
// bytes, written before they are read within each call (no initial value needed).
size_t sparse_decode_pf_workspace(int B, int H, int Hkv, int pos, int topk, int n_init, int n_local,
                                  int d);
cudaError_t launch_sparse_decode_pf(DType dt, const void* q, const void* kc, const void* vc,
                                    const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                    void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap,
                                    int d, int topk, int n_init, int n_local, float scale, void* ws,
                                    size_t ws_bytes, bool pdl, cudaStream_t st, DevCtx ctx);
cudaError_t launch_sparse_decode_attn(DType dt, const void* q, const void* kc, const void* vc,
                                      const int32_t* idx, void* o, int B, int H, int Hkv,
                                      int pos, int Tmax, int d, int slots, float scale, void* ws,
                                      cudaStream_t st, DevCtx ctx);

// Row reversal of [BH][N][d] tensors (out must not overlap in).
cudaError_t launch_flip_rows(DType dt, const void* in, void* out, int64_t BH, int N, int d,
                             cudaStream_t st);

// Weight-free RMS normalisation of q rows [0, q_rows) and k rows [0, k_rows), d elements each;
// outputs may alias their inputs exactly.
cudaError_t launch_qk_norm(DType dt, const void* q, void* q_out, int64_t q_rows, const void* k,
                           void* k_out, int64_t k_rows, int d, float eps, cudaStream_t st);
// The same pass with an optional RoPE: eps > 0 normalises, rope_base > 0 rotates (row r of a
// [B, heads, N, d] tensor at position pos0 + r % N); at least one of the two.
cudaError_t launch_qk_prologue(DType dt, const void* q, void* q_out, int64_t q_rows, const void* k,
                               void* k_out, int64_t k_rows, int d, float eps, int N, int64_t pos0,
                               double rope_base, cudaStream_t st);

// Diagnostics.
cudaError_t launch_selftest_wait(cudaStream_t st, DevCtx ctx);

// Sets the calling thread's sala_last_error() message (printf-style).
void set_last_error(const char* fmt, ...);

// Body of sala_sparse_decode; zero_barrier additionally zeroes the workspace's first 256 bytes on
// the stream after validation, before the kernels; pdl launches the prefetching one-launch kernel
// as a programmatic dependent of the previous kernel (other paths launch as usual).
sala_status sparse_decode_impl(const void* q, const void* kcache, const void* vcache,
                               const void* kbar, const int32_t* idx_in, int32_t* idx_out, void* o,
                               int B, int H, int Hkv, int pos, int Tmax, int nb_cap, int d,
                               int block, int topk, int n_init, int n_local, float scale,
                               void* workspace, size_t workspace_bytes, sala_dtype dt,
                               sala_stream stream, bool zero_barrier, bool pdl);

}  // namespace sala
