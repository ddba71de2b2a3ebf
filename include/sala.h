/*
 * sala.h -- C ABI of the SALA hybrid attention forward for NVIDIA B200 (sm_100a).
 *
 * MiniCPM-SALA mixes two attentions layer by layer, one sparse layer to three linear ones
 * ("MiniCPM-SALA: Hybridizing Sparse and Linear Attention for Efficient Long-Context Modeling",
 * abstract; gist.science technical summaries, section 2 "Method", subsection "hybrid attention"):
 *   - Lightning Attention, a linear attention with a recursive O(N) form   -> sala_linear_*
 *   - InfLLM-V2 sparse attention over a dense KV cache                       -> sala_block_*,
 *                                                                               sala_sparse_*
 * The pages give no formula for either; the operations below are the plain readings:
 *   linear:  o_i = sum_{j<=i} lambda_h^{i-j} (q_i . k_j) v_j   (plus a carried d x d state)
 *   sparse:  mean-pooled block keys, per-query top-k block selection that always keeps the init
 *            and local blocks, then exact causal softmax attention over the selected blocks.
 *
 * Conventions shared by every call
 *   - Tensors are dense, row-major [B, heads, rows, d] in device memory ("device pointer").
 *     Query heads h of batch b use KV head h / (H / Hkv) (grouped-query attention).
 *   - dt selects the element type of q/k/v/o/kbar: SALA_BF16 (tensor-core kernels, fp32
 *     accumulation, bf16 output) or SALA_F32 (CUDA-core fp32 kernels).  Decays, linear states and
 *     softmax statistics are always fp32.
 *   - stream is a cudaStream_t (NULL = the legacy default stream).  Every call only enqueues
 *     work and returns; results are ready when the stream reaches that point.
 *   - Ownership: the caller allocates and frees every buffer, workspace included.  The library
 *     keeps no allocation of its own; its only global state is one per-device status word.
 *   - Errors: arguments are checked on the host before anything is launched.  A bad argument
 *     returns SALA_ERR_INVALID_ARG, a valid but unimplemented case SALA_ERR_UNSUPPORTED, and in
 *     both cases nothing is launched.  A failed launch returns SALA_ERR_CUDA.  Faults detected
 *     on the device (a bounded wait that expired, an index out of range) are recorded in the
 *     status word and reported by sala_check_status.  No call aborts or throws.
 *     sala_last_error() gives a one-line explanation of the calling thread's last failure.
 *   - Empty problems (B, H, N or Nq equal to 0) return SALA_OK and launch nothing.
 */
#ifndef SALA_H_
#define SALA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SALA_OK = 0,
    SALA_ERR_INVALID_ARG = 1,
    SALA_ERR_UNSUPPORTED = 2,
    SALA_ERR_CUDA = 3,
    SALA_ERR_TIMEOUT = 4,
    SALA_ERR_BOUNDS = 5
} sala_status;

typedef enum { SALA_F32 = 0, SALA_BF16 = 1 } sala_dtype;

typedef void* sala_stream; /* a cudaStream_t */

/* ------------------------------------------------------------------------------------------
 * Linear attention prefill (Lightning-style, chunked).  Pages: abstract ("linear attention
 * (Lightning Attention)"), DE technical summary section 2 ("recursive formulations", O(N)).
 *
 *   o_i     = sum_{j<=i} lambda_h^{i-j} (q_i . k_j) v_j  +  lambda_h^{i+1} q_i S_in
 *   S_out   = lambda_h^N S_in + sum_{j<N} lambda_h^{N-1-j} k_j^T v_j
 *
 * q, k, v, o : [B, H, N, d] device, dt.  No feature map, no normalisation of o.
 * decay      : [H] fp32 device, lambda_h in [0, 1].
 * state_in   : [B, H, d, d] fp32 device or NULL (NULL = zero state).  Row index = key dim.
 * state_out  : [B, H, d, d] fp32 device or NULL; may equal state_in (updated in place).
 * chunk      : length of the chunks of the chunked form (0: the kernel's own).  The result does
 *              not depend on it beyond rounding.  Accepted: 0, 64, 128.  The bf16 tensor-core
 *              kernel (d = 128) always computes 128-row tiles -- two 64-row chunks per tile,
 *              the chunk-to-chunk term inside a tile taken directly rather than through the
 *              state; the fp32 CUDA-core kernel uses 64-row chunks.
 * d          : 64 or 128.  All pointers 16-byte aligned.
 */
sala_status sala_linear_prefill(const void* q, const void* k, const void* v, const float* decay,
                                void* o, const float* state_in, float* state_out, int B, int H,
                                int N, int d, int chunk, sala_dtype dt, sala_stream stream);

/* sala_linear_prefill with device scratch, so that long sequences can be split into segments that
 * run in parallel.  The pages have no counterpart; the split is the state recursion's own
 * associativity: each segment's state contribution is computed from a zero state, the segments'
 * incoming states are chained (S_in(p+1) = lambda^len(p) S_in(p) + S_seg(p)), then every
 * segment's output is computed from its incoming state.  K and V are read twice; in exchange
 * every SM has work when B * H alone would leave most of the GPU idle.  The result equals the
 * one-pass result up to rounding (the state is associated differently).
 * workspace       : at least sala_linear_prefill_workspace(B, H, N, d, dt) bytes of device
 *                   scratch (16-byte aligned; no initial value needed), not shared with a
 *                   concurrent call.  A size of 0 means this problem runs in one pass; with
 *                   NULL or too small a workspace the call also runs in one pass.
 * Other arguments, validation and errors are those of sala_linear_prefill. */
sala_status sala_linear_prefill_ws(const void* q, const void* k, const void* v, const float* decay,
                                   void* o, const float* state_in, float* state_out, int B, int H,
                                   int N, int d, int chunk, void* workspace,
                                   size_t workspace_bytes, sala_dtype dt, sala_stream stream);
size_t sala_linear_prefill_workspace(int B, int H, int N, int d, sala_dtype dt);

/* One decode step of the linear attention for every (batch, head).  Pages: the linear layers keep
 * O(1) memory per token through a recursive form (DE technical summary section 2, "recursive
 * formulations"; JA technical summary section 2.1, linear attention at O(N) compute and memory);
 * this is that recursion for one new token.  The state is updated first and then read, so the
 * current token attends to itself with lambda^0:
 *   S <- lambda_h S + k^T v ;  o = q S
 * q, k, v, o : [B, H, d] device, dt.   state : [B, H, d, d] fp32 device, updated in place.
 */
sala_status sala_linear_decode(const void* q, const void* k, const void* v, const float* decay,
                               float* state, void* o, int B, int H, int d, sala_dtype dt,
                               sala_stream stream);

/* The linear layers of the hybrid rotate queries and keys by position before the linear
 * attention (HyPE: MiniCPM-SALA summaries, JA section 2.2 "positional encoding (HyPE)", DE
 * section 2 "HyPE" -- rotary embeddings in the linear layers, none in the sparse layers).  The
 * pages give no RoPE parameters; these calls take the rotate-half form: element i is paired with
 * element i + d/2 (i < d/2), theta_i = rope_base^(-2i/d), and at position p
 *   x'_i = x_i cos(p theta_i) - x_{i+d/2} sin(p theta_i)
 *   x'_{i+d/2} = x_{i+d/2} cos(p theta_i) + x_i sin(p theta_i)
 * for x = q and x = k (not v), then the linear attention above.  The rotation is fused into the
 * kernels' load path (the rotated q and k are never written to memory); on the bf16 tensor-core
 * path the rotated values are rounded to bf16 for the products.
 * pos0      : position of row 0 (a continuation after state_out of an earlier call passes the
 *             number of rows already processed); >= 0.
 * rope_base : > 1 and < 1e30 (the usual value is 10000).
 * workspace : as sala_linear_prefill_ws (NULL or too small: one pass).
 * Other arguments, validation and errors are those of sala_linear_prefill (chunk: the kernel's
 * own). */
sala_status sala_linear_prefill_rope(const void* q, const void* k, const void* v,
                                     const float* decay, void* o, const float* state_in,
                                     float* state_out, int B, int H, int N, int d, int64_t pos0,
                                     double rope_base, void* workspace, size_t workspace_bytes,
                                     sala_dtype dt, sala_stream stream);

/* Backward pass of the linear attention of a fresh sequence (no carried state): the gradients of
 * sum(o * dout) with respect to q, k and v, o as in sala_linear_prefill.  (The method is produced
 * by continual training through these layers: MiniCPM-SALA summaries, JA section 2 "Method", DE
 * section 3 on the training stages.)  With the upstream gradient dout:
 *   dq_i = sum_{j<=i} lambda^{i-j} (dout_i . v_j) k_j
 *   dk_j = sum_{i>=j} lambda^{i-j} (dout_i . v_j) q_i
 *   dv_j = sum_{i>=j} lambda^{i-j} (q_i . k_j) dout_i
 * Each is a linear attention (the anti-causal ones of the reversed sequence), computed by the
 * forward kernels; the decay is not differentiated (it is a fixed per-head constant here).
 * q, k, v, dout, dq, dk, dv : [B, H, N, d] device, dt (outputs must not overlap the inputs).
 * workspace : at least sala_linear_backward_workspace(B, H, N, d, dt) bytes (16-byte aligned).
 * Validation and errors as sala_linear_prefill. */
sala_status sala_linear_backward(const void* q, const void* k, const void* v, const float* decay,
                                 const void* dout, void* dq, void* dk, void* dv, int B, int H, int N,
                                 int d, void* workspace, size_t workspace_bytes, sala_dtype dt,
                                 sala_stream stream);
size_t sala_linear_backward_workspace(int B, int H, int N, int d, sala_dtype dt);

/* sala_linear_decode with q and k rotated at position pos (>= 0), as sala_linear_prefill_rope. */
sala_status sala_linear_decode_rope(const void* q, const void* k, const void* v,
                                    const float* decay, float* state, void* o, int B, int H,
                                    int d, int64_t pos, double rope_base, sala_dtype dt,
                                    sala_stream stream);

/* sala_linear_decode (rope_base == 0) or sala_linear_decode_rope (rope_base in (1, 1e30)),
 * launched as a programmatic dependent of the previous kernel in the stream: the kernel starts
 * while that kernel is still running and requests `state` at once; q, k, v and decay are read
 * only after that kernel has completed and its writes are visible.  A decode step of many
 * layers thus overlaps each layer's state read with the layer before (the state of a layer does
 * not depend on the previous layer's output).  Contract: the previous kernel in the stream does
 * not write `state` (e.g. two steps of the same layer back to back need sala_linear_decode).
 * Captures into CUDA graphs.  Arguments, layouts and errors as sala_linear_decode_rope. */
sala_status sala_linear_decode_pdl(const void* q, const void* k, const void* v, const float* decay,
                                   float* state, void* o, int B, int H, int d, int64_t pos,
                                   double rope_base, sala_dtype dt, sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * QK normalisation (weight-free RMS norm of every head row).  Pages: MiniCPM-SALA normalises
 * queries and keys to keep the activations stable (DE technical summary section 2, "additional
 * improvements"); no formula is given, the reading taken is
 *
 *   y[r, c] = x[r, c] / sqrt( (1/d) * sum_e x[r, e]^2 + eps )
 *
 * over each row of d elements, no learned scale (a per-channel scale is an elementwise product
 * the caller applies after this), for q and k of every layer ahead of RoPE, block compression
 * and selection.  Squares are summed in fp32, the result rounded once to dt.
 *   q, q_out   device, q_rows rows of d elements ([B, H, N, d] is B*H*N rows), dt
 *   k, k_out   device, k_rows rows of d elements; may be NULL when k_rows == 0
 *   eps        > 0 and finite
 * Outputs may alias their inputs exactly (in place); partial overlap is not allowed.  All four
 * pointers 16-byte aligned.  One launch covers both tensors.  d in {64, 128}.
 * Errors: SALA_ERR_INVALID_ARG (negative rows, bad eps or pointer), SALA_ERR_UNSUPPORTED (d).
 * ---------------------------------------------------------------------------------------- */
sala_status sala_qk_norm(const void* q, void* q_out, int64_t q_rows, const void* k, void* k_out,
                         int64_t k_rows, int d, double eps, sala_dtype dt, sala_stream stream);

/* The prologue of a layer in one pass over q and k: the QK normalisation above (eps > 0; eps 0
 * skips it) and/or the rotary embedding of the linear layers (rope_base > 0, as in
 * sala_linear_prefill_rope: rotate-half pairs, theta_i = base^(-2i/d); row r of a [B, heads, N, d]
 * tensor at position pos0 + r % N; rope_base 0 skips it), at least one of the two.  The norm is
 * applied first; a rotation keeps each row's RMS, so the order matters only at rounding level.
 * A linear layer with RoPE can then run the plain sala_linear_prefill on the rotated q and k
 * (one more read and write of them, against the fused rotation's issue cost).  q_rows and
 * k_rows are multiples of N; other arguments and errors as sala_qk_norm. */
sala_status sala_qk_prologue(const void* q, void* q_out, int64_t q_rows, const void* k,
                             void* k_out, int64_t k_rows, int d, int N, double eps,
                             int64_t pos0, double rope_base, sala_dtype dt, sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Block compression of the keys of a sparse layer (mean pooling).  Pages: InfLLM-V2 selects
 * the relevant context parts without extra parameters (JA technical summary section 2.1); the
 * pooling itself is the plain reading of "mean-pooled block keys".
 *
 *   kbar[b, g, j] = round_dt( (1/block) * sum_{t < block} k[b, g, j*block + t] )
 *
 * computed exactly (fp64 sum) and rounded once to dt, for the complete blocks
 * j = first_block .. first_block + n_blocks - 1 (they must end at or before row N).
 * k    : [B, Hkv, N, d] device, dt.
 * kbar : [B, Hkv, nb_cap, d] device, dt; block j is written at row j (nb_cap >= first_block +
 *        n_blocks), other rows are untouched -- decode appends one block at a time.
 * block: 64.
 */
sala_status sala_block_compress(const void* k, void* kbar, int B, int Hkv, int N, int d,
                                int block, int first_block, int n_blocks, int nb_cap,
                                sala_dtype dt, sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Block selection (scoring + top-k).  Pages: InfLLM-V2 picks, for each query, the context parts
 * that matter, with no extra parameters (JA technical summary section 2.1 "hybrid attention";
 * abstract on fugumt.com: sparse attention for local detail and key information); the scoring
 * and the forced init/local blocks are the plain reading of that selection step.  Query row r
 * sits at absolute position p = q_pos0 + r in block c = p / block.  For KV group g:
 *   forced     F = {0 .. n_init-1} U {max(0, c-n_local+1) .. c}          (init + local blocks)
 *   candidates   = {n_init .. c-n_local}                                 (complete, past)
 *   score(j)     = (sum over the group's query heads of q[b, h, r]) . kbar[b, g, j]
 *   selection    = F U top_topk(candidates by score, ties to the lower block index)
 * idx[b, g, r, :] receives the selection in ascending order, padded with -1, in
 * slots = n_init + n_local + topk entries.
 *
 * q    : [B, H, Nq, d] device, dt.    kbar : [B, Hkv, nb, d] device, dt (nb >= c - n_local + 1
 *        for every row).    idx : [B, Hkv, Nq, slots] int32 device.
 * workspace: device scratch of at least sala_block_topk_workspace(...) bytes (may be NULL when
 *        that is 0).  It must not be shared with a call that runs concurrently.
 * Limits: topk <= 64 (or any value when every row has at most topk candidates), n_local >= 1,
 *         n_init >= 0, block 64, d 64 or 128.
 */
sala_status sala_block_topk(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv,
                            int Nq, int q_pos0, int nb, int d, int block, int topk, int n_init,
                            int n_local, void* workspace, size_t workspace_bytes, sala_dtype dt,
                            sala_stream stream);
size_t sala_block_topk_workspace(int B, int Hkv, int Nq, int q_pos0, int nb, int block, int topk);

/* Query-block-granular selection: the tokens of one query block share one selection.  A variant of
 * the selection step, which the pages describe (InfLLM-V2 selects blocks by a coarse score) without
 * fixing its granularity.  For each (batch, KV group, query block c of `block` tokens, the last one
 * possibly partial) the score of candidate b is (sum over the group's heads and the block's tokens
 * of q) . kbar_b; candidates, forced blocks, ties and the row layout are those of sala_block_topk
 * with q_pos0 = 0, and the row is written to every token of the block, so sala_sparse_prefill takes
 * idx unchanged.  The scores are fp32 on CUDA cores.
 * q   : [B, H, Nq, d] device, dt.   kbar : [B, Hkv, nb, d] device, dt.
 * idx : [B, Hkv, Nq, n_init + n_local + topk] int32 device (output).
 * Validation and errors as sala_block_topk (block = 64; topk <= 64 whenever a block has more
 * than topk candidates). */
sala_status sala_block_topk_qblock(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                   int Hkv, int Nq, int nb, int d, int block, int topk, int n_init,
                                   int n_local, sala_dtype dt, sala_stream stream);

/* Query-block-granular selection scored by softmax-probability group aggregation (another reading
 * of the open scoring step).  For each (batch, KV group, query block c) and each of the group's
 * heads h: u_h = the mean of the block's queries of head h, logits scale * (u_h . kbar_j) over the
 * candidates j, a softmax over them; score(j) = the sum over the group's heads of the
 * probabilities.  Candidates, forced blocks, ties, output layout and validation as
 * sala_block_topk_qblock; scale 0 = 1/sqrt(d); at most 16 query heads per KV head.  The scores
 * are fp32 on CUDA cores (two passes over the candidates: per-head max and sum, then the sum of
 * probabilities and the top k). */
sala_status sala_block_topk_qblock_softmax(const void* q, const void* kbar, int32_t* idx, int B,
                                           int H, int Hkv, int Nq, int nb, int d, int block,
                                           int topk, int n_init, int n_local, float scale,
                                           sala_dtype dt, sala_stream stream);

/* Per-query-head selection: every query head chooses its own blocks.  Another reading of the
 * open selection step (the pages: InfLLM-V2 picks the relevant context blocks for each query,
 * gist.science JA technical summary section 2.1, without saying whether a KV group's heads share
 * the choice).  For each (batch, query head h, query row i) the score of candidate b is
 * q[b,h,i] . kbar[b, h / (H/Hkv), b]; candidates (n_init .. c - n_local), forced blocks, ties
 * (the lower block wins) and the row layout are those of sala_block_topk with q_pos0 = 0.  bf16
 * with d 128, Nq > 16 and topk <= 64 scores on the tensor cores (the query split into two bf16
 * terms, as sala_block_topk); other shapes and fp32 on CUDA cores.
 * q   : [B, H, Nq, d] device, dt.   kbar : [B, Hkv, nb, d] device, dt.
 * idx : [B, H, Nq, n_init + n_local + topk] int32 device (output), one row per query head.
 * Validation and errors as sala_block_topk (block = 64; topk <= 64 whenever a row has more than
 * topk candidates). */
sala_status sala_block_topk_per_head(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                     int Hkv, int Nq, int nb, int d, int block, int topk,
                                     int n_init, int n_local, sala_dtype dt, sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Sparse attention prefill: exact causal softmax over the selected blocks.  Pages: sparse
 * layers compute on selected parts but keep the dense KV cache ("sparse compute, dense
 * storage", JA technical summary section 1).
 *
 *   J(b,h,i) = { j <= i : j / block in idx[b, h / (H/Hkv), i, :] }
 *   o[b,h,i] = sum_{j in J} softmax_j(scale * q[b,h,i] . k[b,g,j]) v[b,g,j]
 *
 * q, o : [B, H, N, d] device, dt.   k, v : [B, Hkv, N, d] device, dt.
 * idx  : [B, Hkv, N, slots] int32 device, each row ascending and -1 padded (sala_block_topk's
 *        output); entries must lie in [0, (N-1)/block].  An out-of-range entry is skipped and
 *        flagged SALA_ERR_BOUNDS in the status word.
 * scale: softmax scale; 0 selects 1/sqrt(d).   block 64; d 64 or 128; H / Hkv <= 16.
 *        bf16 with H / Hkv = 16 and d = 128 runs on the tensor cores; other shapes and fp32 run
 *        on CUDA cores.
 */
sala_status sala_sparse_prefill(const void* q, const void* k, const void* v, const int32_t* idx,
                                void* o, int B, int H, int Hkv, int N, int d, int block,
                                int slots, float scale, sala_dtype dt, sala_stream stream);

/* Sparse attention prefill over per-head selections (sala_block_topk_per_head's output):
 *   J(b,h,i) = { j <= i : j / block in idx[b, h, i, :] },  o as sala_sparse_prefill.
 * idx  : [B, H, N, slots] int32 device, each row ascending among its non-negative entries and -1
 *        padded; entries past the row's query block are skipped and flagged SALA_ERR_BOUNDS.
 * Other arguments, shapes and errors as sala_sparse_prefill.  bf16 with H = 16 Hkv, d 128,
 * slots <= 80 and N <= 2^20 runs on the tensor cores: each 16-token unit of a KV group walks the
 * union of its 16 heads' x 16 tokens' selections, and every row keeps only its own blocks; other
 * shapes and fp32 run on CUDA cores, one query head per CTA.
 */
sala_status sala_sparse_prefill_per_head(const void* q, const void* k, const void* v,
                                         const int32_t* idx, void* o, int B, int H, int Hkv, int N,
                                         int d, int block, int slots, float scale, sala_dtype dt,
                                         sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Training path of the sparse layers: the forward with its row statistic, and the backward pass.
 * The method reaches its sparse layers by continual training through them (JA technical summary
 * section 2, training phases; DE section 3 "Trainingsstrategie"); the pages give no formula, and
 * the reading is the gradient of the sparse attention with the block selection held fixed (the
 * top-k choice is piecewise constant in q and k and passes no gradient):
 *   P_ij = exp(scale q_i.k_j - lse_i) over the visible keys j of row i,  D_i = do_i . o_i
 *   dq_i = scale sum_j P_ij (do_i.v_j - D_i) k_j
 *   dk_j = scale sum_i P_ij (do_i.v_j - D_i) q_i      (i over the KV group's query rows)
 *   dv_j = sum_i P_ij do_i
 *
 * sala_sparse_prefill_lse: sala_sparse_prefill plus lse [B, H, N] fp32 (device, output), the
 *   natural log of sum_j exp(scale q_i.k_j) over row i's visible keys (-inf for a row that sees
 *   none).  This training forward takes P V as P_hi V + P_lo V (P split into two bf16 terms) and
 *   every exponential through the same ex2 the backward uses, so o is exact to ~2^-16 before its
 *   rounding; when o_lo is not NULL it receives [B, H, N, d] bf16 (device, output), the rounding
 *   residual o - bf16(o), so o + o_lo carries that accuracy to the backward.  Takes bf16, d 128,
 *   H = 16 Hkv, block 64, slots <= 80 (else SALA_ERR_UNSUPPORTED).
 *
 * sala_sparse_backward: q [B,H,N,d], k, v [B,Hkv,N,d], o, o_lo, dout [B,H,N,d] (bf16, device), idx
 *   [B,Hkv,N,slots] (the selection the forward used: ascending distinct block ids, -1 padded,
 *   none in the future of its token), o, o_lo and lse from sala_sparse_prefill_lse.  D_i =
 *   do_i . (o_i + o_lo_i) enters every dS_ij = P_ij (dP_ij - D_i), a difference that cancels on
 *   peaked softmaxes: o_lo may be NULL, but D then carries bf16 o's rounding (~1 % of max |dq|
 *   on peaked selections).  Writes dq [B,H,N,d] and
 *   dk, dv [B,Hkv,N,d] (bf16, device, outputs; they must not alias the inputs).  scale 0 = 1/sqrt(d).
 *   workspace: >= sala_sparse_backward_workspace(...) bytes, 16-byte aligned, not shared with a
 *   concurrent call.  dk and dv are sums of fp32 atomic additions, so their last bits may vary
 *   from run to run.  Same shape limits as above, and B * Hkv * N * slots < 2^31.  A selection
 *   entry in the future of its token, past the last block or repeated is reported as
 *   SALA_ERR_BOUNDS by sala_check_status and skipped.
 * ---------------------------------------------------------------------------------------- */
sala_status sala_sparse_prefill_lse(const void* q, const void* k, const void* v,
                                    const int32_t* idx, void* o, float* lse, void* o_lo, int B,
                                    int H, int Hkv, int N, int d, int block, int slots, float scale,
                                    sala_dtype dt, sala_stream stream);
size_t sala_sparse_backward_workspace(int B, int H, int Hkv, int N, int d, int slots);
sala_status sala_sparse_backward(const void* q, const void* k, const void* v, const int32_t* idx,
                                 const void* o, const void* o_lo, const float* lse,
                                 const void* dout, void* dq,
                                 void* dk, void* dv, int B, int H, int Hkv, int N, int d, int block,
                                 int slots, float scale, void* workspace, size_t workspace_bytes,
                                 sala_dtype dt, sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Sparse attention decode: one query token per (batch, head) at absolute position pos, over
 * a dense KV cache that holds rows 0 .. pos (capacity Tmax rows).  Pages: the sparse layers keep
 * the whole KV cache and compute on the selected parts only (JA technical summary section 1,
 * "sparse compute, dense storage"), and the model decodes with contexts up to 1M tokens on one
 * GPU (JA technical summary section 4.3; fugumt.com abstract).  The step is block selection as
 * in sala_block_topk for the one query row, then sala_sparse_prefill's softmax over the chosen
 * blocks.
 *
 * q, o          : [B, H, d] device, dt.
 * kcache, vcache: [B, Hkv, Tmax, d] device, dt.
 * kbar          : [B, Hkv, nb_cap, d] device, dt; blocks 0 .. pos/block - n_local compressed.
 * idx_in        : [B, Hkv, slots] int32 or NULL.  NULL = select here (scoring + top-k as in
 *                 sala_block_topk, for q_pos0 = pos); otherwise attend to these blocks.
 * idx_out       : [B, Hkv, slots] int32 or NULL; receives the selection that was used.
 * workspace     : at least sala_sparse_decode_workspace(...) bytes of device scratch, not
 *                 shared with a concurrent call.  Its first 256 bytes hold the counters of a
 *                 grid-wide barrier and must be zero before the first call (e.g. allocate it
 *                 zero-filled once); every call that completes leaves them zero, so the same
 *                 workspace can serve call after call and CUDA-graph replays.  After a call that
 *                 reported an error (SALA_ERR_TIMEOUT from sala_check_status), zero them again.
 *                 The rest needs no initial value.
 * Implementation, by shape:
 *   - bf16, d 64 or 128, k <= 64, slots <= 80, H/Hkv <= 16, at most 16 (batch, KV head) groups
 *     (and as many 16-CTA clusters resident at once), contexts whose candidate blocks fit 256 per
 *     SM: two launches -- a score kernel over every SM (each CTA's share of kbar in shared memory,
 *     tensor-core scores, its best keys stored) and an attend kernel of one 16-CTA cluster per
 *     group (exact top-k from the stored keys, attention over the winners, partials combined in
 *     distributed shared memory).  No device-side waits.
 *   - otherwise, when k <= 64, slots <= 80, H/Hkv <= 16 and the grid fits on the GPU at once: one
 *     cooperative launch with two grid-wide barriers (the counters above).
 *   - otherwise: four launches.
 */
sala_status sala_sparse_decode(const void* q, const void* kcache, const void* vcache,
                               const void* kbar, const int32_t* idx_in, int32_t* idx_out, void* o,
                               int B, int H, int Hkv, int pos, int Tmax, int nb_cap, int d,
                               int block, int topk, int n_init, int n_local, float scale,
                               void* workspace, size_t workspace_bytes, sala_dtype dt,
                               sala_stream stream);
size_t sala_sparse_decode_workspace(int B, int H, int Hkv, int pos, int block, int topk,
                                    int n_init, int n_local, int d);

/* sala_sparse_decode launched as a programmatic dependent of the previous kernel in the stream:
 * on its two-launch path (see sala_sparse_decode) the score kernel starts while that kernel still
 * runs and copies its share of kbar -- the rows of the candidate blocks n_init ..
 * pos/block - n_local -- into shared memory at once; q, the KV cache and idx_in are read only after
 * that kernel has completed and its writes are visible.  A decode step thus overlaps each sparse
 * layer's kbar read (8 MiB at 2^20 tokens, 2 KV heads) with the layer before.  Contract: the
 * previous kernel in the stream does not write those kbar rows (the block a token completes is a
 * local block, never a candidate, so compressing it just before is fine).  Other shapes run as
 * sala_sparse_decode.  Arguments, workspace rules and errors as sala_sparse_decode. */
sala_status sala_sparse_decode_pdl(const void* q, const void* kcache, const void* vcache,
                                   const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                   void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap,
                                   int d, int block, int topk, int n_init, int n_local, float scale,
                                   void* workspace, size_t workspace_bytes, sala_dtype dt,
                                   sala_stream stream);

/* sala_sparse_decode for a batch of sequences that each decode at their own position, with the
 * KV cache held in pages of one block.  The pages have no counterpart (the method stores the
 * whole KV cache densely); paging is how a server keeps many sequences' caches in one pool.
 * k_pages, v_pages : [n_pages, Hkv, 64, d] device, dt.  Page p holds the 64 key (value) rows of
 *                    one block of one sequence, for every KV head.
 * page_table       : [B, max_pages] int32 device.  Entry [b][j] is the page of block j of
 *                    sequence b; only the blocks a sequence attends to are read, and an entry
 *                    outside [0, n_pages) is flagged (SALA_ERR_BOUNDS through
 *                    sala_check_status) and its block left out.
 * kbar             : [B, Hkv, nb_cap, d] device, each sequence's compressed blocks (dense).
 * pos              : [B] int32 device, sequence b's query position (its cache holds pos[b] + 1
 *                    tokens); each in [0, max_pos] (outside: flagged and clamped).
 * max_pos          : the largest position, < max_pages * 64 (sizes the launch and workspace).
 * block            : 64 (the page size).  Selection happens here (no idx_in); idx_out: as
 *                    sala_sparse_decode.
 * workspace        : at least sala_sparse_decode_paged_workspace(...) bytes; its first 256
 *                    bytes follow the rule of sala_sparse_decode's workspace.
 * Runs as the one-launch kernel only: top-k <= 64, n_init + n_local + topk <= 80, at most 16
 * query heads per KV head, d in {64, 128}; otherwise SALA_ERR_UNSUPPORTED.  Other arguments,
 * validation and errors are those of sala_sparse_decode. */
sala_status sala_sparse_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                     int n_pages, const int32_t* page_table, int max_pages,
                                     const void* kbar, int nb_cap, const int32_t* pos,
                                     int max_pos, int32_t* idx_out, void* o, int B, int H,
                                     int Hkv, int d, int block, int topk, int n_init, int n_local,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     sala_dtype dt, sala_stream stream);
size_t sala_sparse_decode_paged_workspace(int B, int H, int Hkv, int max_pos, int block, int topk,
                                          int n_init, int n_local, int d);

/* sala_sparse_decode for callers that cannot allocate device memory.  The pages have no
 * counterpart; this is a property of the library, not of the method.
 *
 * Some callers may not allocate device memory once they are running -- a serving loop that sizes
 * every buffer at start-up so no allocation can stall or fail mid-request, or a plug-in whose
 * host application owns the whole device memory pool and exposes no allocator -- and so cannot
 * provide the workspace sala_sparse_decode needs.  This call takes the same arguments minus the
 * workspace and computes the same result with scratch space built into the library: a fixed
 * 4 MiB area per GPU (a __device__ array that every GPU loading the library keeps until the
 * process exits).  It allocates nothing itself and calls nothing that allocates.
 *   - Problems whose sala_sparse_decode_workspace(...) exceeds 4 MiB are refused with
 *     SALA_ERR_UNSUPPORTED (for example B * Hkv above 7 at a 2^20-token context with
 *     32 query heads, d 128, top-64); nothing is launched.
 *   - The first call on each GPU looks up the area's device address (cudaGetSymbolAddress, with
 *     that GPU current) and caches it; make that first call before any stream capture.
 *   - All calls on a GPU share the one area: calls that can run concurrently on the same GPU
 *     race on it and must not be made.  The area keeps the previous call's contents.  Its first
 *     256 bytes are the barrier counters described under sala_sparse_decode; every call zeroes
 *     them on `stream` before its kernels run (a memset, which allocates nothing), so each call
 *     starts from clean counters and a call that reported SALA_ERR_TIMEOUT does not affect the
 *     calls after it.  Nothing else in the area needs a starting value.
 * Other arguments, validation and errors are those of sala_sparse_decode. */
sala_status sala_sparse_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                       const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                       void* o, int B, int H, int Hkv, int pos, int Tmax,
                                       int nb_cap, int d, int block, int topk, int n_init,
                                       int n_local, float scale, sala_dtype dt,
                                       sala_stream stream);

/* ------------------------------------------------------------------------------------------
 * Status and diagnostics. */

/* Synchronises `stream`, then reads and clears this device's status word: SALA_OK, or
 * SALA_ERR_TIMEOUT / SALA_ERR_BOUNDS when a kernel recorded that fault since the last check,
 * or SALA_ERR_CUDA when the synchronisation itself failed. */
sala_status sala_check_status(sala_stream stream);

/* Static string naming a status code. */
const char* sala_status_string(sala_status status);

/* One-line description of the calling thread's most recent failure ("" if none). */
const char* sala_last_error(void);

/* Upper bound, in nanoseconds, on every bounded wait inside the kernels (default 2e9).  A wait
 * that runs past it gives up, records SALA_ERR_TIMEOUT and lets its kernel return. */
void sala_set_wait_limit_ns(uint64_t ns);

/* Self-test of the timeout path: launches one block that waits on a shared-memory barrier that
 * nothing ever completes, bounded by sala_set_wait_limit_ns.  The kernel gives up, records
 * SALA_ERR_TIMEOUT and returns; sala_check_status then reports it.  Launches on `stream`. */
sala_status sala_selftest_wait_timeout(sala_stream stream);

/* Library version (major * 10000 + minor * 100 + patch). */
int sala_version(void);

/* 1 in the bounds-checking build (libsala_debug.so, compiled with SALA_DEBUG_BOUNDS), 0 in the
 * release build (libsala.so).  The debug build runs the same kernels with checks on the indices
 * that come from data or counters (selection rows, union lists and bitmaps, row buffers, seeds,
 * decode slots, compressed blocks): an index that would leave its buffer records SALA_ERR_BOUNDS
 * in the status word and the access is skipped instead of made.  It stands in for a memory
 * checker on tiny cases; it is slower and not for production. */
int sala_debug_bounds_build(void);

#ifdef __cplusplus
}
#endif

#endif /* SALA_H_ */
