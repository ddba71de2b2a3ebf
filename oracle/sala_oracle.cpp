// SALA hybrid attention -- plain fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct statement of what the
// hybrid attention forward of MiniCPM-SALA computes.  Only the test suite, the smoke check and
// the CPU-baseline leg of the benchmark may load it.  It shares no code, header, table or
// helper with the CUDA library; neither side includes or links the other.
//
// Sources ("MiniCPM-SALA: Hybridizing Sparse and Linear Attention for Efficient Long-Context
// Modeling", as summarised on the gist.science pages, JA technical summary section 2 "Method"
// and DE technical summary section 2 "Methodik"):
//   * 75% of the layers run Lightning Attention, a linear attention with a recursive O(N) form;
//   * 25% of the layers run InfLLM-V2 sparse attention, which attends to the relevant blocks of
//     the context while the KV cache stays dense ("sparse compute, dense storage");
//   * the pages give no formula for either.  The formulas below are the plain readings of the
//     project statement: decayed linear attention O_i = sum_{j<=i} lambda_h^{i-j} (q_i.k_j) v_j,
//     and block-sparse attention over mean-pooled block keys with per-query top-k plus the
//     init and local blocks.
//
// Everything is fp64.  Inputs arrive as fp64 copies of the exact bf16/fp32 values the GPU
// received (bf16 -> fp64 is exact).  Parallelism (std::thread) only splits independent
// outputs between workers; it never changes the order of arithmetic inside one output.
//
// Layout: every tensor is row-major [B, heads, rows, dim]; query head h of batch b reads KV
// head h / (H / Hkv) of batch b (grouped-query attention).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <thread>
#include <vector>

namespace {

// Run body(i) for i in [0, n) on up to nthreads workers (contiguous ranges).
void parallel_for(int64_t n, int nthreads, const std::function<void(int64_t)>& body) {
    if (nthreads <= 1 || n <= 1) {
        for (int64_t i = 0; i < n; ++i) body(i);
        return;
    }
    int64_t nt = std::min<int64_t>(nthreads, n);
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int64_t t = 0; t < nt; ++t) {
        int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
        pool.emplace_back([lo, hi, &body] {
            for (int64_t i = lo; i < hi; ++i) body(i);
        });
    }
    for (auto& th : pool) th.join();
}

double dot(const double* a, const double* b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------------------------
// bfloat16 round-to-nearest-even of an fp64 value (8 significant bits, fp32 exponent range).
// The stored block key of the sparse layers is a bf16 mean (reading: the GPU keeps k_bar in the
// dtype of the KV cache), so the oracle rounds exactly once, from the exact fp64 mean.
double orc_round_bf16(double x) {
    if (x == 0.0 || !std::isfinite(x)) return x;
    int e;
    std::frexp(x, &e);               // |x| = m * 2^e, m in [0.5, 1)
    // bf16 keeps 8 significant bits; its smallest normal is 2^-126 and subnormals share the
    // quantum 2^-133.
    int q_exp = std::max(e - 8, -133);
    double scaled = std::ldexp(x, -q_exp);   // exact (power-of-two scaling)
    double r = std::nearbyint(scaled);       // default rounding mode: ties to even
    double y = std::ldexp(r, q_exp);
    if (std::fabs(y) > 3.3895313892515355e38) y = std::copysign(INFINITY, x);  // past bf16 max
    return y;
}

// ---------------------------------------------------------------------------------------------
// Lightning-style linear attention, three independent statements of the same definition.
//
//   o_i = sum_{j<=i} lambda^{i-j} (q_i . k_j) v_j  +  lambda^{i+1} q_i S_in
//   S_out = lambda^N S_in + sum_{j<N} lambda^{N-1-j} k_j^T v_j
//
// S_in is the d_k x d_v state carried in from earlier tokens (zero when s_in is NULL): the
// pages' "recursive formulation" with O(1) memory in N.  lam[h] is the per-head decay lambda_h
// (shared by every batch entry).  q,k: [B,H,N,dk]; v,o: [B,H,N,dv]; states [B,H,dk,dv].

// (a) recurrent: S <- lambda S + k_i^T v_i ; o_i = q_i S   (update first, then read).
void orc_linear_recurrent(const double* q, const double* k, const double* v, const double* lam,
                          const double* s_in, double* o, double* s_out, int B, int H, int N,
                          int dk, int dv, int nthreads) {
    parallel_for((int64_t)B * H, nthreads, [&](int64_t bh) {
        const double L = lam[bh % H];
        std::vector<double> S((size_t)dk * dv, 0.0);
        if (s_in) std::memcpy(S.data(), s_in + bh * dk * dv, sizeof(double) * dk * dv);
        for (int i = 0; i < N; ++i) {
            const double* qi = q + (bh * N + i) * dk;
            const double* ki = k + (bh * N + i) * dk;
            const double* vi = v + (bh * N + i) * dv;
            for (int a = 0; a < dk; ++a)
                for (int c = 0; c < dv; ++c) S[a * dv + c] = L * S[a * dv + c] + ki[a] * vi[c];
            double* oi = o + (bh * N + i) * dv;
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int a = 0; a < dk; ++a) s += qi[a] * S[a * dv + c];
                oi[c] = s;
            }
        }
        if (s_out) std::memcpy(s_out + bh * dk * dv, S.data(), sizeof(double) * dk * dv);
    });
}

// (b) quadratic, masked: the definition written out, one output row at a time.  The decay
// lambda^{i-j} only ever takes non-negative exponents.  rows == NULL means all rows.
// When rows is given, o is [nrows, dv] and row r is (batch*head index, token index) =
// (rows[2r], rows[2r+1]).
void orc_linear_quadratic(const double* q, const double* k, const double* v, const double* lam,
                          const double* s_in, double* o, int B, int H, int N, int dk, int dv,
                          const int64_t* rows, int64_t nrows, int nthreads) {
    const int64_t total = rows ? nrows : (int64_t)B * H * N;
    parallel_for(total, nthreads, [&](int64_t r) {
        int64_t bh, i;
        if (rows) { bh = rows[2 * r]; i = rows[2 * r + 1]; }
        else { bh = r / N; i = r % N; }
        const double L = lam[bh % H];
        const double* qi = q + (bh * N + i) * dk;
        double* oi = o + r * dv;
        for (int c = 0; c < dv; ++c) oi[c] = 0.0;
        for (int64_t j = 0; j <= i; ++j) {
            double w = std::pow(L, (double)(i - j)) * dot(qi, k + (bh * N + j) * dk, dk);
            const double* vj = v + (bh * N + j) * dv;
            for (int c = 0; c < dv; ++c) oi[c] += w * vj[c];
        }
        if (s_in) {
            const double* S = s_in + bh * dk * dv;
            double w = std::pow(L, (double)(i + 1));
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int a = 0; a < dk; ++a) s += qi[a] * S[a * dv + c];
                oi[c] += w * s;
            }
        }
    });
}

// (c) chunked: the intra-chunk masked product plus the inter-chunk carried state, chunk length
// C (the last chunk may be shorter).  For chunk rows t, s in [0, len):
//   o_t = sum_{s<=t} lambda^{t-s} (q_t.k_s) v_s + lambda^{t+1} q_t S_prev
//   S_next = lambda^len S_prev + sum_s lambda^{len-1-s} k_s^T v_s
void orc_linear_chunked(const double* q, const double* k, const double* v, const double* lam,
                        const double* s_in, double* o, double* s_out, int B, int H, int N, int dk,
                        int dv, int C, int nthreads) {
    parallel_for((int64_t)B * H, nthreads, [&](int64_t bh) {
        const double L = lam[bh % H];
        std::vector<double> S((size_t)dk * dv, 0.0), Sn((size_t)dk * dv);
        if (s_in) std::memcpy(S.data(), s_in + bh * dk * dv, sizeof(double) * dk * dv);
        for (int c0 = 0; c0 < N; c0 += C) {
            const int len = std::min(C, N - c0);
            for (int t = 0; t < len; ++t) {
                const double* qt = q + (bh * N + c0 + t) * dk;
                double* ot = o + (bh * N + c0 + t) * dv;
                for (int c = 0; c < dv; ++c) ot[c] = 0.0;
                for (int s = 0; s <= t; ++s) {  // intra-chunk, decay-masked
                    double w = std::pow(L, (double)(t - s)) * dot(qt, k + (bh * N + c0 + s) * dk, dk);
                    const double* vs = v + (bh * N + c0 + s) * dv;
                    for (int c = 0; c < dv; ++c) ot[c] += w * vs[c];
                }
                const double wq = std::pow(L, (double)(t + 1));  // inter-chunk, carried state
                for (int c = 0; c < dv; ++c) {
                    double s = 0.0;
                    for (int a = 0; a < dk; ++a) s += qt[a] * S[a * dv + c];
                    ot[c] += wq * s;
                }
            }
            const double ws = std::pow(L, (double)len);
            for (size_t e = 0; e < S.size(); ++e) Sn[e] = ws * S[e];
            for (int s = 0; s < len; ++s) {
                const double w = std::pow(L, (double)(len - 1 - s));
                const double* ks = k + (bh * N + c0 + s) * dk;
                const double* vs = v + (bh * N + c0 + s) * dv;
                for (int a = 0; a < dk; ++a)
                    for (int c = 0; c < dv; ++c) Sn[a * dv + c] += w * ks[a] * vs[c];
            }
            S.swap(Sn);
        }
        if (s_out) std::memcpy(s_out + bh * dk * dv, S.data(), sizeof(double) * dk * dv);
    });
}

// One decode step for every (batch, head): S <- lambda S + k^T v, then o = q S.
// q,k: [B,H,dk]; v,o: [B,H,dv]; S: [B,H,dk,dv] updated in place.
void orc_linear_decode(const double* q, const double* k, const double* v, const double* lam,
                       double* S, double* o, int B, int H, int dk, int dv) {
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        const double L = lam[bh % H];
        double* Sb = S + bh * dk * dv;
        for (int a = 0; a < dk; ++a)
            for (int c = 0; c < dv; ++c)
                Sb[a * dv + c] = L * Sb[a * dv + c] + k[bh * dk + a] * v[bh * dv + c];
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < dk; ++a) s += q[bh * dk + a] * Sb[a * dv + c];
            o[bh * dv + c] = s;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// InfLLM-V2-style block-sparse attention.
//
// Block compression: k_bar[b] = mean of the T keys of block b (complete blocks only), rounded
// once to bf16 when round_bf16 != 0.  k: [B,Hkv,N,d]; kbar: [B,Hkv,n_blocks,d] holding blocks
// first_block .. first_block+n_blocks-1.
void orc_block_compress(const double* k, double* kbar, int B, int Hkv, int N, int d, int T,
                        int first_block, int n_blocks, int round_bf16) {
    for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg)
        for (int nb = 0; nb < n_blocks; ++nb) {
            const int blk = first_block + nb;
            double* out = kbar + (bg * n_blocks + nb) * d;
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int t = 0; t < T; ++t) s += k[(bg * N + (int64_t)blk * T + t) * d + c];
                double m = s / T;
                out[c] = round_bf16 ? orc_round_bf16(m) : m;
            }
        }
}

// Score of block blk for query row r of KV group g: (sum over the group's query heads of q).kbar.
// (Reading: one selection per (KV group, query token), shared by the group's query heads.)
static double group_score(const double* q, const double* kbar, int64_t b, int g, int64_t r,
                          int blk, int H, int Hkv, int Nq, int nb, int d) {
    const int G = H / Hkv;
    double s = 0.0;
    for (int c = 0; c < d; ++c) {
        double qs = 0.0;
        for (int hh = 0; hh < G; ++hh) qs += q[(((int64_t)b * H + g * G + hh) * Nq + r) * d + c];
        s += qs * kbar[(((int64_t)b * Hkv + g) * nb + blk) * d + c];
    }
    return s;
}

// Scores for explicit (b, g, r, blk) quadruples -> out[n].
void orc_block_scores_at(const double* q, const double* kbar, const int64_t* quads, int64_t n,
                         double* out, int H, int Hkv, int Nq, int nb, int d) {
    for (int64_t e = 0; e < n; ++e)
        out[e] = group_score(q, kbar, quads[4 * e], (int)quads[4 * e + 1], quads[4 * e + 2],
                             (int)quads[4 * e + 3], H, Hkv, Nq, nb, d);
}

// Block selection for query rows at absolute positions q_pos0 + r.  With c = pos / T:
//   forced     F = {0 .. n_init-1} U {max(0, c-n_local+1) .. c}     (init and local blocks)
//   candidates   = {n_init .. c-n_local}                            (complete, in the past,
//                                                                    never a forced block)
//   selection    = F U top_k(candidates, by score descending, ties to the lower block index)
// written ascending into idx[B,Hkv,Nq,slots] and padded with -1 (slots >= n_init+n_local+topk).
// kth_score[B,Hkv,Nq] (optional) receives the k-th selected candidate score (-inf when fewer
// than topk candidates exist, so every candidate is taken).
void orc_block_select(const double* q, const double* kbar, int32_t* idx, double* kth_score,
                      int B, int H, int Hkv, int Nq, int q_pos0, int nb, int d, int T, int topk,
                      int n_init, int n_local, int slots, int nthreads) {
    parallel_for((int64_t)B * Hkv * Nq, nthreads, [&](int64_t row) {
        const int64_t b = row / ((int64_t)Hkv * Nq);
        const int g = (int)((row / Nq) % Hkv);
        const int64_t r = row % Nq;
        const int64_t pos = q_pos0 + r;
        const int c = (int)(pos / T);
        std::vector<int> sel;
        for (int blk = 0; blk < n_init && blk <= c; ++blk) sel.push_back(blk);
        for (int blk = std::max(0, c - n_local + 1); blk <= c; ++blk)
            if (blk >= n_init) sel.push_back(blk);
        std::vector<std::pair<double, int>> cand;
        for (int blk = n_init; blk <= c - n_local; ++blk)
            cand.push_back({group_score(q, kbar, b, g, r, blk, H, Hkv, Nq, nb, d), blk});
        std::sort(cand.begin(), cand.end(), [](const auto& x, const auto& y) {
            if (x.first != y.first) return x.first > y.first;
            return x.second < y.second;
        });
        const int take = std::min<int>(topk, (int)cand.size());
        for (int e = 0; e < take; ++e) sel.push_back(cand[e].second);
        std::sort(sel.begin(), sel.end());
        int32_t* out = idx + row * slots;
        for (int e = 0; e < slots; ++e) out[e] = e < (int)sel.size() ? sel[e] : -1;
        if (kth_score)
            kth_score[row] = ((int)cand.size() >= topk && topk > 0)
                                 ? cand[topk - 1].first
                                 : -std::numeric_limits<double>::infinity();
    });
}

// Exact softmax attention of query rows over the keys of their selected blocks:
//   J(r) = { j : j <= pos(r), j < Nk, floor(j/T) in idx[b,g,r,:] (entries >= 0) }
//   o = sum_{j in J} softmax_j(scale * q.k_j) v_j     (max-subtracted, fp64)
// q,o: [B,H,Nq,d]; k,v: [B,Hkv,Nk,d]; idx: [B,Hkv,Nq,slots].  An empty J gives o = 0.
// rows != NULL restricts the work to (b*H+h, r) pairs; o is then [nrows, d].
void orc_sparse_attention(const double* q, const double* k, const double* v, const int32_t* idx,
                          double* o, int B, int H, int Hkv, int Nq, int q_pos0, int Nk, int d,
                          int T, int slots, double scale, const int64_t* rows, int64_t nrows,
                          int nthreads) {
    const int G = H / Hkv;
    const int64_t total = rows ? nrows : (int64_t)B * H * Nq;
    parallel_for(total, nthreads, [&](int64_t e) {
        int64_t bh, r;
        if (rows) { bh = rows[2 * e]; r = rows[2 * e + 1]; }
        else { bh = e / Nq; r = e % Nq; }
        const int64_t b = bh / H;
        const int h = (int)(bh % H);
        const int g = h / G;
        const int64_t pos = q_pos0 + r;
        const double* qi = q + (bh * Nq + r) * d;
        const int32_t* sel = idx + ((b * Hkv + g) * Nq + r) * slots;
        std::vector<int64_t> J;
        std::vector<int> blocks;
        for (int s = 0; s < slots; ++s)
            if (sel[s] >= 0) blocks.push_back(sel[s]);
        std::sort(blocks.begin(), blocks.end());
        blocks.erase(std::unique(blocks.begin(), blocks.end()), blocks.end());
        for (int blk : blocks)
            for (int64_t j = (int64_t)blk * T; j < (int64_t)(blk + 1) * T; ++j)
                if (j <= pos && j < Nk) J.push_back(j);
        double* oi = o + e * d;
        for (int c = 0; c < d; ++c) oi[c] = 0.0;
        if (J.empty()) return;
        const int64_t kv = (b * Hkv + g) * (int64_t)Nk;
        std::vector<double> logit(J.size());
        double mx = -std::numeric_limits<double>::infinity();
        for (size_t t = 0; t < J.size(); ++t) {
            logit[t] = scale * dot(qi, k + (kv + J[t]) * d, d);
            mx = std::max(mx, logit[t]);
        }
        double den = 0.0;
        for (size_t t = 0; t < J.size(); ++t) {
            logit[t] = std::exp(logit[t] - mx);
            den += logit[t];
        }
        for (size_t t = 0; t < J.size(); ++t) {
            const double w = logit[t] / den;
            const double* vj = v + (kv + J[t]) * d;
            for (int c = 0; c < d; ++c) oi[c] += w * vj[c];
        }
    });
}

// Plain causal softmax attention (every key j <= pos), the dense special case of the above.
void orc_dense_causal_attention(const double* q, const double* k, const double* v, double* o,
                                int B, int H, int Hkv, int Nq, int q_pos0, int Nk, int d,
                                double scale, int nthreads) {
    const int G = H / Hkv;
    parallel_for((int64_t)B * H * Nq, nthreads, [&](int64_t e) {
        const int64_t bh = e / Nq, r = e % Nq;
        const int64_t b = bh / H;
        const int g = (int)(bh % H) / G;
        const int64_t pos = q_pos0 + r;
        const int64_t nk = std::min<int64_t>(pos + 1, Nk);
        const double* qi = q + e * d;
        const int64_t kv = (b * Hkv + g) * (int64_t)Nk;
        std::vector<double> p(nk);
        double mx = -std::numeric_limits<double>::infinity();
        for (int64_t j = 0; j < nk; ++j) {
            p[j] = scale * dot(qi, k + (kv + j) * d, d);
            mx = std::max(mx, p[j]);
        }
        double den = 0.0;
        for (int64_t j = 0; j < nk; ++j) { p[j] = std::exp(p[j] - mx); den += p[j]; }
        double* oi = o + e * d;
        for (int c = 0; c < d; ++c) oi[c] = 0.0;
        for (int64_t j = 0; j < nk; ++j) {
            const double* vj = v + (kv + j) * d;
            for (int c = 0; c < d; ++c) oi[c] += (p[j] / den) * vj[c];
        }
    });
}

// Rotary position embedding, in place on x [B, H, N, d] (d even), row r at position pos0 + r.
// MiniCPM-SALA summaries, JA section 2.2 "positional encoding (HyPE)" and DE section 2 "HyPE": the
// linear-attention layers rotate queries and keys by position (RoPE); the sparse layers do not.
// The pages give no RoPE parameters; the reading taken is the rotate-half pairing (element i with
// element i + d/2 for i < d/2), frequencies theta_i = base^(-2i/d), angle (pos0 + r) * theta_i:
//   x'_i       = x_i cos(angle) - x_{i+d/2} sin(angle)
//   x'_{i+d/2} = x_{i+d/2} cos(angle) + x_i sin(angle)
void orc_rope(double* x, int B, int H, int N, int d, int64_t pos0, double base) {
    const int half = d / 2;
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh)
        for (int r = 0; r < N; ++r) {
            double* row = x + (bh * N + r) * d;
            const double p = (double)(pos0 + r);
            for (int i = 0; i < half; ++i) {
                const double theta = std::pow(base, -2.0 * i / d);
                const double c = std::cos(p * theta), s = std::sin(p * theta);
                const double x0 = row[i], x1 = row[i + half];
                row[i] = x0 * c - x1 * s;
                row[i + half] = x1 * c + x0 * s;
            }
        }
}

// Query-block-granular selection: one selection per (batch, KV group, query block of T tokens),
// shared by the block's tokens.  A variant the contract lists next to the per-token selection
// (the pages describe InfLLM-V2's block selection without fixing its granularity).  Reading: the
// block's score vector is the sum over the group's heads and over the block's tokens (those
// below Nq in a partial last block) of q, dotted with kbar; candidates, forced blocks, tie rule
// and output layout as orc_block_select, every token row of the block receiving the same row.
void orc_block_select_qblock(const double* q, const double* kbar, int32_t* idx, double* kth_score,
                             int B, int H, int Hkv, int Nq, int nb, int d, int T, int topk,
                             int n_init, int n_local, int slots, int nthreads) {
    const int G = H / Hkv;
    const int nqb = (Nq + T - 1) / T;
    parallel_for((int64_t)B * Hkv * nqb, nthreads, [&](int64_t item) {
        const int64_t b = item / ((int64_t)Hkv * nqb);
        const int g = (int)((item / nqb) % Hkv);
        const int c = (int)(item % nqb);
        const int r0 = c * T, r1 = std::min(Nq, r0 + T);
        std::vector<double> qs(d, 0.0);
        for (int h = g * G; h < (g + 1) * G; ++h)
            for (int r = r0; r < r1; ++r) {
                const double* qr = q + (((int64_t)b * H + h) * Nq + r) * d;
                for (int a = 0; a < d; ++a) qs[a] += qr[a];
            }
        std::vector<int> sel;
        for (int blk = 0; blk < n_init && blk <= c; ++blk) sel.push_back(blk);
        for (int blk = std::max(0, c - n_local + 1); blk <= c; ++blk)
            if (blk >= n_init) sel.push_back(blk);
        std::vector<std::pair<double, int>> cand;
        for (int blk = n_init; blk <= c - n_local; ++blk)
            cand.push_back({dot(qs.data(), kbar + (((int64_t)b * Hkv + g) * nb + blk) * d, d), blk});
        std::sort(cand.begin(), cand.end(), [](const auto& x, const auto& y) {
            if (x.first != y.first) return x.first > y.first;
            return x.second < y.second;
        });
        const int take = std::min<int>(topk, (int)cand.size());
        for (int e = 0; e < take; ++e) sel.push_back(cand[e].second);
        std::sort(sel.begin(), sel.end());
        const double kth = ((int)cand.size() >= topk && topk > 0)
                               ? cand[topk - 1].first
                               : -std::numeric_limits<double>::infinity();
        for (int r = r0; r < r1; ++r) {
            const int64_t row = ((int64_t)b * Hkv + g) * Nq + r;
            int32_t* out = idx + row * slots;
            for (int e = 0; e < slots; ++e) out[e] = e < (int)sel.size() ? sel[e] : -1;
            if (kth_score) kth_score[row] = kth;
        }
    });
}

// Weight-free RMS normalisation of every head row, in place on x [rows, d]:
//   x'_c = x_c / sqrt((1/d) sum_e x_e^2 + eps).
// MiniCPM-SALA summaries, DE section 2 "additional improvements": the model normalises queries
// and keys (QK normalisation) to keep the activations stable.  The pages name the step without a
// formula; the reading taken is an RMS norm over each head's d elements with no learned scale
// (a learned per-channel scale, where a model has one, is an elementwise product after this),
// applied to q and k of every layer before RoPE, block compression and selection.
void orc_qk_norm(double* x, int64_t rows, int d, double eps) {
    for (int64_t r = 0; r < rows; ++r) {
        double* row = x + r * d;
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += row[c] * row[c];
        const double inv = 1.0 / std::sqrt(ss / d + eps);
        for (int c = 0; c < d; ++c) row[c] *= inv;
    }
}

// Query-block selection with softmax-probability group aggregation (a variant the selection
// step leaves open: InfLLM-V2's block scores are not fixed by the pages).  Reading: for each
// (batch, KV group g, query block c of T tokens) and each head h of the group, the mean query
// u_h over the block's tokens scores every candidate block j (n_init .. c - n_local) with the
// logit scale * (u_h . kbar_j); the logits of a head go through a softmax over the candidates;
// the block's score is the sum over the group's heads of those probabilities.  The best topk by
// (score, lower block first) join the forced blocks; layout and kth_score as
// orc_block_select_qblock.  Optionally the candidates' scores of one (b, g, c) are returned.
void orc_block_select_qblock_softmax(const double* q, const double* kbar, int32_t* idx,
                                     double* kth_score, int B, int H, int Hkv, int Nq, int nb,
                                     int d, int T, int topk, int n_init, int n_local, int slots,
                                     double scale, int nthreads) {
    const int G = H / Hkv;
    const int nqb = (Nq + T - 1) / T;
    parallel_for((int64_t)B * Hkv * nqb, nthreads, [&](int64_t item) {
        const int64_t b = item / ((int64_t)Hkv * nqb);
        const int g = (int)((item / nqb) % Hkv);
        const int c = (int)(item % nqb);
        const int r0 = c * T, r1 = std::min(Nq, r0 + T);
        std::vector<int> sel;
        for (int blk = 0; blk < n_init && blk <= c; ++blk) sel.push_back(blk);
        for (int blk = std::max(0, c - n_local + 1); blk <= c; ++blk)
            if (blk >= n_init) sel.push_back(blk);
        const int lo = n_init, hi = c - n_local;
        const int nc = std::max(0, hi - lo + 1);
        std::vector<double> score(nc, 0.0), logit(nc);
        std::vector<double> u(d);
        for (int h = g * G; h < (g + 1) * G; ++h) {
            std::fill(u.begin(), u.end(), 0.0);
            for (int r = r0; r < r1; ++r) {
                const double* qr = q + (((int64_t)b * H + h) * Nq + r) * d;
                for (int a = 0; a < d; ++a) u[a] += qr[a];
            }
            for (int a = 0; a < d; ++a) u[a] /= (double)(r1 - r0);
            double mx = -std::numeric_limits<double>::infinity();
            for (int e = 0; e < nc; ++e) {
                logit[e] = scale * dot(u.data(), kbar + (((int64_t)b * Hkv + g) * nb + lo + e) * d, d);
                mx = std::max(mx, logit[e]);
            }
            double den = 0.0;
            for (int e = 0; e < nc; ++e) den += std::exp(logit[e] - mx);
            for (int e = 0; e < nc; ++e) score[e] += std::exp(logit[e] - mx) / den;
        }
        std::vector<std::pair<double, int>> cand;
        for (int e = 0; e < nc; ++e) cand.push_back({score[e], lo + e});
        std::sort(cand.begin(), cand.end(), [](const auto& x, const auto& y) {
            if (x.first != y.first) return x.first > y.first;
            return x.second < y.second;
        });
        const int take = std::min<int>(topk, (int)cand.size());
        for (int e = 0; e < take; ++e) sel.push_back(cand[e].second);
        std::sort(sel.begin(), sel.end());
        const double kth = ((int)cand.size() >= topk && topk > 0)
                               ? cand[topk - 1].first
                               : -std::numeric_limits<double>::infinity();
        for (int r = r0; r < r1; ++r) {
            const int64_t row = ((int64_t)b * Hkv + g) * Nq + r;
            int32_t* out = idx + row * slots;
            for (int e = 0; e < slots; ++e) out[e] = e < (int)sel.size() ? sel[e] : -1;
            if (kth_score) kth_score[row] = kth;
        }
    });
}

}  // extern "C"
