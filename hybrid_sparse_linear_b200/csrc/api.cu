// C ABI of libsala: host-side validation, dispatch to the kernels, and the status word.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <initializer_list>
#include <mutex>
#include <utility>

#include "../../include/sala.h"
#include "kernels.h"

namespace {

// Per-device status word: kernels atomicOr fault bits into it; sala_check_status reads and
// clears it.  It is the library's only global device state.
__device__ unsigned g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
thread_local char g_err[512] = "";

sala_status fail(sala_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

// Device context of the current device (address of its status word, wait limit).
sala_status get_ctx(sala::DevCtx* ctx) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(SALA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(SALA_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status_word);
        if (e != cudaSuccess)
            return fail(SALA_ERR_CUDA, "cudaGetSymbolAddress(status): %s", cudaGetErrorString(e));
        g_status_ptr[dev] = static_cast<unsigned*>(p);
    }
    ctx->status = g_status_ptr[dev];
    ctx->wait_limit_ns = g_wait_limit_ns.load();
    return SALA_OK;
}

sala_status launched(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return fail(SALA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    g_err[0] = 0;
    return SALA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, code, ...) \
    do {                         \
        if (!(cond)) return fail(code, __VA_ARGS__); \
    } while (0)

#define REQ_PTR(p) REQUIRE((p) != nullptr && aligned16(p), SALA_ERR_INVALID_ARG, \
                           "%s must be a non-NULL 16-byte aligned device pointer", #p)

sala::DType to_dt(sala_dtype dt) { return dt == SALA_BF16 ? sala::DType::BF16 : sala::DType::F32; }

}  // namespace

namespace sala {
// Lets entry points defined in other files report through sala_last_error().
void set_last_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}
}  // namespace sala

extern "C" {

int sala_version(void) { return 100; }

int sala_debug_bounds_build(void) { return sala::kDebugBounds ? 1 : 0; }

const char* sala_status_string(sala_status s) {
    switch (s) {
        case SALA_OK: return "SALA_OK";
        case SALA_ERR_INVALID_ARG: return "SALA_ERR_INVALID_ARG";
        case SALA_ERR_UNSUPPORTED: return "SALA_ERR_UNSUPPORTED";
        case SALA_ERR_CUDA: return "SALA_ERR_CUDA";
        case SALA_ERR_TIMEOUT: return "SALA_ERR_TIMEOUT";
        case SALA_ERR_BOUNDS: return "SALA_ERR_BOUNDS";
    }
    return "SALA_ERR_UNKNOWN";
}

const char* sala_last_error(void) { return g_err; }

void sala_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 1); }

sala_status sala_check_status(sala_stream stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(SALA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    unsigned word = 0;
    e = cudaMemcpy(&word, ctx.status, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(SALA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (word) {
        const unsigned zero = 0;
        e = cudaMemcpy(ctx.status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return fail(SALA_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
    }
    if (word & sala::kStatusTimeout) return fail(SALA_ERR_TIMEOUT, "a device-side wait expired");
    if (word & sala::kStatusBounds) return fail(SALA_ERR_BOUNDS, "a device-side index was out of range");
    g_err[0] = 0;
    return SALA_OK;
}

sala_status sala_selftest_wait_timeout(sala_stream stream) {
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_selftest_wait(static_cast<cudaStream_t>(stream), ctx), "selftest");
}

// ----------------------------------------------------------------------------------------------
static sala_status linear_prefill_impl(const void* q, const void* k, const void* v,
                                       const float* decay, void* o, const float* state_in,
                                       float* state_out, int B, int H, int N, int d, int chunk,
                                       void* workspace, size_t workspace_bytes, sala::Rope rope,
                                       sala_dtype dt, sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && N >= 0, SALA_ERR_INVALID_ARG, "negative size (B=%d H=%d N=%d)", B, H, N);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(chunk == 0 || chunk == 64 || chunk == 128, SALA_ERR_UNSUPPORTED,
            "chunk %d (supported: 0, 64, 128)", chunk);
    if (B == 0 || H == 0) return SALA_OK;
    REQUIRE(decay != nullptr, SALA_ERR_INVALID_ARG, "decay must be a device pointer");
    if (state_in) REQUIRE(aligned16(state_in), SALA_ERR_INVALID_ARG, "state_in must be 16-byte aligned");
    if (state_out) REQUIRE(aligned16(state_out), SALA_ERR_INVALID_ARG, "state_out must be 16-byte aligned");
    if (workspace) REQUIRE(aligned16(workspace), SALA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (N > 0) {
        REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o);
    }
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == SALA_BF16 && N > 0 && sala::linear_prefill_tc_supported(d))
        return launched(sala::launch_linear_prefill_tc(q, k, v, decay, o, state_in, state_out, B,
                                                       H, N, d, workspace, workspace_bytes, rope, st,
                                                       ctx),
                        "linear_prefill_tc");
    return launched(sala::launch_linear_prefill_simt(to_dt(dt), q, k, v, decay, o, state_in,
                                                     state_out, B, H, N, d, rope, st, ctx),
                    "linear_prefill");
}

sala_status sala_linear_prefill(const void* q, const void* k, const void* v, const float* decay,
                                void* o, const float* state_in, float* state_out, int B, int H,
                                int N, int d, int chunk, sala_dtype dt, sala_stream stream) {
    return linear_prefill_impl(q, k, v, decay, o, state_in, state_out, B, H, N, d, chunk, nullptr,
                               0, sala::Rope{0.0, 0}, dt, stream);
}

size_t sala_linear_prefill_workspace(int B, int H, int N, int d, sala_dtype dt) {
    if (dt != SALA_BF16) return 0;
    return sala::linear_prefill_tc_workspace(B, H, N, d);
}

sala_status sala_linear_prefill_ws(const void* q, const void* k, const void* v, const float* decay,
                                   void* o, const float* state_in, float* state_out, int B, int H,
                                   int N, int d, int chunk, void* workspace,
                                   size_t workspace_bytes, sala_dtype dt, sala_stream stream) {
    return linear_prefill_impl(q, k, v, decay, o, state_in, state_out, B, H, N, d, chunk,
                               workspace, workspace_bytes, sala::Rope{0.0, 0}, dt, stream);
}

sala_status sala_linear_prefill_rope(const void* q, const void* k, const void* v,
                                     const float* decay, void* o, const float* state_in,
                                     float* state_out, int B, int H, int N, int d, int64_t pos0,
                                     double rope_base, void* workspace, size_t workspace_bytes,
                                     sala_dtype dt, sala_stream stream) {
    REQUIRE(pos0 >= 0, SALA_ERR_INVALID_ARG, "pos0 %lld is negative", (long long)pos0);
    REQUIRE(rope_base > 1.0 && rope_base < 1e30, SALA_ERR_INVALID_ARG,
            "rope_base %g (must lie in (1, 1e30))", rope_base);
    return linear_prefill_impl(q, k, v, decay, o, state_in, state_out, B, H, N, d, 0, workspace,
                               workspace_bytes, sala::Rope{rope_base, pos0}, dt, stream);
}

// Backward pass of the linear attention of a fresh sequence: with o_i = sum_{j<=i} lambda^{i-j}
// (q_i . k_j) v_j and the upstream gradient do,
//   dq_i = sum_{j<=i} lambda^{i-j} (do_i . v_j) k_j          = LA(q: do, k: v, v: k)_i
//   dk_j = sum_{i>=j} lambda^{i-j} (do_i . v_j) q_i          = flip(LA(flip v, flip do, flip q))_j
//   dv_j = sum_{i>=j} lambda^{i-j} (q_i . k_j) do_i          = flip(LA(flip k, flip q, flip do))_j
// (the anti-causal sums are causal sums of the reversed sequence), so the forward kernels compute
// all three; the workspace holds the reversed copies.
size_t sala_linear_backward_workspace(int B, int H, int N, int d, sala_dtype dt) {
    if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t t = up((size_t)B * H * N * d * (dt == SALA_F32 ? 4 : 2));
    return 5 * t + up(sala_linear_prefill_workspace(B, H, N, d, dt));
}

sala_status sala_linear_backward(const void* q, const void* k, const void* v, const float* decay,
                                 const void* dout, void* dq, void* dk, void* dv, int B, int H, int N,
                                 int d, void* workspace, size_t workspace_bytes, sala_dtype dt,
                                 sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && N >= 0, SALA_ERR_INVALID_ARG, "negative size (B=%d H=%d N=%d)", B, H, N);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    if (B == 0 || H == 0 || N == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(dout); REQ_PTR(dq); REQ_PTR(dk); REQ_PTR(dv);
    REQUIRE(decay != nullptr, SALA_ERR_INVALID_ARG, "decay must be a device pointer");
    const size_t need = sala_linear_backward_workspace(B, H, N, d, dt);
    REQUIRE(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need,
            SALA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu",
            need, workspace_bytes);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t t = up((size_t)B * H * N * d * (dt == SALA_F32 ? 4 : 2));
    char* w = static_cast<char*>(workspace);
    void* fv = w;
    void* fdo = w + t;
    void* fq = w + 2 * t;
    void* fk = w + 3 * t;
    void* fo = w + 4 * t;
    void* lws = w + 5 * t;
    const size_t lws_bytes = workspace_bytes - 5 * t;
    const sala::DType tdt = to_dt(dt);
    const int64_t BH = (int64_t)B * H;
    auto la = [&](const void* a, const void* b_, const void* c, void* o) {
        return linear_prefill_impl(a, b_, c, decay, o, nullptr, nullptr, B, H, N, d, 0, lws,
                                   lws_bytes, sala::Rope{0.0, 0}, dt, stream);
    };
    s = la(dout, v, k, dq);
    if (s != SALA_OK) return s;
    for (auto pr : {std::make_pair(v, fv), std::make_pair(dout, fdo), std::make_pair(q, fq),
                    std::make_pair(k, fk)}) {
        const cudaError_t e = sala::launch_flip_rows(tdt, pr.first, pr.second, BH, N, d, st);
        if (e != cudaSuccess) return launched(e, "linear_backward flip");
    }
    s = la(fv, fdo, fq, fo);
    if (s != SALA_OK) return s;
    cudaError_t e = sala::launch_flip_rows(tdt, fo, dk, BH, N, d, st);
    if (e != cudaSuccess) return launched(e, "linear_backward flip");
    s = la(fk, fq, fdo, fo);
    if (s != SALA_OK) return s;
    e = sala::launch_flip_rows(tdt, fo, dv, BH, N, d, st);
    return launched(e, "linear_backward flip");
}

static sala_status linear_decode_impl(const void* q, const void* k, const void* v,
                                      const float* decay, float* state, void* o, int B, int H,
                                      int d, sala::Rope rope, bool pdl, sala_dtype dt,
                                      sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0, SALA_ERR_INVALID_ARG, "negative size (B=%d H=%d)", B, H);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    if (B == 0 || H == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o); REQ_PTR(state);
    REQUIRE(decay != nullptr, SALA_ERR_INVALID_ARG, "decay must be a device pointer");
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_linear_decode(to_dt(dt), q, k, v, decay, state, o, B, H, d,
                                               rope, pdl, static_cast<cudaStream_t>(stream), ctx),
                    "linear_decode");
}

sala_status sala_linear_decode(const void* q, const void* k, const void* v, const float* decay,
                               float* state, void* o, int B, int H, int d, sala_dtype dt,
                               sala_stream stream) {
    return linear_decode_impl(q, k, v, decay, state, o, B, H, d, sala::Rope{0.0, 0}, false, dt,
                              stream);
}

sala_status sala_linear_decode_pdl(const void* q, const void* k, const void* v, const float* decay,
                                   float* state, void* o, int B, int H, int d, int64_t pos,
                                   double rope_base, sala_dtype dt, sala_stream stream) {
    REQUIRE(pos >= 0, SALA_ERR_INVALID_ARG, "pos %lld is negative", (long long)pos);
    REQUIRE(rope_base == 0.0 || (rope_base > 1.0 && rope_base < 1e30), SALA_ERR_INVALID_ARG,
            "rope_base %g (0, or in (1, 1e30))", rope_base);
    return linear_decode_impl(q, k, v, decay, state, o, B, H, d, sala::Rope{rope_base, pos}, true,
                              dt, stream);
}

sala_status sala_linear_decode_rope(const void* q, const void* k, const void* v,
                                    const float* decay, float* state, void* o, int B, int H,
                                    int d, int64_t pos, double rope_base, sala_dtype dt,
                                    sala_stream stream) {
    REQUIRE(pos >= 0, SALA_ERR_INVALID_ARG, "pos %lld is negative", (long long)pos);
    REQUIRE(rope_base > 1.0 && rope_base < 1e30, SALA_ERR_INVALID_ARG,
            "rope_base %g (must lie in (1, 1e30))", rope_base);
    return linear_decode_impl(q, k, v, decay, state, o, B, H, d, sala::Rope{rope_base, pos}, false,
                              dt, stream);
}

// ----------------------------------------------------------------------------------------------
sala_status sala_qk_norm(const void* q, void* q_out, int64_t q_rows, const void* k, void* k_out,
                         int64_t k_rows, int d, double eps, sala_dtype dt, sala_stream stream) {
    REQUIRE(q_rows >= 0 && k_rows >= 0, SALA_ERR_INVALID_ARG, "negative row count (q %lld, k %lld)",
            (long long)q_rows, (long long)k_rows);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(eps > 0.0 && eps < 1e30, SALA_ERR_INVALID_ARG, "eps %g (must be positive and finite)", eps);
    REQUIRE(q_rows <= ((int64_t)1 << 40) && k_rows <= ((int64_t)1 << 40), SALA_ERR_INVALID_ARG,
            "row count too large");
    if (q_rows == 0 && k_rows == 0) return SALA_OK;
    if (q_rows > 0) {
        REQ_PTR(q); REQ_PTR(q_out);
    }
    if (k_rows > 0) {
        REQ_PTR(k); REQ_PTR(k_out);
    }
    const int esize = dt == SALA_F32 ? 4 : 2;
    auto overlap = [&](const void* a, const void* b, int64_t rows) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        const int64_t n = rows * d * esize;
        return x != y && x < y + n && y < x + n;
    };
    REQUIRE(q_rows == 0 || !overlap(q, q_out, q_rows), SALA_ERR_INVALID_ARG,
            "q_out overlaps q without being the same buffer");
    REQUIRE(k_rows == 0 || !overlap(k, k_out, k_rows), SALA_ERR_INVALID_ARG,
            "k_out overlaps k without being the same buffer");
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_qk_norm(to_dt(dt), q_rows ? q : nullptr, q_rows ? q_out : nullptr,
                                         q_rows, k_rows ? k : nullptr, k_rows ? k_out : nullptr,
                                         k_rows, d, (float)eps, static_cast<cudaStream_t>(stream)),
                    "qk_norm");
}

sala_status sala_qk_prologue(const void* q, void* q_out, int64_t q_rows, const void* k,
                             void* k_out, int64_t k_rows, int d, int N, double eps,
                             int64_t pos0, double rope_base, sala_dtype dt, sala_stream stream) {
    REQUIRE(q_rows >= 0 && k_rows >= 0, SALA_ERR_INVALID_ARG, "negative row count (q %lld, k %lld)",
            (long long)q_rows, (long long)k_rows);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(eps == 0.0 || (eps > 0.0 && eps < 1e30), SALA_ERR_INVALID_ARG,
            "eps %g (0 for no norm, else positive and finite)", eps);
    REQUIRE(rope_base == 0.0 || (rope_base > 1.0 && rope_base < 1e30), SALA_ERR_INVALID_ARG,
            "rope_base %g (0 for no rotation, else in (1, 1e30))", rope_base);
    REQUIRE(eps > 0.0 || rope_base > 0.0, SALA_ERR_INVALID_ARG, "neither a norm nor a rotation asked");
    REQUIRE(N >= 1 && pos0 >= 0, SALA_ERR_INVALID_ARG, "N %d, pos0 %lld", N, (long long)pos0);
    REQUIRE(q_rows % N == 0 && k_rows % N == 0, SALA_ERR_INVALID_ARG,
            "row counts (q %lld, k %lld) must be multiples of N = %d", (long long)q_rows,
            (long long)k_rows, N);
    if (q_rows == 0 && k_rows == 0) return SALA_OK;
    if (q_rows > 0) {
        REQ_PTR(q); REQ_PTR(q_out);
    }
    if (k_rows > 0) {
        REQ_PTR(k); REQ_PTR(k_out);
    }
    const int esize = dt == SALA_F32 ? 4 : 2;
    auto overlap = [&](const void* a, const void* b, int64_t rows) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        const int64_t n = rows * d * esize;
        return x != y && x < y + n && y < x + n;
    };
    REQUIRE(q_rows == 0 || !overlap(q, q_out, q_rows), SALA_ERR_INVALID_ARG,
            "q_out overlaps q without being the same buffer");
    REQUIRE(k_rows == 0 || !overlap(k, k_out, k_rows), SALA_ERR_INVALID_ARG,
            "k_out overlaps k without being the same buffer");
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_qk_prologue(to_dt(dt), q_rows ? q : nullptr, q_rows ? q_out : nullptr,
                                             q_rows, k_rows ? k : nullptr, k_rows ? k_out : nullptr,
                                             k_rows, d, (float)eps, N, pos0, rope_base,
                                             static_cast<cudaStream_t>(stream)),
                    "qk_prologue");
}

// ----------------------------------------------------------------------------------------------
sala_status sala_block_compress(const void* k, void* kbar, int B, int Hkv, int N, int d,
                                int block, int first_block, int n_blocks, int nb_cap,
                                sala_dtype dt, sala_stream stream) {
    REQUIRE(B >= 0 && Hkv >= 0 && N >= 0 && first_block >= 0 && n_blocks >= 0,
            SALA_ERR_INVALID_ARG, "negative size or block range");
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(block == 64, SALA_ERR_UNSUPPORTED, "block %d (supported: 64)", block);
    REQUIRE((int64_t)(first_block + (int64_t)n_blocks) * block <= N, SALA_ERR_INVALID_ARG,
            "blocks %d..%d are not complete within N=%d", first_block, first_block + n_blocks - 1, N);
    REQUIRE(nb_cap >= first_block + n_blocks, SALA_ERR_INVALID_ARG,
            "nb_cap %d < first_block + n_blocks = %d", nb_cap, first_block + n_blocks);
    if (B == 0 || Hkv == 0 || n_blocks == 0) return SALA_OK;
    REQ_PTR(k); REQ_PTR(kbar);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_block_compress(to_dt(dt), k, kbar, B, Hkv, N, d, first_block,
                                                n_blocks, nb_cap, static_cast<cudaStream_t>(stream),
                                                ctx),
                    "block_compress");
}

static sala_status check_select_args(int B, int H, int Hkv, int Nq, int q_pos0, int nb, int d,
                                     int block, int topk, int n_init, int n_local,
                                     sala_dtype dt) {
    REQUIRE(B >= 0 && H >= 0 && Hkv > 0 && Nq >= 0 && q_pos0 >= 0 && nb >= 0,
            SALA_ERR_INVALID_ARG, "bad sizes (B=%d H=%d Hkv=%d Nq=%d q_pos0=%d nb=%d)", B, H, Hkv,
            Nq, q_pos0, nb);
    REQUIRE(H % Hkv == 0, SALA_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(block == 64, SALA_ERR_UNSUPPORTED, "block %d (supported: 64)", block);
    REQUIRE(topk >= 0 && n_init >= 0 && n_local >= 1, SALA_ERR_INVALID_ARG,
            "need topk >= 0, n_init >= 0, n_local >= 1");
    REQUIRE(n_init + n_local + topk <= 1024, SALA_ERR_UNSUPPORTED, "more than 1024 slots");
    if (Nq > 0 && B > 0) {
        const int64_t last_pos = (int64_t)q_pos0 + Nq - 1;
        const int64_t last_c = last_pos / block;
        const int64_t need = last_c - n_local + 1;  // blocks 0 .. c - n_local must be compressed
        REQUIRE(need <= nb, SALA_ERR_INVALID_ARG,
                "kbar holds %d blocks but the last query (position %lld) needs %lld", nb,
                (long long)last_pos, (long long)need);
        const int64_t max_cand = last_c - n_local + 1 - n_init;
        REQUIRE(topk <= 64 || max_cand <= topk, SALA_ERR_UNSUPPORTED,
                "topk %d > 64 with up to %lld candidates", topk, (long long)max_cand);
    }
    return SALA_OK;
}

size_t sala_block_topk_workspace(int B, int Hkv, int Nq, int q_pos0, int nb, int block, int topk) {
    (void)nb; (void)block;
    if (B <= 0 || Hkv <= 0 || Nq <= 0) return 0;
    if (Nq > 16) return 0;  // tiled path needs no scratch
    return sala::rowwise_topk_workspace(B, Hkv, Nq, q_pos0, topk);
}

sala_status sala_block_topk(const void* q, const void* kbar, int32_t* idx, int B, int H, int Hkv,
                            int Nq, int q_pos0, int nb, int d, int block, int topk, int n_init,
                            int n_local, void* workspace, size_t workspace_bytes, sala_dtype dt,
                            sala_stream stream) {
    sala_status s = check_select_args(B, H, Hkv, Nq, q_pos0, nb, d, block, topk, n_init, n_local, dt);
    if (s != SALA_OK) return s;
    if (B == 0 || H == 0 || Nq == 0) return SALA_OK;
    REQ_PTR(q); REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (nb > 0) REQ_PTR(kbar);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t need = sala_block_topk_workspace(B, Hkv, Nq, q_pos0, nb, block, topk);
    if (need > 0) {
        REQUIRE(workspace != nullptr && workspace_bytes >= need && aligned16(workspace),
                SALA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu",
                need, workspace_bytes);
        return launched(sala::launch_block_topk_rowwise(to_dt(dt), q, kbar, idx, B, H, Hkv, Nq,
                                                        q_pos0, nb, d, topk, n_init, n_local,
                                                        workspace, st, ctx),
                        "block_topk_rowwise");
    }
    if (dt == SALA_BF16 && sala::block_topk_tc_supported(H, Hkv, Nq, q_pos0, nb, d, topk))
        return launched(sala::launch_block_topk_tc(q, kbar, idx, B, H, Hkv, Hkv, Nq, nb, topk, n_init,
                                                   n_local, st, ctx),
                        "block_topk_tc");
    return launched(sala::launch_block_topk_tiled(to_dt(dt), q, kbar, idx, B, H, Hkv, Hkv, Nq, q_pos0,
                                                  nb, d, topk, n_init, n_local, st, ctx),
                    "block_topk");
}

sala_status sala_block_topk_qblock_softmax(const void* q, const void* kbar, int32_t* idx, int B,
                                           int H, int Hkv, int Nq, int nb, int d, int block,
                                           int topk, int n_init, int n_local, float scale,
                                           sala_dtype dt, sala_stream stream) {
    sala_status s = check_select_args(B, H, Hkv, Nq, 0, nb, d, block, topk, n_init, n_local, dt);
    if (s != SALA_OK) return s;
    REQUIRE(Hkv > 0 && H / Hkv <= 16, SALA_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    if (B == 0 || H == 0 || Nq == 0) return SALA_OK;
    REQ_PTR(q); REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (nb > 0) REQ_PTR(kbar);
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_block_topk_qblock_softmax(to_dt(dt), q, kbar, idx, B, H, Hkv, Nq,
                                                           nb, d, topk, n_init, n_local, scale,
                                                           static_cast<cudaStream_t>(stream), ctx),
                    "block_topk_qblock_softmax");
}

sala_status sala_block_topk_qblock(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                   int Hkv, int Nq, int nb, int d, int block, int topk, int n_init,
                                   int n_local, sala_dtype dt, sala_stream stream) {
    sala_status s = check_select_args(B, H, Hkv, Nq, 0, nb, d, block, topk, n_init, n_local, dt);
    if (s != SALA_OK) return s;
    if (B == 0 || H == 0 || Nq == 0) return SALA_OK;
    REQ_PTR(q); REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (nb > 0) REQ_PTR(kbar);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_block_topk_qblock(to_dt(dt), q, kbar, idx, B, H, Hkv, Nq, nb, d,
                                                   topk, n_init, n_local,
                                                   static_cast<cudaStream_t>(stream), ctx),
                    "block_topk_qblock");
}

sala_status sala_block_topk_per_head(const void* q, const void* kbar, int32_t* idx, int B, int H,
                                     int Hkv, int Nq, int nb, int d, int block, int topk,
                                     int n_init, int n_local, sala_dtype dt, sala_stream stream) {
    sala_status s = check_select_args(B, H, Hkv, Nq, 0, nb, d, block, topk, n_init, n_local, dt);
    if (s != SALA_OK) return s;
    if (B == 0 || H == 0 || Nq == 0) return SALA_OK;
    REQ_PTR(q); REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (nb > 0) REQ_PTR(kbar);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // One selection group per query head (Hs = H), each scored against its KV head's kbar.
    if (dt == SALA_BF16 && sala::block_topk_tc_supported(H, Hkv, Nq, 0, nb, d, topk))
        return launched(sala::launch_block_topk_tc(q, kbar, idx, B, H, Hkv, H, Nq, nb, topk, n_init,
                                                   n_local, st, ctx),
                        "block_topk_per_head_tc");
    return launched(sala::launch_block_topk_tiled(to_dt(dt), q, kbar, idx, B, H, Hkv, H, Nq, 0, nb,
                                                  d, topk, n_init, n_local, st, ctx),
                    "block_topk_per_head");
}

// ----------------------------------------------------------------------------------------------
sala_status sala_sparse_prefill(const void* q, const void* k, const void* v, const int32_t* idx,
                                void* o, int B, int H, int Hkv, int N, int d, int block,
                                int slots, float scale, sala_dtype dt, sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && Hkv > 0 && N >= 0 && slots >= 1, SALA_ERR_INVALID_ARG,
            "bad sizes (B=%d H=%d Hkv=%d N=%d slots=%d)", B, H, Hkv, N, slots);
    REQUIRE(H % Hkv == 0, SALA_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(block == 64, SALA_ERR_UNSUPPORTED, "block %d (supported: 64)", block);
    REQUIRE(slots <= 1024, SALA_ERR_UNSUPPORTED, "more than 1024 slots");
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    REQUIRE(H / Hkv <= 16, SALA_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    if (B == 0 || H == 0 || N == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o);
    REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == SALA_BF16 && sala::sparse_prefill_tc_supported(H, Hkv, d))
        return launched(sala::launch_sparse_prefill_tc(q, k, v, idx, o, nullptr, nullptr, B, H,
                                                       Hkv, N, d, slots, scale, false, st, ctx),
                        "sparse_prefill_tc");
    return launched(sala::launch_sparse_prefill_simt(to_dt(dt), q, k, v, idx, o, B, H, Hkv, Hkv, N,
                                                     d, slots, scale, st, ctx),
                    "sparse_prefill");
}

sala_status sala_sparse_prefill_per_head(const void* q, const void* k, const void* v,
                                         const int32_t* idx, void* o, int B, int H, int Hkv, int N,
                                         int d, int block, int slots, float scale, sala_dtype dt,
                                         sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && Hkv > 0 && N >= 0 && slots >= 1, SALA_ERR_INVALID_ARG,
            "bad sizes (B=%d H=%d Hkv=%d N=%d slots=%d)", B, H, Hkv, N, slots);
    REQUIRE(H % Hkv == 0, SALA_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", H, Hkv);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(d == 64 || d == 128, SALA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
    REQUIRE(block == 64, SALA_ERR_UNSUPPORTED, "block %d (supported: 64)", block);
    REQUIRE(slots <= 1024, SALA_ERR_UNSUPPORTED, "more than 1024 slots");
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    if (B == 0 || H == 0 || N == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o);
    REQUIRE(idx != nullptr, SALA_ERR_INVALID_ARG, "idx must be a device pointer");
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dt == SALA_BF16 && sala::sparse_prefill_tc_supported(H, Hkv, d) && slots <= 80 &&
        N <= (1 << 20))
        return launched(sala::launch_sparse_prefill_tc(q, k, v, idx, o, nullptr, nullptr, B, H,
                                                       Hkv, N, d, slots, scale, true, st, ctx),
                        "sparse_prefill_per_head_tc");
    return launched(sala::launch_sparse_prefill_simt(to_dt(dt), q, k, v, idx, o, B, H, Hkv, H, N,
                                                     d, slots, scale, st, ctx),
                    "sparse_prefill_per_head");
}

// Sparse decode workspace: [0, 256) the cooperative one-launch path's barrier words, [256, 512)
// unused; from 512 on, the data of whichever path a call takes (every path writes what it reads
// there within the call).
size_t sala_sparse_decode_workspace(int B, int H, int Hkv, int pos, int block, int topk,
                                    int n_init, int n_local, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || pos < 0 || block <= 0) return 0;
    const int slots = n_init + n_local + topk;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t multi = 512 + up(sala::sparse_decode_attn_workspace(B, H, Hkv, slots, d)) +
                         up(sala::rowwise_topk_workspace(B, Hkv, 1, pos, topk)) +
                         up((size_t)B * Hkv * slots * sizeof(int32_t));
    const size_t fused = up(sala::sparse_decode_fused_workspace(B, H, Hkv, pos, topk, n_init, n_local, d));
    const size_t pf = 512 + sala::sparse_decode_pf_workspace(B, H, Hkv, pos, topk, n_init, n_local, d);
    const size_t m = multi > fused ? multi : fused;
    return m > pf ? m : pf;
}



// Forward with the row statistic the backward needs (bf16, d 128, 16 query heads per KV head).
sala_status sala_sparse_prefill_lse(const void* q, const void* k, const void* v,
                                    const int32_t* idx, void* o, float* lse, void* o_lo, int B,
                                    int H, int Hkv, int N, int d, int block, int slots, float scale,
                                    sala_dtype dt, sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && Hkv > 0 && N >= 0 && slots >= 1, SALA_ERR_INVALID_ARG,
            "bad sizes (B=%d H=%d Hkv=%d N=%d slots=%d)", B, H, Hkv, N, slots);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    REQUIRE(dt == SALA_BF16 && d == 128 && H == 16 * Hkv && block == 64 && slots <= 80,
            SALA_ERR_UNSUPPORTED, "the lse forward takes bf16, d 128, 16 query heads per KV head, "
            "block 64 and at most 80 slots (got d=%d H=%d Hkv=%d block=%d slots=%d)", d, H, Hkv,
            block, slots);
    if (B == 0 || H == 0 || N == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o);
    REQUIRE(idx != nullptr && lse != nullptr, SALA_ERR_INVALID_ARG, "idx and lse must be device pointers");
    REQUIRE(o_lo == nullptr || aligned16(o_lo), SALA_ERR_INVALID_ARG, "o_lo must be 16-byte aligned");
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    return launched(sala::launch_sparse_prefill_tc(q, k, v, idx, o, lse, o_lo, B, H, Hkv, N, d, slots,
                                                   scale, false, static_cast<cudaStream_t>(stream),
                                                   ctx),
                    "sparse_prefill_lse");
}

// Backward pass of the sparse attention: D rows, the transposed selection, the query-side and
// key-side passes, then dk / dv rounded from their fp32 sums.
static size_t sparse_bwd_ws_parts(int B, int H, int Hkv, int N, int slots, size_t* o_csr,
                                  size_t* o_dk, size_t* o_dv) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t delta = up((size_t)B * H * N * 4);
    const size_t csr = up(sala::sparse_bwd_csr_layout(nullptr, B, Hkv, N, slots).bytes);
    const size_t acc = up((size_t)B * Hkv * N * 128 * 4);
    *o_csr = delta;
    *o_dk = delta + csr;
    *o_dv = delta + csr + acc;
    return delta + csr + 2 * acc;
}

size_t sala_sparse_backward_workspace(int B, int H, int Hkv, int N, int d, int slots) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0 || d != 128 || slots < 1) return 0;
    size_t a, b, c;
    return sparse_bwd_ws_parts(B, H, Hkv, N, slots, &a, &b, &c);
}

sala_status sala_sparse_backward(const void* q, const void* k, const void* v, const int32_t* idx,
                                 const void* o, const void* o_lo, const float* lse,
                                 const void* dout, void* dq,
                                 void* dk, void* dv, int B, int H, int Hkv, int N, int d, int block,
                                 int slots, float scale, void* workspace, size_t workspace_bytes,
                                 sala_dtype dt, sala_stream stream) {
    REQUIRE(B >= 0 && H >= 0 && Hkv > 0 && N >= 0 && slots >= 1, SALA_ERR_INVALID_ARG,
            "bad sizes (B=%d H=%d Hkv=%d N=%d slots=%d)", B, H, Hkv, N, slots);
    REQUIRE(dt == SALA_F32 || dt == SALA_BF16, SALA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    REQUIRE(dt == SALA_BF16 && d == 128 && H == 16 * Hkv && block == 64 && slots <= 80,
            SALA_ERR_UNSUPPORTED, "the sparse backward takes bf16, d 128, 16 query heads per KV "
            "head, block 64 and at most 80 slots (got d=%d H=%d Hkv=%d block=%d slots=%d)", d, H,
            Hkv, block, slots);
    REQUIRE((int64_t)B * Hkv * N * slots < ((int64_t)1 << 31), SALA_ERR_UNSUPPORTED,
            "B * Hkv * N * slots must stay below 2^31");
    if (B == 0 || H == 0 || N == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k); REQ_PTR(v); REQ_PTR(o); REQ_PTR(dout); REQ_PTR(dq); REQ_PTR(dk);
    REQ_PTR(dv);
    REQUIRE(idx != nullptr && lse != nullptr, SALA_ERR_INVALID_ARG, "idx and lse must be device pointers");
    REQUIRE(o_lo == nullptr || aligned16(o_lo), SALA_ERR_INVALID_ARG, "o_lo must be 16-byte aligned");
    size_t o_csr, o_dk, o_dv;
    const size_t need = sparse_bwd_ws_parts(B, H, Hkv, N, slots, &o_csr, &o_dk, &o_dv);
    REQUIRE(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need,
            SALA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu",
            need, workspace_bytes);
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    sala_status s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(workspace);
    float* delta = reinterpret_cast<float*>(w);
    const sala::SparseBwdCsr csr = sala::sparse_bwd_csr_layout(w + o_csr, B, Hkv, N, slots);
    float* dk_acc = reinterpret_cast<float*>(w + o_dk);
    float* dv_acc = reinterpret_cast<float*>(w + o_dv);
    const size_t acc_bytes = (size_t)B * Hkv * N * 128 * 4;
    cudaError_t e = sala::launch_sparse_bwd_delta(o, o_lo, dout, delta, (int64_t)B * H * N, st);
    if (e == cudaSuccess) e = sala::launch_sparse_bwd_csr(idx, B, Hkv, N, slots, csr, st, ctx);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk_acc, 0, acc_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv_acc, 0, acc_bytes, st);
    if (e != cudaSuccess) return launched(e, "sparse_backward prologue");
    e = sala::launch_sparse_dq_tc(q, k, v, dout, idx, lse, delta, dq, B, H, Hkv, N, slots, scale,
                                  st, ctx);
    if (e != cudaSuccess) return launched(e, "sparse_backward dq");
    e = sala::launch_sparse_dkv_tc(q, k, v, dout, lse, delta, csr, dk_acc, dv_acc, B, H, Hkv, N,
                                   scale, st, ctx);
    if (e != cudaSuccess) return launched(e, "sparse_backward dk dv");
    return launched(sala::launch_sparse_bwd_finish(dk_acc, dv_acc, dk, dv,
                                                   (int64_t)B * Hkv * N * 128, scale, st),
                    "sparse_backward finish");
}

}  // extern "C"

// sala_sparse_decode, optionally zeroing the workspace's barrier counters on the stream once the
// arguments have passed validation (the allocation-free entry point, whose callers cannot reach
// its built-in area to clear them after a timed-out call).
sala_status sala::sparse_decode_impl(const void* q, const void* kcache, const void* vcache,
                                     const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                     void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap,
                                     int d, int block, int topk, int n_init, int n_local,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     sala_dtype dt, sala_stream stream, bool zero_barrier,
                                     bool pdl) {
    REQUIRE(pos >= 0 && pos < Tmax, SALA_ERR_INVALID_ARG, "pos %d outside the cache (Tmax %d)", pos, Tmax);
    sala_status s = check_select_args(B, H, Hkv, 1, pos, nb_cap, d, block, topk, n_init,
                                      n_local, dt);
    if (s != SALA_OK) return s;
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    REQUIRE(H / Hkv <= 16, SALA_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    if (B == 0 || H == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(kcache); REQ_PTR(vcache); REQ_PTR(o);
    if (!idx_in && nb_cap > 0) REQ_PTR(kbar);
    const size_t need = sala_sparse_decode_workspace(B, H, Hkv, pos, block, topk, n_init, n_local, d);
    REQUIRE(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need,
            SALA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu",
            need, workspace_bytes);
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (zero_barrier) {
        const cudaError_t e = cudaMemsetAsync(workspace, 0, 256, st);
        if (e != cudaSuccess) return launched(e, "sparse_decode barrier reset");
    }
    {
        const size_t base = 512;
        const cudaError_t e = sala::launch_sparse_decode_pf(
            to_dt(dt), q, kcache, vcache, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, d,
            topk, n_init, n_local, scale, static_cast<char*>(workspace) + base,
            workspace_bytes - base, pdl, st, ctx);
        if (e != cudaErrorNotSupported) return launched(e, "sparse_decode");
    }
    {
        const cudaError_t e = sala::launch_sparse_decode_fused(
            to_dt(dt), q, kcache, vcache, kbar, idx_in, idx_out, o, B, H, Hkv, pos, Tmax, nb_cap, d,
            topk, n_init, n_local, scale, workspace, workspace_bytes,
            sala::DecodePaging{nullptr, nullptr, 0, 0}, st, ctx);
        if (e != cudaErrorNotSupported) return launched(e, "sparse_decode");
    }
    const int slots = n_init + n_local + topk;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    char* w = static_cast<char*>(workspace) + 512;  // [0, 512): the one-launch paths' words
    void* ws_attn = w;
    w += up(sala::sparse_decode_attn_workspace(B, H, Hkv, slots, d));
    void* ws_sel = w;
    w += up(sala::rowwise_topk_workspace(B, Hkv, 1, pos, topk));
    int32_t* idx_ws = reinterpret_cast<int32_t*>(w);
    const int32_t* idx_use = idx_in;
    if (!idx_in) {
        int32_t* dst = idx_out ? idx_out : idx_ws;
        cudaError_t e = sala::launch_block_topk_rowwise(to_dt(dt), q, kbar, dst, B, H, Hkv, 1, pos,
                                                        nb_cap, d, topk, n_init, n_local, ws_sel,
                                                        st, ctx);
        if (e != cudaSuccess) return launched(e, "sparse_decode select");
        idx_use = dst;
    } else if (idx_out) {
        cudaError_t e = cudaMemcpyAsync(idx_out, idx_in, (size_t)B * Hkv * slots * sizeof(int32_t),
                                        cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return launched(e, "sparse_decode idx copy");
    }
    return launched(sala::launch_sparse_decode_attn(to_dt(dt), q, kcache, vcache, idx_use, o, B, H,
                                                    Hkv, pos, Tmax, d, slots, scale, ws_attn, st,
                                                    ctx),
                    "sparse_decode");
}

extern "C" {

sala_status sala_sparse_decode(const void* q, const void* kcache, const void* vcache,
                               const void* kbar, const int32_t* idx_in, int32_t* idx_out, void* o,
                               int B, int H, int Hkv, int pos, int Tmax, int nb_cap, int d,
                               int block, int topk, int n_init, int n_local, float scale,
                               void* workspace, size_t workspace_bytes, sala_dtype dt,
                               sala_stream stream) {
    return sala::sparse_decode_impl(q, kcache, vcache, kbar, idx_in, idx_out, o, B, H, Hkv, pos,
                                    Tmax, nb_cap, d, block, topk, n_init, n_local, scale,
                                    workspace, workspace_bytes, dt, stream, false, false);
}

sala_status sala_sparse_decode_pdl(const void* q, const void* kcache, const void* vcache,
                                   const void* kbar, const int32_t* idx_in, int32_t* idx_out,
                                   void* o, int B, int H, int Hkv, int pos, int Tmax, int nb_cap,
                                   int d, int block, int topk, int n_init, int n_local, float scale,
                                   void* workspace, size_t workspace_bytes, sala_dtype dt,
                                   sala_stream stream) {
    return sala::sparse_decode_impl(q, kcache, vcache, kbar, idx_in, idx_out, o, B, H, Hkv, pos,
                                    Tmax, nb_cap, d, block, topk, n_init, n_local, scale,
                                    workspace, workspace_bytes, dt, stream, false, true);
}

size_t sala_sparse_decode_paged_workspace(int B, int H, int Hkv, int max_pos, int block, int topk,
                                          int n_init, int n_local, int d) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || max_pos < 0 || block != 64) return 0;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return up(sala::sparse_decode_fused_workspace(B, H, Hkv, max_pos, topk, n_init, n_local, d));
}

sala_status sala_sparse_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                     int n_pages, const int32_t* page_table, int max_pages,
                                     const void* kbar, int nb_cap, const int32_t* pos,
                                     int max_pos, int32_t* idx_out, void* o, int B, int H,
                                     int Hkv, int d, int block, int topk, int n_init, int n_local,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     sala_dtype dt, sala_stream stream) {
    REQUIRE(block == 64, SALA_ERR_UNSUPPORTED, "block %d (pages hold 64 tokens)", block);
    REQUIRE(n_pages >= 0 && max_pages >= 0, SALA_ERR_INVALID_ARG, "negative page counts");
    REQUIRE(max_pos >= 0 && (int64_t)max_pos < (int64_t)max_pages * 64, SALA_ERR_INVALID_ARG,
            "max_pos %d outside the page table (%d pages of 64 tokens)", max_pos, max_pages);
    sala_status s = check_select_args(B, H, Hkv, 1, max_pos, nb_cap, d, block, topk, n_init,
                                      n_local, dt);
    if (s != SALA_OK) return s;
    REQUIRE(isfinite(scale) && scale >= 0.f, SALA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    REQUIRE(H / Hkv <= 16, SALA_ERR_UNSUPPORTED, "more than 16 query heads per KV head");
    if (B == 0 || H == 0) return SALA_OK;
    REQ_PTR(q); REQ_PTR(k_pages); REQ_PTR(v_pages); REQ_PTR(o); REQ_PTR(kbar);
    REQUIRE(page_table != nullptr && pos != nullptr, SALA_ERR_INVALID_ARG,
            "page_table and pos must be device pointers");
    const size_t need = sala_sparse_decode_paged_workspace(B, H, Hkv, max_pos, block, topk, n_init,
                                                           n_local, d);
    REQUIRE(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need,
            SALA_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required, got %zu",
            need, workspace_bytes);
    if (scale == 0.f) scale = 1.0f / sqrtf((float)d);
    sala::DevCtx ctx;
    s = get_ctx(&ctx);
    if (s != SALA_OK) return s;
    const cudaError_t e = sala::launch_sparse_decode_fused(
        to_dt(dt), q, k_pages, v_pages, kbar, nullptr, idx_out, o, B, H, Hkv, max_pos, 0, nb_cap, d,
        topk, n_init, n_local, scale, workspace, workspace_bytes,
        sala::DecodePaging{pos, page_table, max_pages, n_pages}, static_cast<cudaStream_t>(stream),
        ctx);
    if (e == cudaErrorNotSupported)
        return fail(SALA_ERR_UNSUPPORTED, "paged decode runs only as one launch (top-k <= 64, at most "
                    "80 slots, and a grid that fits the GPU)");
    return launched(e, "sparse_decode_paged");
}

}  // extern "C"
