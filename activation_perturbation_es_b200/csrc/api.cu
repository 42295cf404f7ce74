// api.cu -- the C ABI declared in include/dust.h: host-side validation,
// workspace layout, and the sequence of launches for each entry point.
// Nothing here allocates or synchronises (except dust_poll_status, which
// exists to read the device status word back).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;

dust_status fail(dust_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

dust_status ok() { return DUST_OK; }

dust_status cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return DUST_OK;
    return fail(DUST_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define DUST_REQUIRE(cond, code, ...)                 \
    do {                                               \
        if (!(cond)) return fail(code, __VA_ARGS__);   \
    } while (0)

#define DUST_TRY(expr)                                 \
    do {                                               \
        dust_status _s = (expr);                       \
        if (_s != DUST_OK) return _s;                  \
    } while (0)

dust_status check_noise(const dust_noise& nz) {
    DUST_REQUIRE(nz.draw_count > 0, DUST_ERR_INVALID_ARG, "draw_count must be > 0");
    DUST_REQUIRE(nz.K_total > 0, DUST_ERR_INVALID_ARG, "K_total must be > 0");
    DUST_REQUIRE(std::isfinite(nz.sigma) && nz.sigma > 0.0f, DUST_ERR_INVALID_ARG, "sigma must be finite and > 0");
    DUST_REQUIRE(static_cast<uint64_t>(nz.draw_begin) + nz.draw_count <= (1ull << 32), DUST_ERR_INVALID_ARG,
                 "draw_begin + draw_count exceeds 2^32");
    DUST_REQUIRE(nz.token_begin <= 0x7FFFFFFFu, DUST_ERR_INVALID_ARG, "token_begin must be < 2^31");
    return ok();
}

dust_status check_ptr(const void* p, const char* name, bool nullable = false) {
    if (p == nullptr) {
        DUST_REQUIRE(nullable, DUST_ERR_INVALID_ARG, "%s must not be NULL", name);
        return ok();
    }
    DUST_REQUIRE(aligned(p, 16), DUST_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
    return ok();
}

dust_status check_seq(const int32_t* offs, int n_seq, int K, int T) {
    DUST_TRY(check_ptr(offs, "seq_offsets"));
    DUST_REQUIRE(n_seq >= 1, DUST_ERR_INVALID_ARG, "n_seq must be >= 1");
    DUST_REQUIRE(static_cast<long long>(K) * n_seq < (1ll << 31), DUST_ERR_INVALID_ARG,
                 "draws x sequences must be < 2^31");
    (void)T;
    return ok();
}

// Workspace: [status (256 B)][region 0][region 1]...; every region 256-byte aligned.
struct Layout {
    size_t off = dust::kStatusBytes;
    size_t add(size_t bytes) {
        const size_t o = off;
        off = dust::align_up(off + bytes, 256);
        return o;
    }
};

uint8_t* region(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// ---- GEMM dispatch shared by weight_grad, logits and head_step ----------------
struct GemmPlan {
    bool tc = false;
    int splits = 1;
    size_t partial_bytes = 0;
};

GemmPlan plan_gemm(int M, int N, int K, dust_dtype dt, bool a_kmajor, bool b_kmajor) {
    GemmPlan p;
    p.tc = dt == DUST_BF16 && dust::gemm_tc_supported(M, N, K, a_kmajor, b_kmajor);
    p.splits = p.tc ? dust::gemm_tc_splits(M, N, K) : dust::gemm_simt_splits(M, N, K);
    p.partial_bytes = p.splits > 1 ? sizeof(float) * static_cast<size_t>(p.splits) * M * N : 0;
    return p;
}

dust_status run_gemm(const GemmPlan& p, const void* A, bool ak, int lda, const void* B, bool bk, int ldb,
                     dust_dtype dt, int M, int N, int K, float* C, int ldc, int accumulate, float* partial,
                     uint32_t* status, cudaStream_t st) {
    cudaError_t e = p.tc ? dust::launch_gemm_tc(A, ak, lda, B, bk, ldb, M, N, K, C, ldc, accumulate, partial,
                                                p.splits, status, st)
                         : dust::launch_gemm_simt(A, ak, lda, B, bk, ldb, dt, M, N, K, C, ldc, accumulate,
                                                  partial, p.splits, st);
    return cuda_status(e, p.tc ? "tcgen05 GEMM" : "CUDA-core GEMM");
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

namespace dust {
// Lets entry points defined in other translation units report through
// dust_last_error().
dust_status record_error(dust_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace dust

extern "C" {

const char* dust_status_string(dust_status s) {
    switch (s) {
        case DUST_OK: return "DUST_OK";
        case DUST_ERR_INVALID_ARG: return "DUST_ERR_INVALID_ARG";
        case DUST_ERR_UNSUPPORTED: return "DUST_ERR_UNSUPPORTED";
        case DUST_ERR_ALIGNMENT: return "DUST_ERR_ALIGNMENT";
        case DUST_ERR_WORKSPACE: return "DUST_ERR_WORKSPACE";
        case DUST_ERR_CUDA: return "DUST_ERR_CUDA";
        case DUST_ERR_TIMEOUT: return "DUST_ERR_TIMEOUT";
    }
    return "DUST_ERR_UNKNOWN";
}

const char* dust_last_error(void) { return g_last_error.c_str(); }

int dust_abi_version(void) { return DUST_ABI_VERSION; }

dust_status dust_check_offsets(const int32_t* offs, int n_seq, int T) {
    DUST_REQUIRE(offs != nullptr, DUST_ERR_INVALID_ARG, "seq_offsets must not be NULL");
    DUST_REQUIRE(n_seq >= 1, DUST_ERR_INVALID_ARG, "n_seq must be >= 1");
    DUST_REQUIRE(offs[0] == 0, DUST_ERR_INVALID_ARG, "seq_offsets[0] must be 0 (got %d)", offs[0]);
    for (int q = 0; q < n_seq; ++q)
        DUST_REQUIRE(offs[q + 1] >= offs[q], DUST_ERR_INVALID_ARG, "seq_offsets decrease at %d", q);
    DUST_REQUIRE(offs[n_seq] == T, DUST_ERR_INVALID_ARG, "seq_offsets[n_seq] = %d, expected T = %d",
                 offs[n_seq], T);
    return ok();
}

dust_status dust_poll_status(void* ws, void* stream) {
    DUST_REQUIRE(ws != nullptr, DUST_ERR_INVALID_ARG, "ws must not be NULL");
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, as_stream(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
    DUST_TRY(cuda_status(e, "dust_poll_status"));
    if (word == 0) return ok();
    DUST_TRY(cuda_status(cudaMemsetAsync(ws, 0, sizeof word, as_stream(stream)), "dust_poll_status"));
    return fail(DUST_ERR_TIMEOUT, "a kernel's bounded wait ran out (status word 0x%08x)", word);
}

dust_status dust_selftest_bounded_wait(void* ws, uint32_t polls, void* stream) {
    DUST_REQUIRE(ws != nullptr, DUST_ERR_INVALID_ARG, "ws must not be NULL");
    DUST_REQUIRE(polls >= 1 && polls <= (1u << 20), DUST_ERR_INVALID_ARG, "polls must be in [1, 2^20]");
    return cuda_status(dust::launch_bounded_wait_selftest(static_cast<uint32_t*>(ws), polls, as_stream(stream)),
                       "dust_selftest_bounded_wait");
}

// ------------------------------------------------------------------ a4
dust_status dust_reward_scan(const float* c, float* r, int K, int T, const int32_t* seq_offsets, int n_seq,
                             float gamma, void* stream) {
    DUST_REQUIRE(K > 0 && T > 0, DUST_ERR_INVALID_ARG, "K and T must be > 0 (K=%d, T=%d)", K, T);
    DUST_REQUIRE(std::isfinite(gamma) && gamma >= 0.0f && gamma <= 1.0f, DUST_ERR_INVALID_ARG,
                 "gamma must be in [0, 1]");
    DUST_TRY(check_ptr(c, "c"));
    DUST_TRY(check_ptr(r, "r"));
    DUST_TRY(check_seq(seq_offsets, n_seq, K, T));
    return cuda_status(dust::launch_reward_scan(c, r, K, T, seq_offsets, n_seq, gamma, as_stream(stream)),
                       "dust_reward_scan");
}

size_t dust_reward_scan_split_workspace(int K, int T) {
    Layout L;
    if (K > 0 && T > 0) L.add(dust::reward_scan_chunks_workspace(K, T));
    return L.off;
}

dust_status dust_reward_scan_split(const float* c, float* r, int K, int T, const int32_t* seq_offsets, int n_seq,
                                   float gamma, void* ws, size_t ws_bytes, void* stream) {
    DUST_REQUIRE(K > 0 && T > 0, DUST_ERR_INVALID_ARG, "K and T must be > 0 (K=%d, T=%d)", K, T);
    DUST_REQUIRE(std::isfinite(gamma) && gamma >= 0.0f && gamma <= 1.0f, DUST_ERR_INVALID_ARG,
                 "gamma must be in [0, 1]");
    DUST_TRY(check_ptr(c, "c"));
    DUST_TRY(check_ptr(r, "r"));
    DUST_TRY(check_seq(seq_offsets, n_seq, K, T));
    DUST_REQUIRE(static_cast<long long>(K) * dust::ceil_div(T, 1024) < (1ll << 31), DUST_ERR_INVALID_ARG,
                 "draws x token chunks must be < 2^31");
    DUST_TRY(check_ptr(ws, "ws"));
    const size_t need = dust_reward_scan_split_workspace(K, T);
    DUST_REQUIRE(ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    return cuda_status(dust::launch_reward_scan_chunks(c, r, K, T, seq_offsets, n_seq, gamma,
                                                       region(ws, dust::kStatusBytes), as_stream(stream)),
                       "dust_reward_scan_split");
}

// ------------------------------------------------------------------ a5
size_t dust_layer_estimate_workspace(int draw_count, int T, int d_out, int is_r, float gamma) {
    (void)d_out;
    Layout L;
    if (!is_r && gamma != 0.0f && draw_count > 0 && T > 0) {
        L.add(sizeof(float) * static_cast<size_t>(draw_count) * T);          // r
        L.add(dust::reward_scan_chunks_workspace(draw_count, T));             // chunked scan (few long sequences)
    }
    return L.off;
}

dust_status dust_layer_estimate(const float* c_or_r, int is_r, int T, int d_out, const int32_t* seq_offsets,
                                int n_seq, float gamma, dust_noise nz, float* g_hat, void* g_hat_bf16,
                                int accumulate, void* ws, size_t ws_bytes, void* stream) {
    DUST_TRY(check_noise(nz));
    DUST_REQUIRE(T > 0 && d_out > 0, DUST_ERR_INVALID_ARG, "T and d_out must be > 0 (T=%d, d_out=%d)", T, d_out);
    DUST_REQUIRE(std::isfinite(gamma) && gamma >= 0.0f && gamma <= 1.0f, DUST_ERR_INVALID_ARG,
                 "gamma must be in [0, 1]");
    DUST_TRY(check_ptr(c_or_r, "c_or_r"));
    DUST_TRY(check_ptr(g_hat, "g_hat"));
    DUST_TRY(check_ptr(g_hat_bf16, "g_hat_bf16", true));
    const bool need_scan = !is_r && gamma != 0.0f;
    if (need_scan) DUST_TRY(check_seq(seq_offsets, n_seq, static_cast<int>(nz.draw_count), T));
    const size_t need = dust_layer_estimate_workspace(static_cast<int>(nz.draw_count), T, d_out, is_r, gamma);
    // ws may be NULL when no scan is needed (the estimate itself uses no scratch)
    DUST_TRY(check_ptr(ws, "ws", need <= dust::kStatusBytes));
    DUST_REQUIRE(ws == nullptr || ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    cudaStream_t st = as_stream(stream);
    const float* r = c_or_r;
    if (need_scan) {
        const int K = static_cast<int>(nz.draw_count);
        float* rw = reinterpret_cast<float*>(region(ws, dust::kStatusBytes));
        const size_t chunk_off = dust::align_up(dust::kStatusBytes + sizeof(float) * static_cast<size_t>(K) * T, 256);
        const cudaError_t e = dust::reward_scan_prefers_chunks(K, T, n_seq)
                                  ? dust::launch_reward_scan_chunks(c_or_r, rw, K, T, seq_offsets, n_seq, gamma,
                                                                    region(ws, chunk_off), st)
                                  : dust::launch_reward_scan(c_or_r, rw, K, T, seq_offsets, n_seq, gamma, st);
        DUST_TRY(cuda_status(e, "dust_layer_estimate (scan)"));
        r = rw;
    }
    return cuda_status(dust::launch_layer_estimate(r, T, d_out, nz, g_hat, g_hat_bf16, accumulate, st),
                       "dust_layer_estimate");
}

// ------------------------------------------------------------------ a1 + a5 + a6 fused
namespace {
struct FusedWs {
    size_t r_off = 0, chunk_off = 0, part_off = 0, total = 0;
    bool scan = false;
};

FusedWs fused_ws(int K, int T, int d_in, int d_out, int is_r, float gamma) {
    FusedWs w;
    Layout L;
    w.scan = !is_r && gamma != 0.0f;
    if (w.scan) {
        w.r_off = L.add(sizeof(float) * static_cast<size_t>(K) * T);
        w.chunk_off = L.add(dust::reward_scan_chunks_workspace(K, T));
    }
    w.part_off = L.add(dust::fused_estimate_scratch(T, d_in, d_out));
    w.total = L.off;
    return w;
}
}  // namespace

size_t dust_layer_estimate_weight_grad_workspace(int draw_count, int T, int d_in, int d_out, int is_r, float gamma) {
    if (draw_count <= 0 || T <= 0 || !dust::fused_estimate_supported(d_in, d_out)) return dust::kStatusBytes;
    return fused_ws(draw_count, T, d_in, d_out, is_r, gamma).total;
}

dust_status dust_layer_estimate_weight_grad(const float* c_or_r, int is_r, int T, int d_out,
                                            const int32_t* seq_offsets, int n_seq, float gamma, dust_noise nz,
                                            const void* X, int d_in, float* G_W, int accumulate, float* g_hat_out,
                                            void* ws, size_t ws_bytes, void* stream) {
    DUST_TRY(check_noise(nz));
    DUST_REQUIRE(T > 0 && d_out > 0, DUST_ERR_INVALID_ARG, "T and d_out must be > 0 (T=%d, d_out=%d)", T, d_out);
    DUST_REQUIRE(dust::fused_estimate_supported(d_in, d_out), DUST_ERR_UNSUPPORTED,
                 "d_in must be a multiple of 64 in [64, 512] (d_in=%d)", d_in);
    DUST_REQUIRE(std::isfinite(gamma) && gamma >= 0.0f && gamma <= 1.0f, DUST_ERR_INVALID_ARG,
                 "gamma must be in [0, 1]");
    DUST_REQUIRE(static_cast<long long>(nz.draw_count) * T < (1ll << 31), DUST_ERR_INVALID_ARG,
                 "draw_count x T must be < 2^31");
    DUST_REQUIRE(nz.draw_count <= dust::kFusedMaxDraws, DUST_ERR_UNSUPPORTED,
                 "draw_count must be <= %u per call (split the draws over calls with accumulate = 1)",
                 dust::kFusedMaxDraws);
    DUST_TRY(check_ptr(c_or_r, "c_or_r"));
    DUST_TRY(check_ptr(X, "X"));
    DUST_TRY(check_ptr(G_W, "G_W"));
    DUST_TRY(check_ptr(g_hat_out, "g_hat_out", true));
    DUST_TRY(check_ptr(ws, "ws"));
    const int K = static_cast<int>(nz.draw_count);
    const FusedWs w = fused_ws(K, T, d_in, d_out, is_r, gamma);
    DUST_REQUIRE(ws_bytes >= w.total, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, w.total);
    cudaStream_t st = as_stream(stream);
    const float* r = c_or_r;
    if (w.scan) {
        DUST_TRY(check_seq(seq_offsets, n_seq, K, T));
        float* rw = reinterpret_cast<float*>(region(ws, w.r_off));
        const cudaError_t e = dust::reward_scan_prefers_chunks(K, T, n_seq)
                                  ? dust::launch_reward_scan_chunks(c_or_r, rw, K, T, seq_offsets, n_seq, gamma,
                                                                    region(ws, w.chunk_off), st)
                                  : dust::launch_reward_scan(c_or_r, rw, K, T, seq_offsets, n_seq, gamma, st);
        DUST_TRY(cuda_status(e, "dust_layer_estimate_weight_grad (scan)"));
        r = rw;
    }
    const cudaError_t e = dust::launch_fused_estimate(r, T, d_out, X, d_in, nz, G_W, accumulate, g_hat_out,
                                                      region(ws, w.part_off), static_cast<uint32_t*>(ws), st);
    DUST_REQUIRE(e != cudaErrorNotSupported, DUST_ERR_UNSUPPORTED, "shape not supported by the fused kernel");
    return cuda_status(e, "dust_layer_estimate_weight_grad");
}

// ------------------------------------------------------------------ a6
static GemmPlan weight_grad_plan(int T, int d_in, int d_out, dust_dtype dt) {
    // C[d_out][d_in] = sum_t g[t][o] X[t][i]: A = g (M-major), B = X (N-major)
    return plan_gemm(d_out, d_in, T, dt, false, false);
}

// Operands of one type take that type's GEMM (bf16: tcgen05 where the shape
// allows); mixed types take the CUDA-core GEMM with both widened to fp32.
static GemmPlan weight_grad_plan2(int T, int d_in, int d_out, dust_dtype g_dt, dust_dtype x_dt) {
    return g_dt == x_dt ? weight_grad_plan(T, d_in, d_out, g_dt) : plan_gemm(d_out, d_in, T, DUST_F32, false, false);
}

size_t dust_weight_grad_workspace(int T, int d_in, int d_out, dust_dtype g_dt, dust_dtype x_dt) {
    Layout L;
    if (T > 0 && d_in > 0 && d_out > 0) L.add(weight_grad_plan2(T, d_in, d_out, g_dt, x_dt).partial_bytes);
    return L.off;
}

dust_status dust_weight_grad(const void* g_hat, dust_dtype g_dt, const void* X, dust_dtype x_dt, int T, int d_in,
                             int d_out, float* G_W, int accumulate, void* ws, size_t ws_bytes, void* stream) {
    DUST_REQUIRE(g_dt == DUST_F32 || g_dt == DUST_BF16, DUST_ERR_INVALID_ARG, "unknown g dtype %d",
                 static_cast<int>(g_dt));
    DUST_REQUIRE(x_dt == DUST_F32 || x_dt == DUST_BF16, DUST_ERR_INVALID_ARG, "unknown X dtype %d",
                 static_cast<int>(x_dt));
    DUST_REQUIRE(T > 0 && d_in > 0 && d_out > 0, DUST_ERR_INVALID_ARG, "T, d_in, d_out must be > 0");
    DUST_TRY(check_ptr(g_hat, "g_hat"));
    DUST_TRY(check_ptr(X, "X"));
    DUST_TRY(check_ptr(G_W, "G_W"));
    DUST_TRY(check_ptr(ws, "ws"));
    const size_t need = dust_weight_grad_workspace(T, d_in, d_out, g_dt, x_dt);
    DUST_REQUIRE(ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    const GemmPlan p = weight_grad_plan2(T, d_in, d_out, g_dt, x_dt);
    float* partial = reinterpret_cast<float*>(region(ws, dust::kStatusBytes));
    if (g_dt == x_dt)
        return run_gemm(p, g_hat, false, d_out, X, false, d_in, g_dt, d_out, d_in, T, G_W, d_in, accumulate, partial,
                        static_cast<uint32_t*>(ws), as_stream(stream));
    return cuda_status(dust::launch_gemm_simt_mixed(g_hat, g_dt, false, d_out, X, x_dt, false, d_in, d_out, d_in, T,
                                                    G_W, d_in, accumulate, partial, p.splits, as_stream(stream)),
                       "CUDA-core GEMM (mixed operand types)");
}

// ------------------------------------------------------------------ a2
static GemmPlan logits_plan(int T, int d_in, int V, dust_dtype dt) {
    // Z[T][V] = sum_k X[t][k] W[v][k]: A = X (K-major), B = W (K-major)
    return plan_gemm(T, V, d_in, dt, true, true);
}

size_t dust_logits_workspace(int T, int d_in, int V, dust_dtype dt) {
    Layout L;
    if (T > 0 && d_in > 0 && V > 0) L.add(logits_plan(T, d_in, V, dt).partial_bytes);
    return L.off;
}

dust_status dust_logits(const void* X, const void* W, dust_dtype dt, int T, int d_in, int V, float* Z, void* ws,
                        size_t ws_bytes, void* stream) {
    DUST_REQUIRE(dt == DUST_F32 || dt == DUST_BF16, DUST_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
    DUST_REQUIRE(T > 0 && d_in > 0 && V > 0, DUST_ERR_INVALID_ARG, "T, d_in, V must be > 0");
    DUST_TRY(check_ptr(X, "X"));
    DUST_TRY(check_ptr(W, "W"));
    DUST_TRY(check_ptr(Z, "Z"));
    DUST_TRY(check_ptr(ws, "ws"));
    const size_t need = dust_logits_workspace(T, d_in, V, dt);
    DUST_REQUIRE(ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    const GemmPlan p = logits_plan(T, d_in, V, dt);
    return run_gemm(p, X, true, d_in, W, true, d_in, dt, T, V, d_in, Z, V, 0,
                    reinterpret_cast<float*>(region(ws, dust::kStatusBytes)), static_cast<uint32_t*>(ws),
                    as_stream(stream));
}

dust_status dust_head_row_stats(const float* Z, const int32_t* targets, int T, int V, float* lse, float* ell,
                                void* stream) {
    DUST_REQUIRE(T > 0 && V > 0, DUST_ERR_INVALID_ARG, "T and V must be > 0");
    DUST_TRY(check_ptr(Z, "Z"));
    DUST_TRY(check_ptr(targets, "targets"));
    DUST_TRY(check_ptr(lse, "lse"));
    DUST_TRY(check_ptr(ell, "ell", true));
    return cuda_status(dust::launch_row_stats(Z, targets, T, V, lse, ell, as_stream(stream)), "dust_head_row_stats");
}

// ------------------------------------------------------------------ head step
namespace {
struct HeadLayout {
    size_t z = 0, lse = 0, g16 = 0, zpart = 0, wpart = 0, total = 0;
    GemmPlan zplan, wplan;
};

// Vr = the call's vocabulary range (chunk_count x Vc): g and its bf16 copy are
// [T][Vr], G_W [Vr][d_in]; the logits and their statistics cover all V.
HeadLayout head_layout(int T, int d_in, int V, int Vr, dust_dtype dt, int has_Z, int want_G_W) {
    HeadLayout h;
    Layout L;
    if (!has_Z) {
        h.zplan = logits_plan(T, d_in, V, dt);
        h.z = L.add(sizeof(float) * static_cast<size_t>(T) * V);
        h.zpart = L.add(h.zplan.partial_bytes);
    }
    h.lse = L.add(sizeof(float) * static_cast<size_t>(T));
    if (want_G_W) {
        h.wplan = weight_grad_plan(T, d_in, Vr, dt);
        if (dt == DUST_BF16) h.g16 = L.add(sizeof(uint16_t) * static_cast<size_t>(T) * Vr);
        h.wpart = L.add(h.wplan.partial_bytes);
    }
    h.total = L.off;
    return h;
}
}  // namespace

size_t dust_head_step_workspace(int T, int d_in, int V, int Vc, int chunk_count, dust_dtype dt, int has_Z,
                                int want_G_W) {
    if (T <= 0 || V <= 0 || Vc <= 0 || chunk_count <= 0 || ((!has_Z || want_G_W) && d_in <= 0))
        return dust::kStatusBytes;
    return head_layout(T, d_in, V, Vc * chunk_count, dt, has_Z, want_G_W).total;
}

dust_status dust_head_step(const void* X, const void* W, dust_dtype dt, const float* Z, const int32_t* targets, int T,
                           int d_in, int V, int Vc, int chunk_begin, int chunk_count, dust_noise nz, float* c_out,
                           float* g_hat, void* g_hat_bf16, float* G_W, int accumulate, void* ws, size_t ws_bytes,
                           void* stream) {
    DUST_TRY(check_noise(nz));
    DUST_REQUIRE(dt == DUST_F32 || dt == DUST_BF16, DUST_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
    DUST_REQUIRE(T > 0 && V > 0, DUST_ERR_INVALID_ARG, "T and V must be > 0");
    DUST_REQUIRE(Vc > 0 && V % Vc == 0, DUST_ERR_INVALID_ARG, "Vc=%d must divide V=%d", Vc, V);
    DUST_REQUIRE(dust::head_chunk_supported(Vc), DUST_ERR_UNSUPPORTED,
                 "Vc=%d unsupported (multiples of 128 up to 1024, of 256 up to 2048, of 512 up to 4096)", Vc);
    DUST_REQUIRE(V / Vc <= 65535, DUST_ERR_INVALID_ARG, "too many chunks");
    DUST_REQUIRE(chunk_begin >= 0 && chunk_count > 0 && chunk_begin + chunk_count <= V / Vc, DUST_ERR_INVALID_ARG,
                 "chunk range [%d, %d) outside the %d chunks", chunk_begin, chunk_begin + chunk_count, V / Vc);
    const int Vr = chunk_count * Vc;
    const bool has_Z = Z != nullptr, want_G_W = G_W != nullptr;
    if (!has_Z || want_G_W) {
        DUST_REQUIRE(d_in > 0, DUST_ERR_INVALID_ARG, "d_in must be > 0");
        DUST_TRY(check_ptr(X, "X"));
    }
    if (!has_Z) DUST_TRY(check_ptr(W, "W"));
    DUST_TRY(check_ptr(Z, "Z", true));
    DUST_TRY(check_ptr(targets, "targets"));
    DUST_TRY(check_ptr(c_out, "c_out", true));
    DUST_TRY(check_ptr(g_hat, "g_hat"));
    DUST_TRY(check_ptr(g_hat_bf16, "g_hat_bf16", true));
    DUST_TRY(check_ptr(G_W, "G_W", true));
    DUST_TRY(check_ptr(ws, "ws"));
    const HeadLayout h = head_layout(T, d_in, V, Vr, dt, has_Z, want_G_W);
    DUST_REQUIRE(ws_bytes >= h.total, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, h.total);
    cudaStream_t st = as_stream(stream);
    uint32_t* status = static_cast<uint32_t*>(ws);

    const float* Zuse = Z;
    if (!has_Z) {   // a2: clean logits into the workspace
        float* Zw = reinterpret_cast<float*>(region(ws, h.z));
        DUST_TRY(run_gemm(h.zplan, X, true, d_in, W, true, d_in, dt, T, V, d_in, Zw, V, 0,
                          reinterpret_cast<float*>(region(ws, h.zpart)), status, st));
        Zuse = Zw;
    }
    float* lse = reinterpret_cast<float*>(region(ws, h.lse));
    DUST_TRY(cuda_status(dust::launch_row_stats(Zuse, targets, T, V, lse, nullptr, st), "dust_head_step (row stats)"));
    void* g16 = g_hat_bf16;
    if (want_G_W && dt == DUST_BF16 && g16 == nullptr) g16 = region(ws, h.g16);
    DUST_TRY(cuda_status(dust::launch_head_chunks(Zuse, lse, targets, T, V, Vc, chunk_begin, chunk_count, nz, c_out,
                                                  g_hat, g16, accumulate, st),
                         "dust_head_step (chunks)"));
    if (!want_G_W) return ok();
    const void* gA = dt == DUST_BF16 ? g16 : static_cast<const void*>(g_hat);
    return run_gemm(h.wplan, gA, false, Vr, X, false, d_in, dt, Vr, d_in, T, G_W, d_in, 0,
                    reinterpret_cast<float*>(region(ws, h.wpart)), status, st);
}

// ------------------------------------------------------------------ cosine tuner
namespace {
struct BpLayout {
    size_t lse = 0, d = 0, part = 0, total = 0;
    GemmPlan plan;
};

BpLayout bp_layout(int T, int d_in, int V, dust_dtype dt) {
    BpLayout b;
    Layout L;
    b.plan = weight_grad_plan(T, d_in, V, dt);
    b.lse = L.add(sizeof(float) * static_cast<size_t>(T));
    b.d = L.add((dt == DUST_BF16 ? 2 : 4) * static_cast<size_t>(T) * V);
    b.part = L.add(b.plan.partial_bytes);
    b.total = L.off;
    return b;
}
}  // namespace

size_t dust_head_bp_grad_workspace(int T, int d_in, int V, dust_dtype dt) {
    if (T <= 0 || d_in <= 0 || V <= 0) return dust::kStatusBytes;
    return bp_layout(T, d_in, V, dt).total;
}

dust_status dust_head_bp_grad(const float* Z, const int32_t* targets, const void* X, dust_dtype dt, int T, int d_in,
                              int V, float* G_bp, void* ws, size_t ws_bytes, void* stream) {
    DUST_REQUIRE(dt == DUST_F32 || dt == DUST_BF16, DUST_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
    DUST_REQUIRE(T > 0 && d_in > 0 && V > 0, DUST_ERR_INVALID_ARG, "T, d_in, V must be > 0");
    DUST_TRY(check_ptr(Z, "Z"));
    DUST_TRY(check_ptr(targets, "targets"));
    DUST_TRY(check_ptr(X, "X"));
    DUST_TRY(check_ptr(G_bp, "G_bp"));
    DUST_TRY(check_ptr(ws, "ws"));
    const BpLayout b = bp_layout(T, d_in, V, dt);
    DUST_REQUIRE(ws_bytes >= b.total, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, b.total);
    cudaStream_t st = as_stream(stream);
    float* lse = reinterpret_cast<float*>(region(ws, b.lse));
    DUST_TRY(cuda_status(dust::launch_row_stats(Z, targets, T, V, lse, nullptr, st), "dust_head_bp_grad (row stats)"));
    void* D = region(ws, b.d);
    DUST_TRY(cuda_status(dust::launch_softmax_minus_onehot(Z, lse, targets, T, V, D, dt == DUST_BF16, st),
                         "dust_head_bp_grad (softmax - onehot)"));
    return run_gemm(b.plan, D, false, V, X, false, d_in, dt, V, d_in, T, G_bp, d_in, 0,
                    reinterpret_cast<float*>(region(ws, b.part)), static_cast<uint32_t*>(ws), st);
}

size_t dust_cosine_workspace(void) { return dust::align_up(dust::kStatusBytes + dust::cosine_partial_bytes(), 256); }

dust_status dust_cosine(const float* a, const float* b, long long n, double* out, void* ws, size_t ws_bytes,
                        void* stream) {
    DUST_REQUIRE(n > 0, DUST_ERR_INVALID_ARG, "n must be > 0");
    DUST_TRY(check_ptr(a, "a"));
    DUST_TRY(check_ptr(b, "b"));
    DUST_TRY(check_ptr(out, "out"));
    DUST_TRY(check_ptr(ws, "ws"));
    DUST_REQUIRE(ws_bytes >= dust_cosine_workspace(), DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes,
                 dust_cosine_workspace());
    return cuda_status(dust::launch_cosine(a, b, n, reinterpret_cast<double*>(region(ws, dust::kStatusBytes)), out,
                                           as_stream(stream)),
                       "dust_cosine");
}

// ------------------------------------------------------------------ harness
dust_status dust_noise_fill(dust_noise nz, uint32_t stream_id, int t0, int n_tok, int j0, int n_ch, float* out,
                            void* stream) {
    DUST_REQUIRE(nz.draw_count > 0, DUST_ERR_INVALID_ARG, "draw_count must be > 0");
    DUST_REQUIRE(t0 >= 0 && n_tok > 0 && j0 >= 0 && n_ch > 0, DUST_ERR_INVALID_ARG, "bad token/channel range");
    DUST_REQUIRE(static_cast<uint64_t>(nz.token_begin) + static_cast<uint64_t>(t0) + n_tok <= (1ull << 32),
                 DUST_ERR_INVALID_ARG, "token_begin + t0 + n_tok exceeds 2^32");
    DUST_TRY(check_ptr(out, "out"));
    return cuda_status(dust::launch_noise_fill(nz, stream_id, t0, n_tok, j0, n_ch, out, as_stream(stream)),
                       "dust_noise_fill");
}

dust_status dust_noise_sum(dust_noise nz, int T, int d, float* out, void* stream) {
    DUST_REQUIRE(nz.draw_count > 0, DUST_ERR_INVALID_ARG, "draw_count must be > 0");
    DUST_REQUIRE(static_cast<uint64_t>(nz.draw_begin) + nz.draw_count <= (1ull << 32), DUST_ERR_INVALID_ARG,
                 "draw_begin + draw_count exceeds 2^32");
    DUST_REQUIRE(nz.draw_count <= 0x7FFFFFFFu, DUST_ERR_INVALID_ARG, "draw_count must be < 2^31");
    DUST_REQUIRE(T > 0 && d > 0, DUST_ERR_INVALID_ARG, "T and d must be > 0");
    DUST_REQUIRE(nz.token_begin <= 0x7FFFFFFFu, DUST_ERR_INVALID_ARG, "token_begin must be < 2^31");
    DUST_REQUIRE(static_cast<long long>(T) * d < (1ll << 40), DUST_ERR_INVALID_ARG, "T x d too large");
    DUST_TRY(check_ptr(out, "out"));
    return cuda_status(dust::launch_noise_sum(nz, T, d, out, as_stream(stream)), "dust_noise_sum");
}

dust_status dust_box_muller_words(const uint32_t* a, const uint32_t* b, long long n, float* n_even, float* n_odd,
                                  void* stream) {
    DUST_REQUIRE(n > 0, DUST_ERR_INVALID_ARG, "n must be > 0");
    DUST_TRY(check_ptr(a, "a"));
    DUST_TRY(check_ptr(b, "b"));
    DUST_TRY(check_ptr(n_even, "n_even"));
    DUST_TRY(check_ptr(n_odd, "n_odd"));
    return cuda_status(dust::launch_box_muller_words(a, b, n, n_even, n_odd, as_stream(stream)), "dust_box_muller_words");
}

dust_status dust_synth_costs(const float* u, int T, int d_out, dust_noise nz, float eps_scale, float* c, void* stream) {
    DUST_REQUIRE(nz.draw_count > 0, DUST_ERR_INVALID_ARG, "draw_count must be > 0");
    DUST_REQUIRE(std::isfinite(nz.sigma) && nz.sigma >= 0.0f, DUST_ERR_INVALID_ARG, "sigma must be finite and >= 0");
    DUST_REQUIRE(std::isfinite(eps_scale), DUST_ERR_INVALID_ARG, "eps_scale must be finite");
    DUST_REQUIRE(T > 0 && d_out > 0, DUST_ERR_INVALID_ARG, "T and d_out must be > 0");
    DUST_REQUIRE(nz.draw_count <= 65535u * 32u, DUST_ERR_INVALID_ARG, "draw_count must be <= 2097120");
    DUST_REQUIRE(nz.token_begin <= 0x7FFFFFFFu, DUST_ERR_INVALID_ARG, "token_begin must be < 2^31");
    DUST_TRY(check_ptr(u, "u"));
    DUST_TRY(check_ptr(c, "c"));
    return cuda_status(dust::launch_synth_costs(u, T, d_out, nz, eps_scale, c, as_stream(stream)), "dust_synth_costs");
}

size_t dust_toy_suffix_workspace(int draw_count, int T, int d, int dh, int V) {
    if (draw_count <= 0 || T <= 0 || d <= 0 || dh <= 0 || V <= 0) return dust::kStatusBytes;
    return dust::toy_suffix_workspace_bytes(draw_count, T, d, dh, V);
}

dust_status dust_toy_suffix_losses(const float* Y, int T, int d, const int32_t* seq_offsets, int n_seq, const float* Wq,
                                   const float* Wk, const float* Wv, const float* Wo, int dh, const float* Wout, int V,
                                   const int32_t* targets, dust_noise nz, float* loss, float* c, void* ws,
                                   size_t ws_bytes, void* stream) {
    DUST_TRY(check_noise(nz));
    DUST_REQUIRE(T > 0 && d > 0 && dh > 0 && V > 0, DUST_ERR_INVALID_ARG, "T, d, dh, V must be > 0");
    DUST_REQUIRE(d % 4 == 0 && d <= 1024 && dh <= 128, DUST_ERR_UNSUPPORTED,
                 "toy suffix supports d %% 4 == 0, d <= 1024, dh <= 128");
    DUST_TRY(check_seq(seq_offsets, n_seq, 1, T));
    const void* ptrs[] = {Y, Wq, Wk, Wv, Wo, Wout, targets, loss, ws};
    const char* names[] = {"Y", "Wq", "Wk", "Wv", "Wo", "Wout", "targets", "loss", "ws"};
    for (int i = 0; i < 9; ++i) DUST_TRY(check_ptr(ptrs[i], names[i]));
    DUST_TRY(check_ptr(c, "c", true));
    const size_t need = dust_toy_suffix_workspace(static_cast<int>(nz.draw_count), T, d, dh, V);
    DUST_REQUIRE(ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    return cuda_status(dust::run_toy_suffix(Y, T, d, seq_offsets, n_seq, Wq, Wk, Wv, Wo, dh, Wout, V, targets, nz, loss,
                                            c, ws, as_stream(stream)),
                       "dust_toy_suffix_losses");
}

size_t dust_attention_internal_costs_workspace(int draw_count, int T, int d, int dh) {
    if (draw_count <= 0 || T <= 0 || d <= 0 || dh <= 0) return dust::kStatusBytes;
    return dust::attention_scoring_workspace_bytes(draw_count, T, d, dh);
}

dust_status dust_attention_internal_costs(const float* Y, int T, int d, const int32_t* seq_offsets, int n_seq,
                                          const float* Wq, const float* Wk, const float* Wv, const float* Wo,
                                          const float* Wg, const float* E, int dh, int which, const float* G,
                                          dust_noise nz, float* c, void* ws, size_t ws_bytes, void* stream) {
    DUST_TRY(check_noise(nz));
    DUST_REQUIRE(T > 0 && d > 0 && dh > 0, DUST_ERR_INVALID_ARG, "T, d, dh must be > 0");
    DUST_REQUIRE(which >= 0 && which <= 4, DUST_ERR_INVALID_ARG,
                 "which must be 0 (q), 1 (k), 2 (v), 3 (gate) or 4 (value embedding)");
    DUST_REQUIRE(which != 3 || (Wg != nullptr && E != nullptr), DUST_ERR_INVALID_ARG,
                 "gate draws need the gate's weights Wg and the value embeddings E");
    DUST_REQUIRE(which != 4 || E != nullptr, DUST_ERR_INVALID_ARG, "value-embedding draws need E");
    DUST_TRY(check_ptr(Wg, "Wg", true));
    DUST_TRY(check_ptr(E, "E", true));
    DUST_REQUIRE(dh % 4 == 0 && dh <= 128, DUST_ERR_UNSUPPORTED, "attention scoring supports dh %% 4 == 0, dh <= 128");
    DUST_TRY(check_seq(seq_offsets, n_seq, 1, T));
    const void* ptrs[] = {Y, Wq, Wk, Wv, Wo, G, c, ws};
    const char* names[] = {"Y", "Wq", "Wk", "Wv", "Wo", "G", "c", "ws"};
    for (int i = 0; i < 8; ++i) DUST_TRY(check_ptr(ptrs[i], names[i]));
    const size_t need = dust_attention_internal_costs_workspace(static_cast<int>(nz.draw_count), T, d, dh);
    DUST_REQUIRE(ws_bytes >= need, DUST_ERR_WORKSPACE, "workspace %zu bytes < %zu", ws_bytes, need);
    return cuda_status(dust::run_attention_internal_costs(Y, T, d, seq_offsets, n_seq, Wq, Wk, Wv, Wo, Wg, E, dh,
                                                          which, G, nz, c, ws, as_stream(stream)),
                       "dust_attention_internal_costs");
}

}  // extern "C"
