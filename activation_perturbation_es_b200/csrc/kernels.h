// kernels.h -- internal launchers (one per kernel family).  Each enqueues on
// `stream` and returns the launch status; argument validation happens in
// api.cu before any of these is called.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "dust.h"

namespace dust {

// a4 (reward_scan.cu)
cudaError_t launch_reward_scan(const float* c, float* r, int K, int T, const int32_t* offs,
                               int n_seq, float gamma, cudaStream_t stream);

// a4 for few long sequences: chunked three-pass scan; scratch holds
// reward_scan_chunks_workspace(K, T) bytes (chunk maps and carries)
size_t reward_scan_chunks_workspace(int K, int T);
bool reward_scan_prefers_chunks(int K, int T, int n_seq);
cudaError_t launch_reward_scan_chunks(const float* c, float* r, int K, int T, const int32_t* offs, int n_seq,
                                      float gamma, void* scratch, cudaStream_t stream);

// a1 + a5 (layer_estimate.cu): g (+)= scale * sum_k r[k][t] a(draw_begin + k, t, j)
cudaError_t launch_layer_estimate(const float* r, int T, int d_out, const dust_noise& nz,
                                  float* g, void* g_bf16, int accumulate, cudaStream_t stream);

// a1 harness (noise_fill.cu)
cudaError_t launch_noise_fill(const dust_noise& nz, uint32_t stream_id, int t0, int n_tok, int j0,
                              int n_ch, float* out, cudaStream_t stream);
cudaError_t launch_box_muller_words(const uint32_t* a, const uint32_t* b, long long n, float* ne, float* no,
                                    cudaStream_t stream);
cudaError_t launch_synth_costs(const float* u, int T, int d_out, const dust_noise& nz,
                               float eps_scale, float* c, cudaStream_t stream);
// the generator's ceiling (noise_sum.cu): out[t][j] = sum_k a(draw_begin + k, token_begin + t, j)
cudaError_t launch_noise_sum(const dust_noise& nz, int T, int d, float* out, cudaStream_t stream);

// a6 / a2 on CUDA cores (gemm_simt.cu):
//   C[m][n] = sum_k A(m, k) B(k, n), C row-major [M][N] with leading dim ldc.
//   A(m, k) = a_kmajor ? A[m * lda + k] : A[k * lda + m]
//   B(k, n) = b_kmajor ? B[n * ldb + k] : B[k * ldb + n]
// Split over k into `splits` slices; slice s writes partial[s][M][N] (fp32)
// unless splits == 1, in which case it writes (or adds to, accumulate) C.
cudaError_t launch_gemm_simt(const void* A, bool a_kmajor, int lda, const void* B, bool b_kmajor,
                             int ldb, dust_dtype dt, int M, int N, int K, float* C, int ldc,
                             int accumulate, float* partial, int splits, cudaStream_t stream);
// the same with A and B of different types (each widened to fp32 exactly)
cudaError_t launch_gemm_simt_mixed(const void* A, dust_dtype a_dt, bool a_kmajor, int lda, const void* B,
                                   dust_dtype b_dt, bool b_kmajor, int ldb, int M, int N, int K, float* C, int ldc,
                                   int accumulate, float* partial, int splits, cudaStream_t stream);
int gemm_simt_splits(int M, int N, int K);
// C (+)= sum_s partial[s]  (fixed order), C [M][N] leading dim ldc
cudaError_t launch_splitk_reduce(const float* partial, int splits, int M, int N, float* C, int ldc,
                                 int accumulate, cudaStream_t stream);

// a6 / a2 on tcgen05 tensor cores (gemm_tcgen05.cu), bf16 operands, fp32 out.
// Same contract as launch_gemm_simt; returns cudaErrorNotSupported when the
// shape is outside what the kernel handles (multiples of 16 in M, N).
cudaError_t launch_gemm_tc(const void* A, bool a_kmajor, int lda, const void* B, bool b_kmajor,
                           int ldb, int M, int N, int K, float* C, int ldc, int accumulate,
                           float* partial, int splits, uint32_t* status, cudaStream_t stream);
int gemm_tc_splits(int M, int N, int K);
cudaError_t launch_bounded_wait_selftest(uint32_t* status, uint32_t polls, cudaStream_t stream);
bool gemm_tc_supported(int M, int N, int K, bool a_kmajor, bool b_kmajor);
// 2-D bf16 tensor map [outer][inner], row pitch ld elements, box {64, box_outer},
// 128-byte swizzle; false when the driver entry point or the encoding fails
bool tma_map_bf16_2d(CUtensorMap* map, const void* base, int inner, int outer, int ld, int box_outer);
int device_sm_count();

// a1 + a5 + a6 fused (fused_estimate.cu): G (+)= sum_t bf16(g_t) x_t^T with g
// produced in shared memory (never written unless g_hat is given);
// d_in a multiple of 64 up to 512.  scratch holds fused_estimate_scratch()
// bytes (fp32 partial G row blocks, one per token split).
bool fused_estimate_supported(int d_in, int d_out);
// draws per call of the fused kernel: its waits on a stage's production are
// bounded by a time budget that grows with the draw count
constexpr uint32_t kFusedMaxDraws = 1u << 20;
size_t fused_estimate_scratch(int T, int d_in, int d_out);
cudaError_t launch_fused_estimate(const float* r, int T, int d_out, const void* X, int d_in, const dust_noise& nz,
                                  float* G, int accumulate, float* g_hat, void* scratch, uint32_t* status,
                                  cudaStream_t stream);

// a2 row statistics + a3/a5 fused head (head.cu)
cudaError_t launch_row_stats(const float* Z, const int32_t* targets, int T, int V, float* lse,
                             float* ell, cudaStream_t stream);
bool head_chunk_supported(int Vc);
// chunks [chunk_begin, chunk_begin + chunk_count) of width Vc; g and g_bf16 are
// [T][chunk_count Vc] (the range's columns), c_out [chunk_count][draw_count][T]
cudaError_t launch_head_chunks(const float* Z, const float* lse, const int32_t* targets, int T,
                               int V, int Vc, int chunk_begin, int chunk_count, const dust_noise& nz,
                               float* c_out, float* g, void* g_bf16, int accumulate, cudaStream_t stream);

// harness: toy causal suffix (toy_suffix.cu)
size_t toy_suffix_workspace_bytes(int draw_count, int T, int d, int dh, int V);
cudaError_t run_toy_suffix(const float* Y, int T, int d, const int32_t* offs, int n_seq, const float* Wq,
                           const float* Wk, const float* Wv, const float* Wo, int dh, const float* Wout, int V,
                           const int32_t* targets, const dust_noise& nz, float* loss, float* c, void* ws,
                           cudaStream_t st);

// cosine tuner support (tuner.cu)
cudaError_t launch_softmax_minus_onehot(const float* Z, const float* lse, const int32_t* targets, int T, int V,
                                        void* D, bool bf16, cudaStream_t stream);
size_t cosine_partial_bytes();
cudaError_t launch_cosine(const float* a, const float* b, long long n, double* part, double* out,
                          cudaStream_t stream);

// error reporting for entry points outside api.cu
dust_status record_error(dust_status s, const char* msg);

// causal softmax attention per sequence (toy_suffix.cu); q, k, v [nb][T][dh]
// with batch strides in elements (0: shared by the batch), o [nb][T][dh]
cudaError_t launch_causal_attention(const float* q, const float* k, const float* v, long long q_bs, long long k_bs,
                                    long long v_bs, int nb, int T, int dh, const int32_t* offs, int n_seq,
                                    float* o, cudaStream_t stream);

// attention-internal scoring (attention_scoring.cu)
size_t attention_scoring_workspace_bytes(int draw_count, int T, int d, int dh);
// which: 0 q, 1 k, 2 v, 3 the gate's pre-activation Y Wg^T, 4 the value
// embedding E; the values are Y Wv^T + s(Y Wg^T) E (Wg, E nullable)
cudaError_t run_attention_internal_costs(const float* Y, int T, int d, const int32_t* offs, int n_seq,
                                         const float* Wq, const float* Wk, const float* Wv, const float* Wo,
                                         const float* Wg, const float* E, int dh, int which, const float* G,
                                         const dust_noise& nz, float* c, void* ws, cudaStream_t st);

// fp32 -> bf16 (RNE) copy
cudaError_t launch_to_bf16(const float* src, void* dst, size_t n, cudaStream_t stream);

}  // namespace dust
