/*
 * dust.h -- C ABI of libdust.so, the B200 (sm_100a) hot path of the Dust
 * virtual-population gradient estimator for one linear layer and for the LM
 * head.
 *
 * Sources.  The method is stated in the cnblogs explainer "Dust: Pretraining
 * Transformers Without Backpropagation" (cnblogs.com/32bin/p/23212811):
 *   [CA]  section "信用分配：一次前向，两种奖励" (credit assignment):
 *         noise a_t ~ N(0, I) added as y_t + sigma a_t; centred per-token
 *         loss change c_s = l~_s - l_s; discounted reward
 *         r_t = sum_{s>=t} gamma^(s-t) c_s (reward equation); output-side
 *         error g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i) (error equation);
 *         weight estimate G_W = sum_t g_t x_t^T (weight equation).
 *   [IS3] section "真正的工作量：压住干扰" (interference suppression), third
 *         measure: the LM head perturbs the cached logits and recomputes only
 *         the cross entropy over one chunk of the vocabulary.
 * The noise a is regenerated from its coordinates by Philox4x32-10 (Salmon et
 * al., SC'11) and a Box-Muller transform with series ln/sin/cos; the exact
 * operation sequence is the library's noise specification and is identical,
 * bit for bit, to the one any conforming implementation produces.
 *
 * Conventions (every entry point):
 *   - All tensors are row-major, last index contiguous, in DEVICE memory of
 *     the current CUDA device unless a parameter says "host".
 *   - The caller owns every buffer, including the workspace.  The library
 *     never allocates, frees or synchronises; every call only enqueues work
 *     on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream) and returns.
 *   - Device pointers must be 16-byte aligned (DUST_ERR_ALIGNMENT otherwise).
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call launches nothing and returns a non-zero status.
 *     dust_last_error() then gives a message (thread-local).
 *   - Sequence offsets `seq_offsets` (device, int32 [n_seq + 1]) are read
 *     only by the kernels: offsets[0] = 0, non-decreasing, offsets[n_seq] = T.
 *     Kernels clamp every offset into [0, T], so offsets that break these
 *     rules cannot make a kernel touch memory outside its tensors, but the
 *     results are then unspecified; dust_check_offsets() validates a host
 *     copy.
 */
#ifndef DUST_H
#define DUST_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DUST_ABI_VERSION 2

typedef enum {
    DUST_OK = 0,
    DUST_ERR_INVALID_ARG = 1,   /* a size, pointer or value is out of range */
    DUST_ERR_UNSUPPORTED = 2,   /* a valid combination this build does not implement */
    DUST_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
    DUST_ERR_WORKSPACE = 4,     /* ws_bytes below the size the *_workspace query returns */
    DUST_ERR_CUDA = 5,          /* a CUDA launch or driver call failed */
    DUST_ERR_TIMEOUT = 6        /* a kernel's bounded wait ran out (reported by dust_poll_status) */
} dust_status;

typedef enum { DUST_F32 = 0, DUST_BF16 = 1 } dust_dtype;

/* Which draws of which layer a call handles, and where its tokens sit in the
 * global batch.  The noise element of draw i, token t (row t of the call's
 * tensors), channel j is a(seed, layer, i, token_begin + t, j).  A call
 * handles the global draws [draw_begin, draw_begin + draw_count) and scales by
 * the whole population K_total, so that splitting the draws of one estimate
 * over several calls (accumulate = 1) gives the same sum [CA, error equation];
 * token_begin is the global index of the call's first token, so that a batch
 * split by whole sequences over several calls or ranks draws, token for
 * token, the noise of one call over the whole batch ([CA]: a_t is drawn per
 * token). */
typedef struct {
    uint32_t seed;        /* Philox key word 0 */
    uint32_t layer;       /* Philox key word 1 (one value per perturbed layer) */
    uint32_t draw_begin;  /* first global draw index handled by this call */
    uint32_t draw_count;  /* number of draws handled by this call (> 0) */
    uint32_t K_total;     /* population size K of the 1/(K sigma) scale (> 0) */
    float sigma;          /* noise scale (> 0, finite) */
    uint32_t token_begin; /* global index of row 0 of the call's tokens (< 2^31) */
} dust_noise;

/* ------------------------------------------------------------------ status */

const char *dust_status_string(dust_status s);
/* Message of the last failed call on this host thread ("" if none). */
const char *dust_last_error(void);
int dust_abi_version(void);

/* Host-side validation of sequence offsets (HOST pointer, n_seq + 1 entries). */
dust_status dust_check_offsets(const int32_t *seq_offsets_host, int n_seq, int T);

/* Reads and clears the device status word at the start of a workspace that a
 * previous call on `stream` was given (synchronises `stream`).  Returns
 * DUST_ERR_TIMEOUT if a kernel's bounded wait ran out, else DUST_OK. */
dust_status dust_poll_status(void *ws, void *stream);

/* Failure-detection self-test: one thread waits, through the same bounded
 * mbarrier wait the tcgen05 pipeline uses, on a barrier that nothing
 * completes; after `polls` polls (1 .. 2^20, with back-off: well under a
 * second) it gives up and sets the status word of `ws`, so that a following
 * dust_poll_status(ws) returns DUST_ERR_TIMEOUT.  Nothing faults or hangs and
 * the context stays usable. */
dust_status dust_selftest_bounded_wait(void *ws, uint32_t polls, void *stream);

/* ------------------------------------------------------------------ a4: reward
 * [CA, reward equation] r[i][t] = sum_{s>=t, s in seq(t)} gamma^(s-t) c[i][s].
 * c, r: [K][T] fp32; r may alias c (in place).  The sum stays inside the
 * token's sequence (causal attention does not cross sequences).  gamma = 0
 * gives r = c bit for bit.  0 <= gamma <= 1.  No workspace. */
dust_status dust_reward_scan(const float *c, float *r, int K, int T,
                             const int32_t *seq_offsets, int n_seq, float gamma,
                             void *stream);

/* Same result as dust_reward_scan, computed over fixed 1024-token chunks of
 * every draw row in parallel (the chunk maps x -> c + g x are composed per
 * chunk, the carries between chunks resolved in a second step, then every
 * chunk rescanned with its carry).  For few, long sequences, where the
 * per-sequence scan has too few blocks to fill the GPU.  Reads c twice.
 * r may alias c.  Workspace: dust_reward_scan_split_workspace(). */
dust_status dust_reward_scan_split(const float *c, float *r, int K, int T,
                                   const int32_t *seq_offsets, int n_seq, float gamma,
                                   void *ws, size_t ws_bytes, void *stream);
size_t dust_reward_scan_split_workspace(int K, int T);

/* ------------------------------------------------------------------ a5: error
 * [CA, error equation] g_hat[t][j] (+)= -(1/(K_total sigma))
 *     sum_{k < draw_count} r[k][t] a(seed, layer, draw_begin + k, t, j).
 * c_or_r: [draw_count][T] fp32, row k belongs to draw draw_begin + k.  If
 * is_r == 0 it holds the costs c and the reward scan (a4) runs first into the
 * workspace (skipped when gamma == 0, where r = c); otherwise it holds r.
 * g_hat: [T][d_out] fp32, overwritten (accumulate = 0) or added to
 * (accumulate = 1).  g_hat_bf16: nullable [T][d_out] bf16, receives
 * round-to-nearest-even of the final g_hat.  Workspace:
 * dust_layer_estimate_workspace(). */
dust_status dust_layer_estimate(const float *c_or_r, int is_r, int T, int d_out,
                                const int32_t *seq_offsets, int n_seq, float gamma,
                                dust_noise nz, float *g_hat, void *g_hat_bf16,
                                int accumulate, void *ws, size_t ws_bytes, void *stream);
size_t dust_layer_estimate_workspace(int draw_count, int T, int d_out, int is_r, float gamma);

/* Allocation-free form of dust_layer_estimate with is_r = 0, for callers that
 * cannot call cudaMalloc: for example a plugin inside a host framework that
 * owns all device memory and hands it only the device pointers of its inputs
 * and outputs, or a caller whose memory pool is fully reserved.  The pages
 * have no counterpart: it is a deployment variant of the same computation
 * (reward scan into scratch, then the draw reduction) whose scratch is a fixed
 * device array inside the library image instead of a workspace: 16 MiB for
 * the rewards plus 64 KiB for the chunk maps of the chunked scan.
 *   c: [draw_count][T] fp32 costs; other arguments as dust_layer_estimate.
 *   The scan takes dust_layer_estimate's path (per sequence, or over
 *   1024-token chunks for few long sequences), so the result is the same bits.
 *   Limit: draw_count * T <= 4194304 when gamma > 0 (DUST_ERR_WORKSPACE
 *   otherwise, nothing launched); split the draws over calls with
 *   accumulate = 1 for more.  gamma = 0 uses no scratch.
 *   The array costs 16.06 MiB on every GPU that loads the library, until exit.
 *   It is shared by all calls: calls whose kernels may overlap on the GPU race
 *   on it and must be serialised by the caller.  It keeps the last call's
 *   contents; nothing needs to start at zero (the scan rewrites every r the
 *   reduction reads).
 *   Set-up: the first call on a device looks the array's device address up
 *   (cudaGetSymbolAddress) with that device current and caches it for the
 *   process; make that first call before any stream capture.  After
 *   cudaDeviceReset of a device the cached address is stale: do not call this
 *   entry point on that device again.  The call allocates nothing (no
 *   cudaMalloc, cudaFree or allocating library routine). */
dust_status dust_layer_estimate_noalloc(const float *c, int T, int d_out,
                                        const int32_t *seq_offsets, int n_seq, float gamma,
                                        dust_noise nz, float *g_hat, void *g_hat_bf16,
                                        int accumulate, void *stream);

/* ------------------------------------------------------------------ a1 + a5 + a6 fused
 * [CA, error and weight equations] G_W[o][i] (+)= sum_t bf16(g_hat[t][o]) X[t][i]
 * with g_hat as dust_layer_estimate computes it, produced tile by tile in
 * shared memory as the tensor cores' operand and never written to device
 * memory (unless g_hat_out is given): one kernel runs the draw reduction and
 * the tcgen05 weight GEMM, with the d_in-wide row block of G_W held in TMEM.
 *   c_or_r, is_r, T, d_out, seq_offsets, n_seq, gamma, nz: as
 *     dust_layer_estimate (the reward scan, when needed, runs first into the
 *     workspace);
 *   X: [T][d_in] bf16, 16-byte aligned; d_in a multiple of 64, at most 512
 *     (one CTA's TMEM holds 512 fp32 columns), else DUST_ERR_UNSUPPORTED;
 *   G_W: [d_out][d_in] fp32, overwritten (accumulate = 0) or added to;
 *   g_hat_out: nullable [T][d_out] fp32, receives g_hat (the same bits as
 *     dust_layer_estimate's g_hat) for checks.
 *   draw_count: at most 1048576 per call (DUST_ERR_UNSUPPORTED otherwise);
 *     split larger populations over calls with accumulate = 1.  The kernel's
 *     waits on a stage's production are bounded by a time budget that grows
 *     with the draw count (2 s + 20 us per draw), after which it sets the
 *     status word (DUST_ERR_TIMEOUT from dust_poll_status) and returns.
 * The bf16 g values are those of dust_layer_estimate's g_hat_bf16, so G_W
 * agrees with dust_layer_estimate followed by dust_weight_grad up to the
 * order of the fp32 accumulation.  Token splits are summed in a fixed order.
 * Workspace: dust_layer_estimate_weight_grad_workspace(); its first 256 bytes
 * are the status block read by dust_poll_status. */
dust_status dust_layer_estimate_weight_grad(const float *c_or_r, int is_r, int T, int d_out,
                                            const int32_t *seq_offsets, int n_seq, float gamma,
                                            dust_noise nz, const void *X, int d_in, float *G_W,
                                            int accumulate, float *g_hat_out, void *ws, size_t ws_bytes,
                                            void *stream);
size_t dust_layer_estimate_weight_grad_workspace(int draw_count, int T, int d_in, int d_out, int is_r,
                                                 float gamma);

/* ------------------------------------------------------------------ a6: weight
 * [CA, weight equation] G_W[o][i] (+)= sum_t g_hat[t][o] X[t][i].
 * g_hat: [T][d_out] of dtype g_dt, X: [T][d_in] of dtype x_dt.  Both bf16:
 * the tcgen05 tensor cores with fp32 accumulation in TMEM when d_in and d_out
 * are multiples of 8 (16-byte rows for the TMA; else CUDA cores), any T;
 * both fp32: fp32 CUDA cores; mixed (fp32 g with bf16 X, or bf16 g with fp32
 * X): CUDA cores, each bf16 element widened to fp32 exactly, fp32 products.
 * G_W: [d_out][d_in] fp32 (the layout of W).  Split over T with a fixed-order
 * reduction: results do not depend on the launch.
 * Workspace: dust_weight_grad_workspace(). */
dust_status dust_weight_grad(const void *g_hat, dust_dtype g_dt, const void *X, dust_dtype x_dt,
                             int T, int d_in, int d_out, float *G_W, int accumulate,
                             void *ws, size_t ws_bytes, void *stream);
size_t dust_weight_grad_workspace(int T, int d_in, int d_out, dust_dtype g_dt, dust_dtype x_dt);

/* ------------------------------------------------------------------ a2: logits
 * Clean head forward Z[t][v] = sum_k X[t][k] W[v][k] (no bias), fp32 out.
 * X: [T][d_in], W: [V][d_in] of dtype dt (bf16: tcgen05 when d_in is a
 * multiple of 8, else CUDA cores; f32: CUDA cores).  Z: [T][V] fp32, 16-byte
 * aligned; written by TMA stores when V is a multiple of 4, by row stores
 * otherwise (the same values).
 * Workspace: dust_logits_workspace(). */
dust_status dust_logits(const void *X, const void *W, dust_dtype dt, int T, int d_in,
                        int V, float *Z, void *ws, size_t ws_bytes, void *stream);
size_t dust_logits_workspace(int T, int d_in, int V, dust_dtype dt);

/* Per-token clean statistics of cached logits: lse[t] = log sum_v exp Z[t][v],
 * ell[t] = lse[t] - Z[t][targets[t]] (the clean loss l_t).  ell nullable.
 * targets: [T] int32 in [0, V). */
dust_status dust_head_row_stats(const float *Z, const int32_t *targets, int T, int V,
                                float *lse, float *ell, void *stream);

/* ------------------------------------------------------------------ a2+a3+a5+a6: head
 * [IS3] LM-head step over the vocabulary chunks [chunk_begin, chunk_begin +
 * chunk_count) of width Vc (all of them: chunk_begin = 0, chunk_count = V/Vc).
 * The chunk passes are independent given the clean logits, so the chunks can
 * be split over calls or ranks (head sharding by vocabulary); their g columns
 * and G_W rows are disjoint.  For chunk
 * [v0, v0 + Vc) and draw i, the logits of the chunk are perturbed,
 * z~ = z + sigma a(i, t, v) for v in the chunk, and the change of the
 * full-vocabulary cross entropy is [CA] c = CE(z~, y) - CE(z, y), computed as
 * log1p(sum_{v in chunk} p_v expm1(sigma a_v)) - sigma a_y [y in chunk] with
 * p = softmax(z) (an exact identity).  With gamma = 0 (head) r = c and
 * g_hat[t][v] (+)= -(1/(K_total sigma)) sum_i c a(i, t, v) for v in the chunk.
 * Noise channel = global vocab id v, so results do not depend on Vc.
 *   X: [T][d_in], W: [V][d_in] of dtype dt; used when Z is NULL (Z is then
 *      recomputed into the workspace, a2) and when G_W is requested.
 *   Z: nullable cached logits [T][V] fp32.
 *   targets: [T] int32 in [0, V).
 *   Vc: chunk width; must divide V; supported: multiples of 128 up to 1024,
 *      of 256 up to 2048 and of 512 up to 4096 (Vc = V is the reading where
 *      every draw perturbs the whole vocabulary).
 *   chunk_begin, chunk_count: the chunk range (0 <= chunk_begin,
 *      chunk_count >= 1, chunk_begin + chunk_count <= V/Vc); below,
 *      Vr = chunk_count Vc and column / row m of the outputs is vocabulary id
 *      chunk_begin Vc + m.  The statistics lse and the softmax p always cover
 *      the whole vocabulary.
 *   c_out: nullable [chunk_count][draw_count][T] fp32, the costs of every pass.
 *   g_hat: [T][Vr] fp32 (overwritten, or added to when accumulate = 1).
 *   g_hat_bf16: nullable [T][Vr] bf16 copy of the final g_hat.
 *   G_W: nullable [Vr][d_in] fp32, overwritten with g_hat^T X (a6) computed
 *      from the final g_hat (requires X): rows chunk_begin Vc .. + Vr of the
 *      full head's estimate.
 * Workspace: dust_head_step_workspace() with the same chunk_count. */
dust_status dust_head_step(const void *X, const void *W, dust_dtype dt, const float *Z,
                           const int32_t *targets, int T, int d_in, int V, int Vc,
                           int chunk_begin, int chunk_count, dust_noise nz, float *c_out,
                           float *g_hat, void *g_hat_bf16, float *G_W, int accumulate,
                           void *ws, size_t ws_bytes, void *stream);
size_t dust_head_step_workspace(int T, int d_in, int V, int Vc, int chunk_count, dust_dtype dt,
                                int has_Z, int want_G_W);

/* ------------------------------------------------------------------ cosine tuner
 * cnblogs Dust explainer, section "真正的工作量：压住干扰" (last paragraph): the
 * hyper-parameters can be chosen by maximising, on one batch, the cosine
 * between the Dust estimate and the backprop gradient; section
 * "梯度是"长"出来的": cos(K) = c_max / sqrt(1 + c/K).
 *
 * Backprop gradient of the head's summed cross entropy on cached logits:
 * G_bp[v][i] = sum_t (softmax(Z_t)[v] - [v == y_t]) X[t][i]  ([V][d_in] fp32).
 * With the literal sign of the error equation the Dust head estimate
 * approaches -G_bp.  X: [T][d_in] of dtype dt (bf16: tensor cores, the
 * softmax difference rounded to bf16; f32: CUDA cores).  Workspace:
 * dust_head_bp_grad_workspace(). */
dust_status dust_head_bp_grad(const float *Z, const int32_t *targets, const void *X, dust_dtype dt,
                              int T, int d_in, int V, float *G_bp, void *ws, size_t ws_bytes,
                              void *stream);
size_t dust_head_bp_grad_workspace(int T, int d_in, int V, dust_dtype dt);

/* out (device, 4 doubles) = { sum a b, sum a a, sum b b, cosine } over n fp32
 * elements, accumulated in double in a fixed order (deterministic).
 * Workspace: dust_cosine_workspace(). */
dust_status dust_cosine(const float *a, const float *b, long long n, double *out, void *ws,
                        size_t ws_bytes, void *stream);
size_t dust_cosine_workspace(void);

/* ------------------------------------------------------------------ harness / debug
 * Noise: out[k][t][j] = a(seed, layer, draw_begin + k, t0 + t, j0 + j) from
 * Philox stream `stream_id` (0: activation noise, 1: synthetic observation
 * noise).  out: [draw_count][n_tok][n_ch] fp32. */
dust_status dust_noise_fill(dust_noise nz, uint32_t stream_id, int t0, int n_tok,
                            int j0, int n_ch, float *out, void *stream);

/* The generator's empirical ceiling, for measurement: the noise of a draw
 * range summed per token and channel,
 *   out[t][j] = sum_{k < draw_count} a(seed, layer, draw_begin + k, token_begin + t, j),
 * with the noise of the per-token, per-draw N(0, I) activation perturbation
 * (cnblogs Dust explainer, section "信用分配：一次前向，两种奖励").  Each
 * Gaussian is consumed by one fused multiply-add that also applies the
 * Box-Muller radius (acc + rho cos, rounded once), and nothing but out touches
 * HBM, so its Gaussians/s bound every noise consumer of this library.  The sum
 * runs in fp32 in a fixed order (even draws and odd draws in two partial sums
 * added at the end); it equals the sum of the binary32 noise values to within
 * fp32 rounding.  sigma and K_total are not used.  out: [T][d] fp32 (device,
 * 16-byte aligned), overwritten.  Errors: DUST_ERR_INVALID_ARG for T, d or
 * draw_count <= 0, draw_count >= 2^31, a draw or token range beyond 2^32 or
 * token_begin >= 2^31; DUST_ERR_ALIGNMENT; DUST_ERR_CUDA for a launch error. */
dust_status dust_noise_sum(dust_noise nz, int T, int d, float *out, void *stream);

/* The noise generator's Box-Muller step on caller-given Philox word pairs:
 * (n_even[i], n_odd[i]) = transform(a[i], b[i]).  a, b: [n] uint32; outputs
 * [n] fp32.  For exhaustive bit-exactness checks of the specification. */
dust_status dust_box_muller_words(const uint32_t *a, const uint32_t *b, long long n,
                                  float *n_even, float *n_odd, void *stream);

/* Synthetic linear costs standing in for a perturbed forward:
 * c[k][s] = sigma <u[s], a(draw_begin+k, s, .)> + eps_scale * a_stream1(draw_begin+k, s, 0).
 * u: [T][d_out] fp32, c: [draw_count][T] fp32. */
dust_status dust_synth_costs(const float *u, int T, int d_out, dust_noise nz,
                             float eps_scale, float *c, void *stream);

/* Toy causal suffix scoring a perturbed hidden linear layer (fp32 CUDA cores):
 * y~ = Y + sigma a(draw), h = y~ + Attn(y~) Wo^T (one causal softmax head of
 * width dh per sequence; q, k, v = y~ Wq^T, y~ Wk^T, y~ Wv^T, scores scaled by
 * 1/sqrt(dh)), z = h Wout^T, loss = logsumexp(z) - z[target].
 * Y: [T][d] clean layer output; Wq, Wk, Wv: [dh][d]; Wo: [d][dh]; Wout: [V][d].
 * loss: [draw_count + 1][T]; row 0 is the clean loss, row 1 + k draw
 * draw_begin + k.  If c is non-NULL it receives c[k][t] = row(1+k) - row(0).
 * Supported: d <= 1024, dh <= 128, d % 4 == 0.  Workspace: dust_toy_suffix_workspace(). */
dust_status dust_toy_suffix_losses(const float *Y, int T, int d, const int32_t *seq_offsets,
                                   int n_seq, const float *Wq, const float *Wk, const float *Wv,
                                   const float *Wo, int dh, const float *Wout, int V,
                                   const int32_t *targets, dust_noise nz, float *loss, float *c,
                                   void *ws, size_t ws_bytes, void *stream);
size_t dust_toy_suffix_workspace(int draw_count, int T, int d, int dh, int V);

/* Attention-internal scoring (cnblogs Dust explainer, section
 * "真正的工作量：压住干扰", second measure): the draws of one internal quantity
 * of a causal softmax attention head (query, key, value, gate, value
 * embedding; noise channel = that quantity's channel, dh wide) are scored
 * through the attention output z = Attn(q, k, v) Wo^T against its estimated
 * error G:
 *   c[k][t] = -< z~_t - z_t, G_t >   (first order: the loss change l~ - l),
 * computed as -< o~_t - o_t, G_t Wo > since z is linear in the attention's
 * value output o.  q, k = Y Wq^T, Y Wk^T (scores / sqrt(dh)), one head per
 * sequence.  The values carry each token's value embedding through a gate:
 *   v_t = Y_t Wv^T + s(Y_t Wg^T) * E_t   (s = logistic sigmoid per channel;
 *                                         s = 1 when Wg is NULL; E NULL: no
 *                                         embedding, v = Y Wv^T).
 * The library's reading of the pages, which name the gate and the value
 * embedding among the attention's internals and say both are read by later
 * tokens (credit-assignment section): both act on the values.
 *   which: 0 = q, 1 = k, 2 = v (the noise is added to the projection),
 *          3 = the gate's pre-activation Y Wg^T (needs Wg and E),
 *          4 = the value embedding E (needs E).
 * Y, G: [T][d]; Wq, Wk, Wv, Wg: [dh][d]; Wo: [d][dh]; E: [T][dh];
 * c: [draw_count][T].  The costs feed dust_layer_estimate with d_out = dh
 * (the pages give keys, values, gates and value embeddings a discount gamma
 * close to 1).  Supported: dh % 4 == 0, dh <= 128.  fp32 CUDA cores.
 * Workspace: dust_attention_internal_costs_workspace(). */
dust_status dust_attention_internal_costs(const float *Y, int T, int d, const int32_t *seq_offsets,
                                          int n_seq, const float *Wq, const float *Wk,
                                          const float *Wv, const float *Wo, const float *Wg,
                                          const float *E, int dh, int which, const float *G,
                                          dust_noise nz, float *c, void *ws, size_t ws_bytes,
                                          void *stream);
size_t dust_attention_internal_costs_workspace(int draw_count, int T, int d, int dh);

#ifdef __cplusplus
}
#endif
#endif /* DUST_H */
