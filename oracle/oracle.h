/*
 * oracle.h -- plain CPU oracle for the Dust estimator hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never includes, links or calls it, and
 * the two share no code: the noise specification is implemented here a second
 * time, independently, from its written definition.
 *
 * Conventions
 *   - Row-major arrays, last index contiguous.
 *   - Noise values are binary32 and bit-exact by construction (every step of
 *     the noise specification is a correctly rounded IEEE operation).
 *   - Everything downstream of the noise (losses, rewards, the error estimate,
 *     the weight estimate) is accumulated in double.
 *   - Draws are summed in ascending order, tokens in ascending order.
 *
 * Sources (cited per function):
 *   [P2]  cnblogs explainer "Dust: Pretraining Transformers Without
 *         Backpropagation" (cnblogs.com/32bin/p/23212811).  Section
 *         "信用分配：一次前向，两种奖励" (credit assignment) holds the noise
 *         definition a_t ~ N(0, I), the centred loss change c_s, the reward
 *         equation r_t, the error-estimate equation g_t and the weight-estimate
 *         equation G_W.  Section "真正的工作量：压住干扰" (interference
 *         suppression), third measure, describes the LM-head variant that
 *         perturbs cached logits over one vocabulary chunk.
 *   [PHILOX] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *         1, 2, 3", SC'11 -- the Philox4x32 bijection, 10 rounds.
 *   [BM]  Box & Muller, "A Note on the Generation of Random Normal Deviates",
 *         Ann. Math. Statist. 29 (1958).
 */
#ifndef DUST_ORACLE_H
#define DUST_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------- noise specification (a_t^(i)[j] ~ N(0,1)) ---------------- */

/* Philox4x32-10 [PHILOX]: out = bijection(ctr) under key. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* Natural log of u in [2^-23, 1] by the spec's atanh series (binary32). */
float orc_ln(float u);

/* sin(phi), cos(phi) for phi in [0, pi/4] by the spec's Taylor series. */
void orc_sincos_quarter(float phi, float *s, float *c);

/* Box-Muller pair [BM] from two Philox words: n_even = rho cos(theta),
 * n_odd = rho sin(theta). */
void orc_box_muller(uint32_t a, uint32_t b, float *n_even, float *n_odd);

/* One Gaussian: key (seed, layer), counter (channel>>2, token, draw, stream). */
float orc_gauss(uint32_t seed, uint32_t layer, uint32_t draw, uint32_t token,
                uint32_t channel, uint32_t stream);

/* Batch forms of the above (elementwise), for exhaustive checks. */
void orc_philox_batch(const uint32_t *ctr, const uint32_t *key, int n, uint32_t *out);
void orc_ln_batch(const float *u, int n, float *out);
void orc_sincos_batch(const float *phi, int n, float *s, float *c);
void orc_box_muller_batch(const uint32_t *a, const uint32_t *b, int n, float *ne, float *no);

/* out[d][t][c] = gauss(seed, layer, draw0+d, tokens[t], ch0+c, stream). */
void orc_noise_block(uint32_t seed, uint32_t layer, uint32_t stream,
                     uint32_t draw0, int nd, const int32_t *tokens, int nt,
                     uint32_t ch0, int nc, float *out);

/* ---------------- a4: discounted reward [P2, reward equation] ---------------- */

/* r[i][t] = sum_{s >= t, s in seq(t)} gamma^(s-t) c[i][s], by the backward
 * recurrence r_t = c_t + gamma r_{t+1} inside each sequence. */
int orc_reward_scan(const float *c, double *r, int K, int T,
                    const int32_t *seq_offsets, int n_seq, double gamma);

/* Same quantity as an explicit double sum with gamma^(s-t) by repeated
 * multiplication (0^0 = 1).  O(L^2) per sequence: brute force for pins. */
int orc_reward_scan_brute(const float *c, double *r, int K, int T,
                          const int32_t *seq_offsets, int n_seq, double gamma);

/* ---------------- a5: output-side error estimate [P2, g_t equation] ---------------- */

/* g[n][m] = -(1/(K_total sigma)) sum_{k<K} r[k][toks[n]] a(draw_begin+k, token_begin+toks[n], chans[m])
 * where r is c_or_r itself (is_r != 0) or the reward of c_or_r (is_r == 0).
 * c_or_r is [K][T]; chans == NULL means all d_out channels (n_chans = d_out).
 * token_begin is the global index of column 0 (a part of a batch split by
 * sequences draws the noise of its tokens' places in the whole batch). */
int orc_layer_estimate(const float *c_or_r, int is_r, int K, int T, int d_out,
                       const int32_t *seq_offsets, int n_seq, double gamma,
                       uint32_t seed, uint32_t layer, uint32_t draw_begin, uint32_t token_begin,
                       int K_total, double sigma,
                       const int32_t *toks, int n_toks,
                       const int32_t *chans, int n_chans, double *g);

/* ---------------- a6: weight estimate [P2, G_W equation] ---------------- */

/* G[n][i] = sum_t g[t][rows[n]] X[t][i]; g is [T][d_out], X is [T][d_in]. */
int orc_weight_grad(const float *g, const float *X, int T, int d_in, int d_out,
                    const int32_t *rows, int n_rows, double *G);

/* ---------------- a2/a3: LM head [P2, interference suppression, 3rd] ---------------- */

/* Z[n][v] = sum_k X[toks[n]][k] W[v][k]  (clean logits, no bias). */
int orc_logits(const float *X, const float *W, int T, int d_in, int V,
               const int32_t *toks, int n, double *Z);

/* Clean per-token loss: lse = log sum_v exp z_v, ell = lse - z_y. */
int orc_head_clean(const float *Zrows, const int32_t *y, int n, int V,
                   double *lse, double *ell);

/* Head step for n tokens (rows of Z, targets y, global token ids toks):
 * for each chunk [ch*Vc, (ch+1)*Vc) and draw k, perturbed logits
 * z + sigma a 1[v in chunk] give the loss l~, c = l~ - l (direct definition),
 * and g[n][v] = -(1/(K_total sigma)) sum_k c_chunk(v)[k][n] a(k, tok, v).
 * c (nullable) is [V/Vc][nd][n]; g is [n][V]. */
int orc_head_step(const float *Zrows, const int32_t *y, const int32_t *toks,
                  int n, int V, int Vc, uint32_t seed, uint32_t layer,
                  uint32_t draw_begin, int nd, int K_total, double sigma,
                  double *c, double *g);

/* Backprop gradient of the head's summed cross entropy, rows of [V][d_in]:
 * G[n][i] = sum_t (softmax(z_t)[rows[n]] - [rows[n] == y_t]) X[t][i]. */
int orc_head_bp_grad(const float *Z, const int32_t *y, const float *X, int T, int d_in, int V,
                     const int32_t *rows, int n_rows, double *G);

/* Cosine similarity in double. */
double orc_cosine(const float *a, const float *b, long long n);

/* ---------------- synthetic costs (estimator-only workloads) ---------------- */

/* c = sigma <u_s, a_s^(i)> + eps_scale * eps(i, s),
 * eps(i, s) = gauss(seed, layer, i, s, 0, stream 1).  u is [T][d_out]. */
int orc_synth_costs(const float *u, int T, int d_out, uint32_t seed,
                    uint32_t layer, double sigma, double eps_scale,
                    const int32_t *draws, const int32_t *toks, int n_pairs,
                    double *c);

/* ---------------- toy causal suffix (hidden-layer scoring) ---------------- */

/* Per-token cross-entropy after the perturbed layer output
 *   y~ = Y + sigma a(draw),  Y = X W^T  (W is [d][d_in]),
 *   h  = y~ + Attn(y~) Wo^T,  Attn = one causal softmax head per sequence
 *        (q,k,v = y~ Wq^T, y~ Wk^T, y~ Wv^T; scores / sqrt(dh)),
 *   z  = h Wout^T,  loss = logsumexp(z) - z_target.
 * loss is [nd][T]; with_noise == 0 gives the clean losses (nd rows all equal). */
int orc_toy_suffix_losses(const float *X, const float *W, int T, int d_in, int d,
                          const int32_t *seq_offsets, int n_seq,
                          const float *Wq, const float *Wk, const float *Wv,
                          const float *Wo, int dh, const float *Wout, int V,
                          const int32_t *targets, uint32_t seed, uint32_t layer,
                          double sigma, int with_noise,
                          const int32_t *draws, int nd, double *loss);

/* ---------------- attention-internal scoring ---------------- */

/* c[n][t] = -< z~_t - z_t, G_t > where z = Attn(Y Wq^T, Y Wk^T, Y Wv^T) Wo^T and
 * z~ has sigma a(draws[n]) added to projection `which` (0 = q, 1 = k, 2 = v;
 * channel = projection channel).  Y, G: [T][d]; Wq, Wk, Wv: [dh][d]; Wo: [d][dh]. */
int orc_attention_internal_costs(const float *Y, int T, int d, const int32_t *offs, int n_seq,
                                 const float *Wq, const float *Wk, const float *Wv, const float *Wo,
                                 const float *Wg, const float *E,
                                 int dh, int which, const float *G, uint32_t seed, uint32_t layer,
                                 double sigma, const int32_t *draws, int nd, double *c);

#ifdef __cplusplus
}
#endif
#endif
