/*
 * estimator.c -- oracle for the hidden-layer estimator: reward scan (a4),
 * output-side error estimate (a5), weight estimate (a6), synthetic costs.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Plain nested loops in double.
 *
 * Definitions ([P2] section "信用分配：一次前向，两种奖励"):
 *   c_s     = l~_s - l_s                      centred per-token loss change
 *   r_t     = sum_{s >= t} gamma^(s-t) c_s    discounted reward (reward eq.)
 *   g_t     = -(1/(K sigma)) sum_i r_t^(i) a_t^(i)          (error-estimate eq.)
 *   G_W     = sum_t g_t x_t^T                               (weight-estimate eq.)
 * Readings taken where the page is silent:
 *   - s ranges over the same sequence as t only (causal attention does not
 *     cross sequences); sequences are given by seq_offsets[0..n_seq], with
 *     seq_offsets[0] = 0 and seq_offsets[n_seq] = T.
 *   - gamma = 0 gives r = c (0^0 = 1).
 *   - When the draws are split, the scale uses the whole population K_total.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#include "oracle.h"

static int check_offsets(const int32_t *off, int n_seq, int T)
{
    if (n_seq < 1 || off[0] != 0 || off[n_seq] != T) return -1;
    for (int q = 0; q < n_seq; ++q)
        if (off[q + 1] < off[q]) return -1;
    return 0;
}

int orc_reward_scan(const float *c, double *r, int K, int T,
                    const int32_t *seq_offsets, int n_seq, double gamma)
{
    if (check_offsets(seq_offsets, n_seq, T)) return -1;
    for (int i = 0; i < K; ++i) {
        const float *ci = c + (size_t)i * T;
        double *ri = r + (size_t)i * T;
        for (int q = 0; q < n_seq; ++q) {
            double acc = 0.0;
            for (int t = seq_offsets[q + 1] - 1; t >= seq_offsets[q]; --t) {
                acc = (double)ci[t] + gamma * acc;
                ri[t] = acc;
            }
        }
    }
    return 0;
}

int orc_reward_scan_brute(const float *c, double *r, int K, int T,
                          const int32_t *seq_offsets, int n_seq, double gamma)
{
    if (check_offsets(seq_offsets, n_seq, T)) return -1;
    for (int i = 0; i < K; ++i) {
        for (int q = 0; q < n_seq; ++q) {
            for (int t = seq_offsets[q]; t < seq_offsets[q + 1]; ++t) {
                double sum = 0.0;
                for (int s = t; s < seq_offsets[q + 1]; ++s) {
                    double w = 1.0;                 /* gamma^(s-t), 0^0 = 1 */
                    for (int e = 0; e < s - t; ++e) w *= gamma;
                    sum += w * (double)c[(size_t)i * T + s];
                }
                r[(size_t)i * T + t] = sum;
            }
        }
    }
    return 0;
}

static int seq_of(const int32_t *off, int n_seq, int t)
{
    for (int q = 0; q < n_seq; ++q)
        if (t >= off[q] && t < off[q + 1]) return q;
    return -1;
}

int orc_layer_estimate(const float *c_or_r, int is_r, int K, int T, int d_out,
                       const int32_t *seq_offsets, int n_seq, double gamma,
                       uint32_t seed, uint32_t layer, uint32_t draw_begin, uint32_t token_begin,
                       int K_total, double sigma,
                       const int32_t *toks, int n_toks,
                       const int32_t *chans, int n_chans, double *g)
{
    if (check_offsets(seq_offsets, n_seq, T)) return -1;
    if (chans == NULL) n_chans = d_out;
    const double scale = -1.0 / ((double)K_total * sigma);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (int n = 0; n < n_toks; ++n) {
        const int t = toks[n];
        const int q = seq_of(seq_offsets, n_seq, t);
        if (q < 0) { err = -1; continue; }
        double *gn = g + (size_t)n * n_chans;
        for (int m = 0; m < n_chans; ++m) gn[m] = 0.0;
        for (int k = 0; k < K; ++k) {
            const float *row = c_or_r + (size_t)k * T;
            double r;
            if (is_r) {
                r = (double)row[t];
            } else {
                /* reward of token t: backward recurrence from the end of its sequence */
                double acc = 0.0;
                for (int s = seq_offsets[q + 1] - 1; s >= t; --s) acc = (double)row[s] + gamma * acc;
                r = acc;
            }
            for (int m = 0; m < n_chans; ++m) {
                const uint32_t j = (uint32_t)(chans ? chans[m] : m);
                const float a = orc_gauss(seed, layer, draw_begin + (uint32_t)k, token_begin + (uint32_t)t, j, 0);
                gn[m] += r * (double)a;
            }
        }
        for (int m = 0; m < n_chans; ++m) gn[m] *= scale;
    }
    return err;
}

int orc_weight_grad(const float *g, const float *X, int T, int d_in, int d_out,
                    const int32_t *rows, int n_rows, double *G)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < n_rows; ++n) {
        const int o = rows[n];
        double *Gn = G + (size_t)n * d_in;
        for (int i = 0; i < d_in; ++i) Gn[i] = 0.0;
        for (int t = 0; t < T; ++t) {
            const double gto = (double)g[(size_t)t * d_out + o];
            const float *xt = X + (size_t)t * d_in;
            for (int i = 0; i < d_in; ++i) Gn[i] += gto * (double)xt[i];
        }
    }
    return 0;
}

int orc_synth_costs(const float *u, int T, int d_out, uint32_t seed,
                    uint32_t layer, double sigma, double eps_scale,
                    const int32_t *draws, const int32_t *toks, int n_pairs,
                    double *c)
{
    (void)T;
#pragma omp parallel for schedule(static)
    for (int p = 0; p < n_pairs; ++p) {
        const uint32_t i = (uint32_t)draws[p], s = (uint32_t)toks[p];
        double dot = 0.0;
        for (int j = 0; j < d_out; ++j)
            dot += (double)u[(size_t)s * d_out + j] * (double)orc_gauss(seed, layer, i, s, (uint32_t)j, 0);
        c[p] = sigma * dot + eps_scale * (double)orc_gauss(seed, layer, i, s, 0, 1);
    }
    return 0;
}
