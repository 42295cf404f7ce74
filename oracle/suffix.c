/*
 * suffix.c -- oracle for the toy causal suffix that scores a perturbed hidden
 * linear layer (the per-token losses l~ and l behind c_s).
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Plain loops in double.
 *
 * [P2] section "真正的工作量：压住干扰", first measure: perturbed draws of a
 * block rerun the network from that block onward on the cached clean forward.
 * The pages do not give the model; this build's reading is the smallest suffix
 * that lets the noise on one token reach later tokens (which is what the
 * discount gamma of the reward equation is for): the perturbed layer output
 * feeds a residual stream with one causal softmax attention head, then a
 * linear readout to the vocabulary and the per-token cross entropy.
 *   y~ = X W^T + sigma a          (a from the noise spec, stream 0)
 *   q, k, v = y~ Wq^T, y~ Wk^T, y~ Wv^T          (head width dh)
 *   o_t = sum_{u <= t, u in seq(t)} softmax_u(q_t.k_u / sqrt(dh)) v_u
 *   h_t = y~_t + Wo o_t,   z_t = Wout h_t,   loss_t = logsumexp(z_t) - z_t[target]
 * No norm, no bias, no positional encoding.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#include "oracle.h"

int orc_toy_suffix_losses(const float *X, const float *W, int T, int d_in, int d,
                          const int32_t *seq_offsets, int n_seq,
                          const float *Wq, const float *Wk, const float *Wv,
                          const float *Wo, int dh, const float *Wout, int V,
                          const int32_t *targets, uint32_t seed, uint32_t layer,
                          double sigma, int with_noise,
                          const int32_t *draws, int nd, double *loss)
{
    if (n_seq < 1 || seq_offsets[0] != 0 || seq_offsets[n_seq] != T) return -1;
    double *Y = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *yt = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *q = (double *)malloc(sizeof(double) * (size_t)T * dh);
    double *k = (double *)malloc(sizeof(double) * (size_t)T * dh);
    double *v = (double *)malloc(sizeof(double) * (size_t)T * dh);
    if (!Y || !yt || !q || !k || !v) { free(Y); free(yt); free(q); free(k); free(v); return -1; }
    const double inv_sqrt_dh = 1.0 / sqrt((double)dh);

    /* clean layer output Y = X W^T */
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < d_in; ++i) acc += (double)X[(size_t)t * d_in + i] * (double)W[(size_t)j * d_in + i];
            Y[(size_t)t * d + j] = acc;
        }

    int err = 0;
    for (int n = 0; n < nd; ++n) {
        const uint32_t draw = (uint32_t)draws[n];
        /* perturbed layer output */
#pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < d; ++j) {
                double a = with_noise ? (double)orc_gauss(seed, layer, draw, (uint32_t)t, (uint32_t)j, 0) : 0.0;
                yt[(size_t)t * d + j] = Y[(size_t)t * d + j] + sigma * a;
            }
        /* q, k, v projections */
#pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t)
            for (int e = 0; e < dh; ++e) {
                double aq = 0.0, ak = 0.0, av = 0.0;
                for (int j = 0; j < d; ++j) {
                    const double y = yt[(size_t)t * d + j];
                    aq += y * (double)Wq[(size_t)e * d + j];
                    ak += y * (double)Wk[(size_t)e * d + j];
                    av += y * (double)Wv[(size_t)e * d + j];
                }
                q[(size_t)t * dh + e] = aq;
                k[(size_t)t * dh + e] = ak;
                v[(size_t)t * dh + e] = av;
            }
        /* attention, residual, readout, cross entropy -- token by token */
#pragma omp parallel for schedule(dynamic)
        for (int t = 0; t < T; ++t) {
            int sq = 0;
            while (!(t >= seq_offsets[sq] && t < seq_offsets[sq + 1])) ++sq;
            const int s0 = seq_offsets[sq];
            double *p = (double *)malloc(sizeof(double) * (size_t)(t - s0 + 1));
            double *o = (double *)malloc(sizeof(double) * (size_t)dh);
            double *h = (double *)malloc(sizeof(double) * (size_t)d);
            double *z = (double *)malloc(sizeof(double) * (size_t)V);
            if (!p || !o || !h || !z) { err = -1; free(p); free(o); free(h); free(z); continue; }
            double mx = -INFINITY;
            for (int u = s0; u <= t; ++u) {
                double sc = 0.0;
                for (int e = 0; e < dh; ++e) sc += q[(size_t)t * dh + e] * k[(size_t)u * dh + e];
                sc *= inv_sqrt_dh;
                p[u - s0] = sc;
                if (sc > mx) mx = sc;
            }
            double den = 0.0;
            for (int u = s0; u <= t; ++u) { p[u - s0] = exp(p[u - s0] - mx); den += p[u - s0]; }
            for (int e = 0; e < dh; ++e) {
                double acc = 0.0;
                for (int u = s0; u <= t; ++u) acc += p[u - s0] * v[(size_t)u * dh + e];
                o[e] = acc / den;
            }
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int e = 0; e < dh; ++e) acc += (double)Wo[(size_t)j * dh + e] * o[e];
                h[j] = yt[(size_t)t * d + j] + acc;
            }
            double zmax = -INFINITY;
            for (int c = 0; c < V; ++c) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += (double)Wout[(size_t)c * d + j] * h[j];
                z[c] = acc;
                if (acc > zmax) zmax = acc;
            }
            double se = 0.0;
            for (int c = 0; c < V; ++c) se += exp(z[c] - zmax);
            loss[(size_t)n * T + t] = zmax + log(se) - z[targets[t]];
            free(p); free(o); free(h); free(z);
        }
    }
    free(Y); free(yt); free(q); free(k); free(v);
    return err;
}
