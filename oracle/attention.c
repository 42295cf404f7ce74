/*
 * attention.c -- oracle for attention-internal scoring.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Plain loops in double.
 *
 * [P2] section "真正的工作量：压住干扰", second measure: the attention's
 * internals (query, key, value, gate, value embedding) are perturbed
 * separately, and because the per-token loss barely sees those perturbations
 * their draws are scored through the attention output: the change the
 * perturbation makes to the attention output, Delta o_s, against that
 * output's estimated error g_s.  Reading taken here (consistent with
 * c_s = l~_s - l_s and g ~ -dl/dz):
 *   z = Attn(q, k, v) Wo^T          (attention output, [T][d])
 *   z~ = the same with sigma a(draw) added to one internal quantity (noise
 *        channel = its channel, dh wide)
 *   c_s = -< z~_s - z_s, g_s >      (first order: l~_s - l_s)
 * q, k = Y Wq^T, Y Wk^T; causal softmax attention inside each sequence with
 * scores scaled by 1/sqrt(dh).  The values carry the token's value embedding
 * e_t (E [T][dh], optional) through a gate (optional; the credit-assignment
 * section's remark that gates and value embeddings need gamma near 1, since
 * later tokens read them, places both on the values):
 *   v_t = Y_t Wv^T + s(Y_t Wg^T) * e_t     (s = logistic sigmoid, per channel;
 *                                           s = 1 without a gate; no e: Y Wv^T)
 * The perturbed quantity: 0 q, 1 k, 2 v, 3 the gate's pre-activation
 * Y Wg^T, 4 the value embedding e.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* o[t] = sum_{u <= t, u in seq(t)} softmax_u(q_t . k_u / sqrt(dh)) v_u */
static void causal_attention(const double *q, const double *k, const double *v, int T, int dh,
                             const int32_t *offs, int n_seq, double *o)
{
    (void)T;
    const double scale = 1.0 / sqrt((double)dh);
    for (int sq = 0; sq < n_seq; ++sq) {
        const int s0 = offs[sq], s1 = offs[sq + 1];
        for (int t = s0; t < s1; ++t) {
            double mx = -INFINITY;
            for (int u = s0; u <= t; ++u) {
                double sc = 0.0;
                for (int e = 0; e < dh; ++e) sc += q[(size_t)t * dh + e] * k[(size_t)u * dh + e];
                sc *= scale;
                if (sc > mx) mx = sc;
            }
            double den = 0.0;
            double *ot = o + (size_t)t * dh;
            for (int e = 0; e < dh; ++e) ot[e] = 0.0;
            for (int u = s0; u <= t; ++u) {
                double sc = 0.0;
                for (int e = 0; e < dh; ++e) sc += q[(size_t)t * dh + e] * k[(size_t)u * dh + e];
                const double p = exp(sc * scale - mx);
                den += p;
                for (int e = 0; e < dh; ++e) ot[e] += p * v[(size_t)u * dh + e];
            }
            for (int e = 0; e < dh; ++e) ot[e] /= den;
        }
    }
}

static void project(const float *Y, const float *Wp, int T, int d, int dh, double *out)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < dh; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += (double)Y[(size_t)t * d + j] * (double)Wp[(size_t)e * d + j];
            out[(size_t)t * dh + e] = acc;
        }
}

static void output(const double *o, const float *Wo, int T, int d, int dh, double *z)
{
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int e = 0; e < dh; ++e) acc += o[(size_t)t * dh + e] * (double)Wo[(size_t)j * dh + e];
            z[(size_t)t * d + j] = acc;
        }
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

int orc_attention_internal_costs(const float *Y, int T, int d, const int32_t *offs, int n_seq,
                                 const float *Wq, const float *Wk, const float *Wv, const float *Wo,
                                 const float *Wg, const float *E,
                                 int dh, int which, const float *G, uint32_t seed, uint32_t layer,
                                 double sigma, const int32_t *draws, int nd, double *c)
{
    if (which < 0 || which > 4 || n_seq < 1 || offs[0] != 0 || offs[n_seq] != T) return -1;
    if ((which == 3 && (Wg == NULL || E == NULL)) || (which == 4 && E == NULL)) return -1;
    const size_t P = (size_t)T * dh;
    double *q = malloc(sizeof(double) * P), *k = malloc(sizeof(double) * P), *v = malloc(sizeof(double) * P);
    double *o = malloc(sizeof(double) * P), *z = malloc(sizeof(double) * (size_t)T * d);
    double *gp = malloc(sizeof(double) * P);   /* gate pre-activation (0 when no gate: s = 1 is used) */
    if (!q || !k || !v || !o || !z || !gp) { free(q); free(k); free(v); free(o); free(z); free(gp); return -1; }
    project(Y, Wq, T, d, dh, q);
    project(Y, Wk, T, d, dh, k);
    project(Y, Wv, T, d, dh, v);
    if (Wg) project(Y, Wg, T, d, dh, gp);
    if (E)
        for (size_t i = 0; i < P; ++i) v[i] += (Wg ? sigmoid(gp[i]) : 1.0) * (double)E[i];
    causal_attention(q, k, v, T, dh, offs, n_seq, o);
    output(o, Wo, T, d, dh, z);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (int n = 0; n < nd; ++n) {
        double *pp = malloc(sizeof(double) * P), *op = malloc(sizeof(double) * P);
        double *zp = malloc(sizeof(double) * (size_t)T * d);
        if (!pp || !op || !zp) { err = -1; free(pp); free(op); free(zp); continue; }
        const double *base = which == 0 ? q : (which == 1 ? k : v);
        for (int t = 0; t < T; ++t)
            for (int e = 0; e < dh; ++e) {
                const size_t i = (size_t)t * dh + e;
                const double a = (double)orc_gauss(seed, layer, (uint32_t)draws[n], (uint32_t)t, (uint32_t)e, 0);
                if (which <= 2) {
                    pp[i] = base[i] + sigma * a;
                } else if (which == 3) {   /* gate pre-activation perturbed: the value's gated term changes */
                    pp[i] = v[i] + (sigmoid(gp[i] + sigma * a) - sigmoid(gp[i])) * (double)E[i];
                } else {                   /* value embedding perturbed */
                    pp[i] = v[i] + (Wg ? sigmoid(gp[i]) : 1.0) * sigma * a;
                }
            }
        const int on_v = which >= 2;
        causal_attention(which == 0 ? pp : q, which == 1 ? pp : k, on_v ? pp : v, T, dh, offs, n_seq, op);
        output(op, Wo, T, d, dh, zp);
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += (zp[(size_t)t * d + j] - z[(size_t)t * d + j]) * (double)G[(size_t)t * d + j];
            c[(size_t)n * T + t] = -acc;
        }
        free(pp); free(op); free(zp);
    }
    free(q); free(k); free(v); free(o); free(z); free(gp);
    return err;
}
