/*
 * head.c -- oracle for the LM-head path: clean logits (a2), perturbed
 * cross-entropy over one vocabulary chunk (a3) and the head's error estimate.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Plain loops in double.
 *
 * [P2] section "真正的工作量：压住干扰", third measure: the LM head is perturbed
 * directly on the cached logits, and each perturbed pass recomputes only the
 * cross entropy, over one chunk of the vocabulary.  Reading taken here: a head
 * step runs one pass per chunk [ch*Vc, (ch+1)*Vc); in that pass draw i adds
 * sigma a^(i)_v to the logits v of the chunk only, the per-token change of
 * the full-vocabulary cross entropy is c = l~ - l ([P2] "信用分配", c_s), and
 * the error estimate of the chunk's outputs is the g_t equation with that c
 * (gamma = 0 for the head, so r = c).  The noise channel is the global vocab
 * id v, so the noise does not depend on the chunking.  No bias, no softcap.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#include "oracle.h"

int orc_logits(const float *X, const float *W, int T, int d_in, int V,
               const int32_t *toks, int n, double *Z)
{
    (void)T;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < n; ++m) {
        const float *x = X + (size_t)toks[m] * d_in;
        for (int v = 0; v < V; ++v) {
            const float *w = W + (size_t)v * d_in;
            double acc = 0.0;
            for (int k = 0; k < d_in; ++k) acc += (double)x[k] * (double)w[k];
            Z[(size_t)m * V + v] = acc;
        }
    }
    return 0;
}

/* log sum_v exp(z_v) with the maximum factored out */
static double logsumexp(const double *z, int V)
{
    double mx = z[0];
    for (int v = 1; v < V; ++v)
        if (z[v] > mx) mx = z[v];
    double s = 0.0;
    for (int v = 0; v < V; ++v) s += exp(z[v] - mx);
    return mx + log(s);
}

int orc_head_clean(const float *Zrows, const int32_t *y, int n, int V,
                   double *lse, double *ell)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)V);
    if (!z) return -1;
    for (int m = 0; m < n; ++m) {
        for (int v = 0; v < V; ++v) z[v] = (double)Zrows[(size_t)m * V + v];
        lse[m] = logsumexp(z, V);
        ell[m] = lse[m] - z[y[m]];
    }
    free(z);
    return 0;
}

int orc_head_step(const float *Zrows, const int32_t *y, const int32_t *toks,
                  int n, int V, int Vc, uint32_t seed, uint32_t layer,
                  uint32_t draw_begin, int nd, int K_total, double sigma,
                  double *c, double *g)
{
    if (Vc <= 0 || V % Vc != 0) return -1;
    const int n_chunks = V / Vc;
    const double scale = -1.0 / ((double)K_total * sigma);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (int m = 0; m < n; ++m) {
        double *zt = (double *)malloc(sizeof(double) * (size_t)V);
        double *a = (double *)malloc(sizeof(double) * (size_t)Vc);
        if (!zt || !a) { err = -1; free(zt); free(a); continue; }
        const float *zrow = Zrows + (size_t)m * V;
        const uint32_t tok = (uint32_t)toks[m];
        /* clean loss l_t */
        for (int v = 0; v < V; ++v) zt[v] = (double)zrow[v];
        const double ell = logsumexp(zt, V) - zt[y[m]];
        double *gm = g + (size_t)m * V;
        for (int v = 0; v < V; ++v) gm[v] = 0.0;
        for (int ch = 0; ch < n_chunks; ++ch) {
            const int v0 = ch * Vc;
            for (int k = 0; k < nd; ++k) {
                const uint32_t draw = draw_begin + (uint32_t)k;
                /* perturbed logits: noise on the chunk only */
                for (int v = 0; v < V; ++v) zt[v] = (double)zrow[v];
                for (int j = 0; j < Vc; ++j) {
                    a[j] = (double)orc_gauss(seed, layer, draw, tok, (uint32_t)(v0 + j), 0);
                    zt[v0 + j] += sigma * a[j];
                }
                const double ell_pert = logsumexp(zt, V) - zt[y[m]];
                const double cc = ell_pert - ell;
                if (c) c[((size_t)ch * nd + k) * n + m] = cc;
                for (int j = 0; j < Vc; ++j) gm[v0 + j] += cc * a[j];
            }
        }
        for (int v = 0; v < V; ++v) gm[v] *= scale;
        free(zt);
        free(a);
    }
    return err;
}

/* Backprop gradient of sum_t l_t with respect to W for the listed output rows:
 * G[n][i] = sum_t (softmax(z_t)[rows[n]] - [rows[n] == y_t]) X[t][i]. */
int orc_head_bp_grad(const float *Z, const int32_t *y, const float *X, int T, int d_in, int V,
                     const int32_t *rows, int n_rows, double *G)
{
    double *lse = (double *)malloc(sizeof(double) * (size_t)T);
    double *zt = (double *)malloc(sizeof(double) * (size_t)V);
    if (!lse || !zt) { free(lse); free(zt); return -1; }
    for (int t = 0; t < T; ++t) {
        for (int v = 0; v < V; ++v) zt[v] = (double)Z[(size_t)t * V + v];
        lse[t] = logsumexp(zt, V);
    }
    free(zt);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < n_rows; ++n) {
        const int v = rows[n];
        double *Gn = G + (size_t)n * d_in;
        for (int i = 0; i < d_in; ++i) Gn[i] = 0.0;
        for (int t = 0; t < T; ++t) {
            const double d = exp((double)Z[(size_t)t * V + v] - lse[t]) - (y[t] == v ? 1.0 : 0.0);
            for (int i = 0; i < d_in; ++i) Gn[i] += d * (double)X[(size_t)t * d_in + i];
        }
    }
    free(lse);
    return 0;
}

/* Cosine similarity of two vectors, accumulated in double. */
double orc_cosine(const float *a, const float *b, long long n)
{
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (long long i = 0; i < n; ++i) {
        ab += (double)a[i] * (double)b[i];
        aa += (double)a[i] * (double)a[i];
        bb += (double)b[i] * (double)b[i];
    }
    return ab / (sqrt(aa) * sqrt(bb));
}
