/*
 * noise.c -- the oracle's implementation of the noise specification.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * The pages fix only the distribution of the activation noise: a_t ~ N(0, I),
 * drawn independently per token and per draw, scaled by sigma and added to the
 * layer output ([P2] section "信用分配", first paragraph).  Everything below is
 * this build's reading, chosen so that the CUDA kernels can regenerate any
 * element from its coordinates and so that this plain C code reproduces the
 * same binary32 value bit for bit:
 *
 *   1. Philox4x32-10 [PHILOX], key (seed, layer), counter
 *      (channel >> 2, token, draw, stream) -> words (x0, x1, x2, x3).
 *   2. Channel j takes the Box-Muller pair (x0,x1) if (j>>1)&1 == 0 else
 *      (x2,x3); even j takes the cosine branch, odd j the sine branch.
 *   3. Radius uniform u = 2 - float(0x3F800000 | a>>9), exact, in [2^-23, 1].
 *      rho = sqrt(-2 ln u) with ln from an atanh series (orc_ln).
 *   4. Angle: octant o = b>>29, fraction f = float(0x3F800000 | (b>>6 & 0x7FFFFF)) - 1,
 *      theta = (pi/4)(o + f).  The octant is folded to phi in [0, pi/4]
 *      (phi = f pi/4 in even octants, (1-f) pi/4 in odd ones), sin/cos of phi
 *      come from Taylor series (orc_sincos_quarter), then are swapped and
 *      signed by octant.
 *
 * Every operation is a correctly rounded binary32 operation (+ - * / sqrt fma);
 * this file must be compiled with -ffp-contract=off so that nothing is fused
 * behind the spec's back.  Coefficients are the exact series values 1/(2k+1)
 * and (-1)^k/n! rounded to nearest binary32; ln 2 is split Cody-Waite style
 * (high part with 15 significant bits, so e*LN2_HI is exact for |e| <= 23).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "oracle.h"

static float from_bits(uint32_t b) { float f; memcpy(&f, &b, sizeof f); return f; }
static uint32_t to_bits(float f) { uint32_t b; memcpy(&b, &f, sizeof b); return b; }

/* Philox constants [PHILOX]: round multipliers and Weyl key increments. */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {            /* key schedule: bump before rounds 2..10 */
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* atanh-series coefficients 1/(2k+1), k = 1..5, rounded to binary32. */
static const float LN_C3  = 0x1.555556p-2f;
static const float LN_C5  = 0x1.99999ap-3f;
static const float LN_C7  = 0x1.24924ap-3f;
static const float LN_C9  = 0x1.c71c72p-4f;
static const float LN_C11 = 0x1.745d18p-4f;
/* ln 2 = LN2_HI + LN2_LO; LN2_HI keeps 15 significant bits, so e * LN2_HI is
 * exact for |e| < 2^9 (here |e| <= 23). */
static const float LN2_HI = 0x1.62e4p-1f;
static const float LN2_LO = 0x1.7f7d1cp-20f;

float orc_ln(float u)
{
    /* u = m * 2^e with m in [sqrt(1/2), sqrt(2)): subtract the bit pattern of
     * sqrt(1/2) so that the exponent field of the difference is e. */
    uint32_t b = to_bits(u);
    int32_t i = (int32_t)(b - 0x3F3504F3u);
    int32_t e = i >> 23;                      /* arithmetic shift (gcc) */
    float m = from_bits(b - ((uint32_t)e << 23));
    /* ln m = 2 atanh(s), s = (m-1)/(m+1), |s| <= 0.1716 */
    float s = (m - 1.0f) / (m + 1.0f);
    float z = s * s;
    float p = LN_C11;
    p = fmaf(p, z, LN_C9);
    p = fmaf(p, z, LN_C7);
    p = fmaf(p, z, LN_C5);
    p = fmaf(p, z, LN_C3);
    p = fmaf(p, z, 1.0f);
    float lnm = (s + s) * p;
    float fe = (float)e;
    return fmaf(fe, LN2_HI, fmaf(fe, LN2_LO, lnm));
}

/* Taylor coefficients (-1)^k/(2k+1)! for sin and (-1)^k/(2k)! for cos. */
static const float SIN_3  = -0x1.555556p-3f;
static const float SIN_5  =  0x1.111112p-7f;
static const float SIN_7  = -0x1.a01a02p-13f;
static const float SIN_9  =  0x1.71de3ap-19f;
static const float SIN_11 = -0x1.ae6456p-26f;
static const float COS_2  = -0x1p-1f;
static const float COS_4  =  0x1.555556p-5f;
static const float COS_6  = -0x1.6c16c2p-10f;
static const float COS_8  =  0x1.a01a02p-16f;
static const float COS_10 = -0x1.27e4fcp-22f;
static const float PI_4   =  0x1.921fb6p-1f;

void orc_sincos_quarter(float phi, float *s, float *c)
{
    float z = phi * phi;
    float ps = SIN_11;
    ps = fmaf(ps, z, SIN_9);
    ps = fmaf(ps, z, SIN_7);
    ps = fmaf(ps, z, SIN_5);
    ps = fmaf(ps, z, SIN_3);
    *s = fmaf(phi * z, ps, phi);
    float pc = COS_10;
    pc = fmaf(pc, z, COS_8);
    pc = fmaf(pc, z, COS_6);
    pc = fmaf(pc, z, COS_4);
    pc = fmaf(pc, z, COS_2);
    *c = fmaf(z, pc, 1.0f);
}

void orc_box_muller(uint32_t a, uint32_t b, float *n_even, float *n_odd)
{
    /* radius */
    float u = 2.0f - from_bits(0x3F800000u | (a >> 9));
    float rho = sqrtf(-2.0f * orc_ln(u));
    /* angle theta = 2 pi w, w = (o + f) / 8 */
    uint32_t o = b >> 29;
    float f = from_bits(0x3F800000u | ((b >> 6) & 0x007FFFFFu)) - 1.0f;
    float g = (o & 1u) ? (1.0f - f) : f;
    float phi = g * PI_4;
    float sp, cp;
    orc_sincos_quarter(phi, &sp, &cp);
    /* octant o: theta = o*pi/4 + f*pi/4.  Odd octants were reflected
     * (phi measured back from the next multiple of pi/4); octants whose
     * nearest multiple of pi/2 is odd swap sine and cosine. */
    uint32_t swap = ((o + 1u) >> 1) & 1u;
    float S = swap ? cp : sp;
    float C = swap ? sp : cp;
    uint32_t neg_s = o >> 2;                 /* theta in [pi, 2pi) */
    uint32_t neg_c = ((o + 2u) >> 2) & 1u;   /* theta in [pi/2, 3pi/2) */
    float sin_t = from_bits(to_bits(S) ^ (neg_s << 31));
    float cos_t = from_bits(to_bits(C) ^ (neg_c << 31));
    *n_even = rho * cos_t;
    *n_odd = rho * sin_t;
}

float orc_gauss(uint32_t seed, uint32_t layer, uint32_t draw, uint32_t token,
                uint32_t channel, uint32_t stream)
{
    const uint32_t ctr[4] = {channel >> 2, token, draw, stream};
    const uint32_t key[2] = {seed, layer};
    uint32_t x[4];
    orc_philox4x32_10(ctr, key, x);
    uint32_t pair = (channel >> 1) & 1u;
    float ne, no;
    orc_box_muller(x[2 * pair], x[2 * pair + 1], &ne, &no);
    return (channel & 1u) ? no : ne;
}

void orc_noise_block(uint32_t seed, uint32_t layer, uint32_t stream,
                     uint32_t draw0, int nd, const int32_t *tokens, int nt,
                     uint32_t ch0, int nc, float *out)
{
    for (int d = 0; d < nd; ++d)
        for (int t = 0; t < nt; ++t)
            for (int c = 0; c < nc; ++c)
                out[((size_t)d * nt + t) * nc + c] =
                    orc_gauss(seed, layer, draw0 + (uint32_t)d, (uint32_t)tokens[t],
                              ch0 + (uint32_t)c, stream);
}

/* ---- batch forms, for exhaustive checks of the specification ---- */

void orc_philox_batch(const uint32_t *ctr, const uint32_t *key, int n, uint32_t *out)
{
    for (int p = 0; p < n; ++p) orc_philox4x32_10(ctr + 4 * p, key + 2 * p, out + 4 * p);
}

void orc_ln_batch(const float *u, int n, float *out)
{
    for (int p = 0; p < n; ++p) out[p] = orc_ln(u[p]);
}

void orc_sincos_batch(const float *phi, int n, float *s, float *c)
{
    for (int p = 0; p < n; ++p) orc_sincos_quarter(phi[p], s + p, c + p);
}

void orc_box_muller_batch(const uint32_t *a, const uint32_t *b, int n, float *ne, float *no)
{
    for (int p = 0; p < n; ++p) orc_box_muller(a[p], b[p], ne + p, no + p);
}
