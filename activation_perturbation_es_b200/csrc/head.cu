// head.cu -- a2 row statistics and the fused LM-head kernel (a1 + a3 + a5).
//
// cnblogs Dust explainer, section "真正的工作量：压住干扰", third measure: the LM
// head is perturbed directly on the cached logits and each perturbed pass
// recomputes only the cross entropy, over one chunk of the vocabulary.  With
// the credit-assignment section's c = l~ - l and gamma = 0 (r = c):
//   c_t^(i)  = log sum_v exp(z_v + sigma a_v 1[v in chunk]) - z~_y - (lse_t - z_y)
//            = log1p( sum_{v in chunk} p_v expm1(sigma a_v) ) - sigma a_y 1[y in chunk],
//   p = softmax(z_t), an exact identity that needs no running maximum because
//   the perturbation only rescales the chunk's share of the clean partition
//   function; then g_t[v] = -(1/(K sigma)) sum_i c_t^(i) a_t^(i)[v].
//
// Design (B200): one warp owns one (token, chunk).  Its lanes hold the chunk's
// probabilities p, the current draw's noise a and the running g in registers
// (Vc/32 values each); per draw they regenerate the noise (one Philox call per
// 4 vocab ids), form their share of the sum, a 5-step xor-shuffle reduction
// gives c, and each lane folds c a into g.  Nothing per draw touches memory
// (except the optional c output); Z is read once per (token, chunk).  The
// kernel is bound by the SM issue rate, like the hidden-layer reduction.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "noise.cuh"

namespace dust {

namespace {

// One warp per token: online max / sum-exp over the row.
__global__ void __launch_bounds__(256)
row_stats_kernel(const float* __restrict__ Z, const int32_t* __restrict__ targets, int T, int V,
                 float* __restrict__ lse, float* __restrict__ ell) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const float* z = Z + static_cast<size_t>(t) * V;
    float m = -INFINITY, s = 0.0f;
    auto push = [&](float x) {
        if (x > m) { s = s * expf(m - x) + 1.0f; m = x; }
        else s += expf(x - m);
    };
    if ((V & 3) == 0) {
        for (int v = 4 * lane; v < V; v += 128) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(z + v));
            push(x.x); push(x.y); push(x.z); push(x.w);
        }
    } else {
        for (int v = lane; v < V; v += 32) push(__ldg(z + v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const float mn = fmaxf(m, m2);
        s = (m == -INFINITY ? 0.0f : s * expf(m - mn)) + (m2 == -INFINITY ? 0.0f : s2 * expf(m2 - mn));
        m = mn;
    }
    if (lane == 0) {
        const float l = m + logf(s);
        lse[t] = l;
        if (ell) ell[t] = l - z[clamp_int(targets[t], 0, V - 1)];
    }
}

// expm1(x) by its Taylor series, for the small |x| = |sigma a| of the head's
// perturbations (|a| <= sqrt(46 ln 2) < 5.66 for every a the generator makes):
//   tier 1, sigma <= 0.02  (|x| <= 0.114): to x^5, relative truncation < x^5/720 < 3e-8;
//   tier 2, sigma <= 0.01  (|x| <= 0.057): to x^4, relative truncation < x^4/120 < 9e-8 < 2^-23.
// Larger sigma (tier 0) uses expm1f.
template <int TIER>
__device__ __forceinline__ float expm1_series(float x) {
    float t;
    if (TIER == 1) {
        t = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
        t = fmaf(x, t, 1.0f / 6.0f);
    } else {
        t = fmaf(x, 1.0f / 24.0f, 1.0f / 6.0f);
    }
    t = fmaf(x, t, 0.5f);
    return fmaf(x * x, t, x);
}

constexpr int kHeadWarps = 4;   // tokens per block

template <int QPL, int TIER>   // channel quads per lane: Vc = 128 * QPL; expm1 tier (see expm1_series)
__global__ void __launch_bounds__(32 * kHeadWarps)
head_chunk_kernel(const float* __restrict__ Z, const float* __restrict__ lse,
                  const int32_t* __restrict__ targets, int T, int V, int Vc, uint32_t seed, uint32_t layer,
                  uint32_t draw_begin, int nd, float sigma, float scale, float* __restrict__ c_out,
                  float* __restrict__ g, __nv_bfloat16* __restrict__ g16, int accumulate) {
    // the chunk's softmax probabilities of each warp's token: read every draw,
    // so they live in shared memory and leave the registers to a and g
    __shared__ float4 p_s[kHeadWarps][32 * QPL];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kHeadWarps + warp;
    if (t >= T) return;
    const int chunk = blockIdx.y;
    const int v0 = chunk * Vc;
    const float* zt = Z + static_cast<size_t>(t) * V;
    const float l = __ldg(lse + t);
    float4* p = p_s[warp];
#pragma unroll
    for (int k = 0; k < QPL; ++k) {
        const float4 z = __ldg(reinterpret_cast<const float4*>(zt + v0 + 4 * (lane + 32 * k)));
        p[lane + 32 * k] = make_float4(expf(z.x - l), expf(z.y - l), expf(z.z - l), expf(z.w - l));
    }
    __syncwarp();
    const int rel = clamp_int(__ldg(targets + t), 0, V - 1) - v0;
    const bool in_chunk = rel >= 0 && rel < Vc;
    const int owner = in_chunk ? ((rel >> 2) & 31) : 0;
    const int ky = in_chunk ? (rel >> 7) : -1;
    const int wy = rel & 3;
    const bool i_own = in_chunk && lane == owner;

    float gacc[QPL][4];
#pragma unroll
    for (int k = 0; k < QPL; ++k) gacc[k][0] = gacc[k][1] = gacc[k][2] = gacc[k][3] = 0.0f;
    const uint32_t quad0 = static_cast<uint32_t>(v0 / 4 + lane);

    for (int i = 0; i < nd; ++i) {
        const uint32_t draw = draw_begin + static_cast<uint32_t>(i);
        float a[QPL][4];
        float S = 0.0f, ay = 0.0f;
#pragma unroll
        for (int k = 0; k < QPL; ++k) {
            const float4 n = gauss4(seed, layer, draw, static_cast<uint32_t>(t), quad0 + 32u * k, 0);
            a[k][0] = n.x; a[k][1] = n.y; a[k][2] = n.z; a[k][3] = n.w;
            const float4 pk = p[lane + 32 * k];
            const float pv[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float x = sigma * a[k][w];
                S = fmaf(pv[w], TIER == 0 ? expm1f(x) : expm1_series<TIER>(x), S);
            }
            if (i_own && k == ky) ay = wy == 0 ? n.x : (wy == 1 ? n.y : (wy == 2 ? n.z : n.w));
        }
        S = warp_sum(S);
        ay = __shfl_sync(0xffffffffu, ay, owner);
        const float c = log1pf(S) - (in_chunk ? sigma * ay : 0.0f);
        if (c_out != nullptr && lane == 0) c_out[(static_cast<size_t>(chunk) * nd + i) * T + t] = c;
#pragma unroll
        for (int k = 0; k < QPL; ++k)
#pragma unroll
            for (int w = 0; w < 4; ++w) gacc[k][w] = fmaf(c, a[k][w], gacc[k][w]);
    }

#pragma unroll
    for (int k = 0; k < QPL; ++k) {
        const size_t off = static_cast<size_t>(t) * V + v0 + 4 * (lane + 32 * k);
        float4 out = make_float4(gacc[k][0] * scale, gacc[k][1] * scale, gacc[k][2] * scale, gacc[k][3] * scale);
        float4* gp = reinterpret_cast<float4*>(g + off);
        if (accumulate) {
            const float4 o = *gp;
            out.x += o.x; out.y += o.y; out.z += o.z; out.w += o.w;
        }
        *gp = out;
        if (g16) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(out.x, out.y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(out.z, out.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(g16 + off) = pk;
        }
    }
}

}  // namespace

cudaError_t launch_row_stats(const float* Z, const int32_t* targets, int T, int V, float* lse, float* ell,
                             cudaStream_t stream) {
    row_stats_kernel<<<static_cast<unsigned>(ceil_div(T, 8)), 256, 0, stream>>>(Z, targets, T, V, lse, ell);
    return cudaGetLastError();
}

cudaError_t launch_head_chunks(const float* Z, const float* lse, const int32_t* targets, int T, int V, int Vc,
                               const dust_noise& nz, float* c_out, float* g, void* g_bf16, int accumulate,
                               cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(ceil_div(T, kHeadWarps)), static_cast<unsigned>(V / Vc));
    // |a| < 5.66 for every draw the generator produces (see expm1_series)
    const int tier = nz.sigma <= 0.01f ? 2 : (nz.sigma <= 0.02f ? 1 : 0);
    const float scale = static_cast<float>(-1.0 / (static_cast<double>(nz.K_total) * nz.sigma));
    auto* g16 = static_cast<__nv_bfloat16*>(g_bf16);
    const int nd = static_cast<int>(nz.draw_count);
#define DUST_HEAD_TIER(Q, TIER_)                                                                           \
    head_chunk_kernel<Q, TIER_><<<grid, 32 * kHeadWarps, 0, stream>>>(Z, lse, targets, T, V, Vc, nz.seed,     \
                                                                      nz.layer, nz.draw_begin, nd, nz.sigma,  \
                                                                      scale, c_out, g, g16, accumulate)
#define DUST_HEAD_LAUNCH(Q)                          \
    do {                                             \
        if (tier == 2) DUST_HEAD_TIER(Q, 2);         \
        else if (tier == 1) DUST_HEAD_TIER(Q, 1);    \
        else DUST_HEAD_TIER(Q, 0);                   \
    } while (0)
    if (Vc % 128 != 0) return cudaErrorNotSupported;
    switch (Vc / 128) {
        case 1: DUST_HEAD_LAUNCH(1); break;
        case 2: DUST_HEAD_LAUNCH(2); break;
        case 3: DUST_HEAD_LAUNCH(3); break;
        case 4: DUST_HEAD_LAUNCH(4); break;
        case 5: DUST_HEAD_LAUNCH(5); break;
        case 6: DUST_HEAD_LAUNCH(6); break;
        case 7: DUST_HEAD_LAUNCH(7); break;
        case 8: DUST_HEAD_LAUNCH(8); break;
        default: return cudaErrorNotSupported;
    }
#undef DUST_HEAD_LAUNCH
#undef DUST_HEAD_TIER
    return cudaGetLastError();
}

}  // namespace dust
