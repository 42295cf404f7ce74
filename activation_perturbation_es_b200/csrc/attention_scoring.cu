// attention_scoring.cu -- harness: attention-internal scoring of the draws of
// one of the attention's internal projections (q, k or v).
//
// cnblogs Dust explainer, section "真正的工作量：压住干扰", second measure: the
// per-token loss barely sees perturbations of the attention internals, so
// their draws are scored through the attention output instead, by the change
// a perturbation makes to that output against the output's estimated error.
// With c_s = l~_s - l_s and the error estimate g ~ -dl/dz (literal signs):
//   c_s = -< z~_s - z_s, g_s >,   z = Attn(q, k, v) Wo^T,
// and since z is linear in the attention's value output o,
//   c_s = -< o~_s - o_s, e_s >,   e_s = g_s Wo  (computed once per call).
// The costs then go through the ordinary reward scan, draw reduction and
// weight estimate with d_out = dh.  fp32 CUDA cores, batched over draws.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "noise.cuh"

namespace dust {

namespace {

// out[b][t][e] = P[t][e] + sigma a(first_draw + b, tok0 + t, e)
__global__ void perturb_projection_kernel(const float* __restrict__ P, int T, int dh, uint32_t seed, uint32_t layer,
                                          uint32_t tok0, uint32_t first_draw, int nb, float sigma,
                                          float* __restrict__ out) {
    const int nq = dh / 4;
    const long long total = static_cast<long long>(nb) * T * nq;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int q = static_cast<int>(idx % nq);
        const long long rest = idx / nq;
        const int t = static_cast<int>(rest % T);
        const int b = static_cast<int>(rest / T);
        float4 p = __ldg(reinterpret_cast<const float4*>(P + static_cast<size_t>(t) * dh) + q);
        const float4 a = gauss4(seed, layer, first_draw + static_cast<uint32_t>(b), tok0 + static_cast<uint32_t>(t),
                                static_cast<uint32_t>(q), 0);
        p.x = fmaf(sigma, a.x, p.x);
        p.y = fmaf(sigma, a.y, p.y);
        p.z = fmaf(sigma, a.z, p.z);
        p.w = fmaf(sigma, a.w, p.w);
        reinterpret_cast<float4*>(out + static_cast<size_t>(b * static_cast<long long>(T) + t) * dh)[q] = p;
    }
}

__device__ __forceinline__ float logistic(float x) { return 1.0f / (1.0f + expf(-x)); }

// v[t][e] += s(gp[t][e]) E[t][e] (s = 1 without a gate): the clean values carry
// the token's gated value embedding
__global__ void gated_values_kernel(float* __restrict__ v, const float* __restrict__ gp,
                                    const float* __restrict__ E, long long n) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        v[i] = fmaf(gp ? logistic(__ldg(gp + i)) : 1.0f, __ldg(E + i), v[i]);
}

// The perturbed values of a draw batch when the gate's pre-activation (GATE)
// or the value embedding (else) takes the noise h = sigma a(first_draw + b, tok0 + t, e):
//   gate:  v~ = v + (s(g + h) - s(g)) E, the difference formed without
//          cancellation as (1 - s(g)) s(g + h) (-expm1(-h));
//   value embedding: v~ = v + s(g) h (s = 1 without a gate).
template <bool GATE>
__global__ void perturb_values_kernel(const float* __restrict__ v, const float* __restrict__ gp,
                                      const float* __restrict__ E, int T, int dh, uint32_t seed, uint32_t layer,
                                      uint32_t tok0, uint32_t first_draw, int nb, float sigma,
                                      float* __restrict__ out) {
    const int nq = dh / 4;
    const long long total = static_cast<long long>(nb) * T * nq;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int q = static_cast<int>(idx % nq);
        const long long rest = idx / nq;
        const int t = static_cast<int>(rest % T);
        const int b = static_cast<int>(rest / T);
        const size_t i0 = static_cast<size_t>(t) * dh + 4 * q;
        const float4 a = gauss4(seed, layer, first_draw + static_cast<uint32_t>(b), tok0 + static_cast<uint32_t>(t),
                                static_cast<uint32_t>(q), 0);
        const float av[4] = {a.x, a.y, a.z, a.w};
        float o[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float h = sigma * av[w];
            const float g = gp ? __ldg(gp + i0 + w) : 0.0f;
            float dv;
            if (GATE) dv = (1.0f - logistic(g)) * logistic(g + h) * (-expm1f(-h)) * __ldg(E + i0 + w);
            else dv = (gp ? logistic(g) : 1.0f) * h;
            o[w] = __ldg(v + i0 + w) + dv;
        }
        reinterpret_cast<float4*>(out + static_cast<size_t>(b * static_cast<long long>(T) + t) * dh)[q] =
            make_float4(o[0], o[1], o[2], o[3]);
    }
}

// c[b][t] = -sum_e (o~[b][t][e] - o[t][e]) e_s[t][e]; one warp per (b, t)
__global__ void __launch_bounds__(256)
attention_score_kernel(const float* __restrict__ o_pert, const float* __restrict__ o_clean,
                       const float* __restrict__ err, int nb, int T, int dh, float* __restrict__ c) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.x * 8LL + warp;
    if (row >= static_cast<long long>(nb) * T) return;
    const int t = static_cast<int>(row % T);
    float acc = 0.0f;
    for (int e = lane; e < dh; e += 32)
        acc = fmaf(o_pert[row * dh + e] - o_clean[static_cast<size_t>(t) * dh + e], err[static_cast<size_t>(t) * dh + e],
                   acc);
    acc = warp_sum(acc);
    if (lane == 0) c[row] = -acc;
}

unsigned grid_for(long long n) {
    const long long b = ceil_div(n, 256);
    return static_cast<unsigned>(b < 16 * 1184 ? b : 16 * 1184);
}

struct ScoreLayout {
    size_t q, k, v, gp, o, err, pp, op, part, total;
    int nb;
};

ScoreLayout score_layout(int draw_count, int T, int d, int dh) {
    ScoreLayout L{};
    L.nb = std::min(draw_count, 16);
    size_t off = kStatusBytes;
    auto add = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 256); return o; };
    const size_t P = sizeof(float) * static_cast<size_t>(T) * dh;
    L.q = add(P);
    L.k = add(P);
    L.v = add(P);
    L.gp = add(P);
    L.o = add(P);
    L.err = add(P);
    L.pp = add(P * L.nb);
    L.op = add(P * L.nb);
    size_t part = 0;
    const int shapes[2][3] = {{T, dh, d}, {T, dh, d}};
    for (auto& s : shapes) {
        const int sp = gemm_simt_splits(s[0], s[1], s[2]);
        if (sp > 1) part = std::max(part, sizeof(float) * static_cast<size_t>(sp) * s[0] * s[1]);
    }
    L.part = add(part);
    L.total = off;
    return L;
}

}  // namespace

size_t attention_scoring_workspace_bytes(int draw_count, int T, int d, int dh) {
    return score_layout(draw_count, T, d, dh).total;
}

cudaError_t run_attention_internal_costs(const float* Y, int T, int d, const int32_t* offs, int n_seq,
                                         const float* Wq, const float* Wk, const float* Wv, const float* Wo,
                                         const float* Wg, const float* E, int dh, int which, const float* G,
                                         const dust_noise& nz, float* c, void* ws, cudaStream_t st) {
    const ScoreLayout L = score_layout(static_cast<int>(nz.draw_count), T, d, dh);
    auto* base = static_cast<uint8_t*>(ws);
    float* q = reinterpret_cast<float*>(base + L.q);
    float* k = reinterpret_cast<float*>(base + L.k);
    float* v = reinterpret_cast<float*>(base + L.v);
    float* gp = Wg ? reinterpret_cast<float*>(base + L.gp) : nullptr;
    float* o = reinterpret_cast<float*>(base + L.o);
    float* err = reinterpret_cast<float*>(base + L.err);
    float* pp = reinterpret_cast<float*>(base + L.pp);
    float* op = reinterpret_cast<float*>(base + L.op);
    float* part = reinterpret_cast<float*>(base + L.part);
    cudaError_t e = cudaSuccess;
    // clean projections, clean attention, projected error e = G Wo
    const float* Ws[3] = {Wq, Wk, Wv};
    float* outs[3] = {q, k, v};
    for (int w = 0; w < 3 && e == cudaSuccess; ++w)
        e = launch_gemm_simt(Y, true, d, Ws[w], true, d, DUST_F32, T, dh, d, outs[w], dh, 0, part,
                             gemm_simt_splits(T, dh, d), st);
    if (e == cudaSuccess && gp)      // the gate's pre-activation Y Wg^T
        e = launch_gemm_simt(Y, true, d, Wg, true, d, DUST_F32, T, dh, d, gp, dh, 0, part,
                             gemm_simt_splits(T, dh, d), st);
    if (e == cudaSuccess && E) {
        gated_values_kernel<<<grid_for(static_cast<long long>(T) * dh), 256, 0, st>>>(
            v, gp, E, static_cast<long long>(T) * dh);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = launch_causal_attention(q, k, v, 0, 0, 0, 1, T, dh, offs, n_seq, o, st);
    if (e == cudaSuccess)   // err[t][e] = sum_j G[t][j] Wo[j][e]: B = Wo is [K = d][N = dh]
        e = launch_gemm_simt(G, true, d, Wo, false, dh, DUST_F32, T, dh, d, err, dh, 0, part,
                             gemm_simt_splits(T, dh, d), st);
    const float* P = which == 0 ? q : (which == 1 ? k : v);
    const long long bs = static_cast<long long>(T) * dh;
    const bool on_v = which >= 2;    // v, the gate and the value embedding all act through the values
    for (int b0 = 0; b0 < static_cast<int>(nz.draw_count) && e == cudaSuccess; b0 += L.nb) {
        const int nb = std::min(L.nb, static_cast<int>(nz.draw_count) - b0);
        const unsigned blocks = grid_for(static_cast<long long>(nb) * T * (dh / 4));
        const uint32_t first = nz.draw_begin + static_cast<uint32_t>(b0);
        if (which <= 2)
            perturb_projection_kernel<<<blocks, 256, 0, st>>>(P, T, dh, nz.seed, nz.layer, nz.token_begin, first, nb,
                                                              nz.sigma, pp);
        else if (which == 3)
            perturb_values_kernel<true><<<blocks, 256, 0, st>>>(v, gp, E, T, dh, nz.seed, nz.layer, nz.token_begin,
                                                                first, nb, nz.sigma, pp);
        else
            perturb_values_kernel<false><<<blocks, 256, 0, st>>>(v, gp, E, T, dh, nz.seed, nz.layer, nz.token_begin,
                                                                 first, nb, nz.sigma, pp);
        if ((e = cudaGetLastError()) != cudaSuccess) break;
        e = launch_causal_attention(which == 0 ? pp : q, which == 1 ? pp : k, on_v ? pp : v,
                                    which == 0 ? bs : 0, which == 1 ? bs : 0, on_v ? bs : 0, nb, T, dh, offs,
                                    n_seq, op, st);
        if (e != cudaSuccess) break;
        const long long rows = static_cast<long long>(nb) * T;
        attention_score_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, st>>>(
            op, o, err, nb, T, dh, c + static_cast<size_t>(b0) * T);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace dust
