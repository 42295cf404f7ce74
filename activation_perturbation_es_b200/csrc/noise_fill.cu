// noise_fill.cu -- harness kernels built on the noise generator:
//   * noise_fill: materialise a block of the noise a(seed, layer, draw, token,
//     channel) (for bit-exact checks of the generator; never on the hot path);
//   * synth_costs: synthetic linear costs c = sigma <u_s, a_s> + eps_scale eps
//     that stand in for a perturbed forward in the estimator-only workloads
//     (first order, c_s = l~_s - l_s of the cnblogs Dust explainer's credit
//     assignment section is exactly this with u_s = dl/dy_s).
#include "common.cuh"
#include "kernels.h"
#include "noise.cuh"

namespace dust {

namespace {

__global__ void noise_fill_kernel(uint32_t seed, uint32_t layer, uint32_t stream_id,
                                  uint32_t draw_begin, int nd, uint32_t tok0, int t0, int n_tok, int j0, int n_ch,
                                  float* __restrict__ out) {
    const long long total = static_cast<long long>(nd) * n_tok * n_ch;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(idx % n_ch);
        const long long rest = idx / n_ch;
        const int t = static_cast<int>(rest % n_tok);
        const int k = static_cast<int>(rest / n_tok);
        const uint32_t ch = static_cast<uint32_t>(j0 + j);
        const float4 a = gauss4(seed, layer, draw_begin + k, tok0 + static_cast<uint32_t>(t0 + t), ch >> 2, stream_id);
        const uint32_t w = ch & 3u;
        out[idx] = w == 0 ? a.x : (w == 1 ? a.y : (w == 2 ? a.z : a.w));
    }
}

// For n = 2h (+1): element i < h runs in lane .x and element i + h in lane .y
// of the packed generator (the one the hot kernels inline); an odd last
// element n - 1 runs in lane .x with a copy of itself in lane .y.
__global__ void box_muller_words_kernel(const uint32_t* __restrict__ a, const uint32_t* __restrict__ b, long long n,
                                        float* __restrict__ ne, float* __restrict__ no) {
    const long long h = n >> 1, pairs = (n + 1) >> 1;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < pairs;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long i0 = i < h ? i : n - 1, i1 = i < h ? i + h : n - 1;
        const Polar2 p = box_muller_polar2(a[i0], b[i0], a[i1], b[i1]);
        const float2 e = __fmul2_rn(p.rho, p.cos_t), o = __fmul2_rn(p.rho, p.sin_t);
        ne[i0] = e.x;
        no[i0] = o.x;
        if (i1 != i0) {
            ne[i1] = e.y;
            no[i1] = o.y;
        }
    }
}

// Block: 8 warps; warp w owns token s = blockIdx.x * 8 + w, lane l owns draw
// k = blockIdx.y * 32 + l, so the u row is a warp-wide broadcast.  The 8 x 32
// results are transposed through shared memory into 32-byte runs of c.
__global__ void __launch_bounds__(256)
synth_costs_kernel(const float* __restrict__ u, int T, int d_out, uint32_t seed, uint32_t layer,
                   uint32_t draw_begin, uint32_t tok0, int nd, float sigma, float eps_scale,
                   float* __restrict__ c) {
    __shared__ float tile[32][9];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x * 8 + warp;
    const int k = blockIdx.y * 32 + lane;
    float val = 0.0f;
    if (s < T && k < nd) {
        const uint32_t draw = draw_begin + static_cast<uint32_t>(k);
        const float* us = u + static_cast<size_t>(s) * d_out;
        const int nq = (d_out + 3) / 4;
        float dot0 = 0.0f, dot1 = 0.0f;
        for (int q = 0; q < nq; ++q) {
            float4 uv;
            if ((d_out & 3) == 0) {
                uv = __ldg(reinterpret_cast<const float4*>(us) + q);
            } else {
                const int j = 4 * q;
                uv.x = __ldg(us + j);
                uv.y = j + 1 < d_out ? __ldg(us + j + 1) : 0.0f;
                uv.z = j + 2 < d_out ? __ldg(us + j + 2) : 0.0f;
                uv.w = j + 3 < d_out ? __ldg(us + j + 3) : 0.0f;
            }
            const float4 a = gauss4(seed, layer, draw, tok0 + static_cast<uint32_t>(s), static_cast<uint32_t>(q), 0);
            dot0 = __fmaf_rn(uv.x, a.x, dot0);
            dot1 = __fmaf_rn(uv.y, a.y, dot1);
            dot0 = __fmaf_rn(uv.z, a.z, dot0);
            dot1 = __fmaf_rn(uv.w, a.w, dot1);
        }
        const float eps = gauss4(seed, layer, draw, tok0 + static_cast<uint32_t>(s), 0, 1).x;
        val = sigma * (dot0 + dot1) + eps_scale * eps;
    }
    tile[lane][warp] = val;
    __syncthreads();
    const int kk = threadIdx.x >> 3, ss = threadIdx.x & 7;
    const int k2 = blockIdx.y * 32 + kk, s2 = blockIdx.x * 8 + ss;
    if (k2 < nd && s2 < T) c[static_cast<size_t>(k2) * T + s2] = tile[kk][ss];
}

}  // namespace

cudaError_t launch_noise_fill(const dust_noise& nz, uint32_t stream_id, int t0, int n_tok, int j0,
                              int n_ch, float* out, cudaStream_t stream) {
    const long long total = static_cast<long long>(nz.draw_count) * n_tok * n_ch;
    if (total == 0) return cudaSuccess;
    const long long blocks = ceil_div(total, 256);
    noise_fill_kernel<<<static_cast<unsigned>(blocks < 65536 ? blocks : 65536), 256, 0, stream>>>(
        nz.seed, nz.layer, stream_id, nz.draw_begin, static_cast<int>(nz.draw_count), nz.token_begin, t0, n_tok, j0,
        n_ch, out);
    return cudaGetLastError();
}

cudaError_t launch_box_muller_words(const uint32_t* a, const uint32_t* b, long long n, float* ne, float* no,
                                    cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const long long blocks = ceil_div((n + 1) / 2, 256);
    box_muller_words_kernel<<<static_cast<unsigned>(blocks < 8 * 1184 ? blocks : 8 * 1184), 256, 0, stream>>>(a, b, n,
                                                                                                            ne, no);
    return cudaGetLastError();
}

cudaError_t launch_synth_costs(const float* u, int T, int d_out, const dust_noise& nz, float eps_scale,
                               float* c, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(ceil_div(T, 8)), static_cast<unsigned>(ceil_div(nz.draw_count, 32)));
    synth_costs_kernel<<<grid, 256, 0, stream>>>(u, T, d_out, nz.seed, nz.layer, nz.draw_begin, nz.token_begin,
                                                 static_cast<int>(nz.draw_count), nz.sigma, eps_scale, c);
    return cudaGetLastError();
}

}  // namespace dust
