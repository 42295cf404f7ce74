// noise_sum.cu -- the generator's empirical ceiling: the noise of a draw range
// summed per (token, channel), out[t][j] = sum_k a(seed, layer, draw_begin + k,
// token_begin + t, j).
//
// The noise is a_t^(i) ~ N(0, I) per draw and token (cnblogs Dust explainer,
// section "信用分配：一次前向，两种奖励"); every consumer regenerates it.  This
// kernel does that with the least possible work around the generator: each
// Gaussian is consumed by one fused multiply-add, which also applies the
// Box-Muller radius (acc + rho cos, rounded once), and nothing is read from
// HBM.  Its Gaussians/s bound what any noise consumer in this library can
// reach on the same GPU, so the draw reduction and the head's cross entropy
// are reported against it as well as against the issue-slot roofline.  The
// loop is the draw reduction's without r: the quad half of Philox round 1 is
// computed once per thread, the draw half M1 d is stepped by a 64-bit add, and
// four draws per iteration alternate between two accumulator pairs.
#include "common.cuh"
#include "kernels.h"
#include "noise.cuh"

namespace dust {

namespace {

// M1 d stepped to M1 (d + 1) as one plain 64-bit add: the same value as
// next_draw's carry chain, left to the compiler's choice of form, which runs
// this kernel about 1% faster (the draw reduction is unchanged by it).
__device__ __forceinline__ void next_draw_u64(DrawProduct& p) {
    const unsigned long long v = ((static_cast<unsigned long long>(p.hi) << 32) | p.lo) + kPhiloxM1;
    p.lo = static_cast<uint32_t>(v);
    p.hi = static_cast<uint32_t>(v >> 32);
}

// xz += rho (cos) and yw += rho (sin) for the 4 channels of one Philox call,
// as two packed lanes (channels (4q, 4q+2) and (4q+1, 4q+3))
__device__ __forceinline__ void sum_quad_after_round1(float2& xz, float2& yw, uint4 c1, uint32_t seed,
                                                      uint32_t layer) {
    const uint4 x = philox4x32_10_after_round1(c1, seed, layer);
    const Polar2 p = box_muller_polar2(x.x, x.y, x.z, x.w);
    xz = __ffma2_rn(p.rho, p.cos_t, xz);
    yw = __ffma2_rn(p.rho, p.sin_t, yw);
}

template <bool kVec>
__global__ void __launch_bounds__(256)
noise_sum_kernel(int T, int d, int nq, uint32_t seed, uint32_t layer, uint32_t draw_begin, uint32_t tok0, int nd,
                 float* __restrict__ out) {
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= nq) return;                  // no warp-wide operations below
    const uint2 rq = philox_round1_quad(static_cast<uint32_t>(q), 0u, layer);
    for (int t = blockIdx.y * blockDim.y + threadIdx.y; t < T; t += gridDim.y * blockDim.y) {
        const uint32_t tok = tok0 + static_cast<uint32_t>(t);
        float2 xz0 = splat(0.0f), yw0 = splat(0.0f), xz1 = splat(0.0f), yw1 = splat(0.0f);
        DrawProduct dp = draw_product(draw_begin);
        int k = 0;
        for (; k + 4 <= nd; k += 4) {
            sum_quad_after_round1(xz0, yw0, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
            sum_quad_after_round1(xz1, yw1, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
            sum_quad_after_round1(xz0, yw0, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
            sum_quad_after_round1(xz1, yw1, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
        }
        for (; k + 2 <= nd; k += 2) {
            sum_quad_after_round1(xz0, yw0, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
            sum_quad_after_round1(xz1, yw1, philox_round1_state(dp, tok, seed, rq), seed, layer);
            next_draw_u64(dp);
        }
        if (k < nd) sum_quad_after_round1(xz0, yw0, philox_round1_state(dp, tok, seed, rq), seed, layer);
        const float v[4] = {xz0.x + xz1.x, yw0.x + yw1.x, xz0.y + xz1.y, yw0.y + yw1.y};
        const size_t base = static_cast<size_t>(t) * d + 4 * static_cast<size_t>(q);
        if constexpr (kVec) {
            *reinterpret_cast<float4*>(out + base) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (4 * q + w < d) out[base + w] = v[w];
        }
    }
}

}  // namespace

cudaError_t launch_noise_sum(const dust_noise& nz, int T, int d, float* out, cudaStream_t stream) {
    const int nq = (d + 3) / 4;
    const int bx = nq >= 128 ? 128 : ((nq + 31) / 32) * 32;
    const int by = 256 / bx;
    const long long ty = ceil_div(T, by);
    const dim3 grid(static_cast<unsigned>(ceil_div(nq, bx)), static_cast<unsigned>(ty < 65535 ? ty : 65535));
    const dim3 block(bx, by);
    const int nd = static_cast<int>(nz.draw_count);
    if ((d & 3) == 0)
        noise_sum_kernel<true><<<grid, block, 0, stream>>>(T, d, nq, nz.seed, nz.layer, nz.draw_begin, nz.token_begin,
                                                           nd, out);
    else
        noise_sum_kernel<false><<<grid, block, 0, stream>>>(T, d, nq, nz.seed, nz.layer, nz.draw_begin,
                                                            nz.token_begin, nd, out);
    return cudaGetLastError();
}

}  // namespace dust
