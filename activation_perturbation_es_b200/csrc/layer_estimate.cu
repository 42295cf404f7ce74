// layer_estimate.cu -- a1 + a5: noise regeneration and the noise-weighted
// reduction over draws.
//
// cnblogs Dust explainer, section "信用分配：一次前向，两种奖励", error
// equation: g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i).
//
// Design (B200): the work is K x T x d_out Gaussians, each regenerated from its
// coordinates (noise.cuh) and consumed by one FMA; nothing K x T x d is ever
// stored, and the only HBM traffic is r (4 bytes per draw x token, a warp-wide
// broadcast) and g (written once).  The kernel is therefore bound by the SM's
// fp32/integer-multiply datapath, not by HBM.  One thread owns (token t,
// channel quad q): a single Philox call per draw yields its 4 channels, whose
// two Box-Muller pairs run in lock-step on the packed fp32 pipes.  Work that
// does not change along the draw loop leaves it: the key schedule, and the
// quad's half of Philox round 1 (philox_round1_quad); the draw's half is the
// 64-bit product M1 d, stepped by an add from one draw to the next instead of a
// wide multiply on the busiest datapath.  A warp shares its token, so lane j
// loads r for draw k0 + j once per 32 draws and the loop takes them by shuffle,
// with no per-draw address arithmetic.  Four draws per iteration alternate
// between two accumulator pairs (even and odd draws), which gives the scheduler
// independent chains and fixes the summation order.  Blocks are 256 threads:
// quads along x (coalesced 128-bit stores of g), tokens along y.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "estimate.cuh"
#include "noise.cuh"

namespace dust {

namespace {

// The epilogue's options are template parameters (kVec: d_out % 4 == 0, 128-bit
// stores; kAcc: add into g; kG16: also write the bf16 copy): with runtime flags
// the compiler's register allocation of the draw loop cost ~1% on B200.
template <bool kVec, bool kAcc, bool kG16>
__global__ void __launch_bounds__(256)
layer_estimate_kernel(const float* __restrict__ r, int T, int d_out, int nq, uint32_t seed,
                      uint32_t layer, uint32_t draw_begin, uint32_t tok0, int nd, float scale,
                      float* __restrict__ g, __nv_bfloat16* __restrict__ g16) {
    // a warp shares one token (blockDim.x >= 32): lane j loads the r of draw
    // k0 + j and the draws of a 32-draw group are passed round by shuffles
    const int q_raw = blockIdx.x * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    if (__all_sync(0xffffffffu, q_raw >= nq)) return;
    const int q = q_raw < nq ? q_raw : nq - 1;
    const uint2 rq = philox_round1_quad(static_cast<uint32_t>(q), 0u, layer);
    for (int t = blockIdx.y * blockDim.y + threadIdx.y; t < T; t += gridDim.y * blockDim.y) {
        float2 xz0 = splat(0.0f), yw0 = splat(0.0f), xz1 = splat(0.0f), yw1 = splat(0.0f);
        const float* rt = r + t;
        const uint32_t tok = tok0 + static_cast<uint32_t>(t);     // the token's global index: its noise
        DrawProduct dp = draw_product(draw_begin);
        for (int k0 = 0; k0 < nd; k0 += 32) {
            const int n = nd - k0 < 32 ? nd - k0 : 32;
            const float rv = lane < n ? __ldg(rt + static_cast<size_t>(k0 + lane) * T) : 0.0f;
            int j = 0;
            for (; j + 4 <= n; j += 4) {
                const float r0 = __shfl_sync(0xffffffffu, rv, j), r1 = __shfl_sync(0xffffffffu, rv, j + 1);
                const float r2 = __shfl_sync(0xffffffffu, rv, j + 2), r3 = __shfl_sync(0xffffffffu, rv, j + 3);
                accumulate_quad_after_round1(xz0, yw0, r0, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
                accumulate_quad_after_round1(xz1, yw1, r1, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
                accumulate_quad_after_round1(xz0, yw0, r2, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
                accumulate_quad_after_round1(xz1, yw1, r3, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
            }
            for (; j + 2 <= n; j += 2) {
                const float r0 = __shfl_sync(0xffffffffu, rv, j), r1 = __shfl_sync(0xffffffffu, rv, j + 1);
                accumulate_quad_after_round1(xz0, yw0, r0, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
                accumulate_quad_after_round1(xz1, yw1, r1, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
            }
            if (j < n) {
                const float r0 = __shfl_sync(0xffffffffu, rv, j);
                accumulate_quad_after_round1(xz0, yw0, r0, philox_round1_state(dp, tok, seed, rq), seed, layer);
                next_draw(dp);
            }
        }
        if (q_raw >= nq) continue;
        float4 out = make_float4((xz0.x + xz1.x) * scale, (yw0.x + yw1.x) * scale,
                                 (xz0.y + xz1.y) * scale, (yw0.y + yw1.y) * scale);
        const size_t base = static_cast<size_t>(t) * d_out + 4 * static_cast<size_t>(q);
        if constexpr (kVec) {
            float4* gp = reinterpret_cast<float4*>(g + base);
            if constexpr (kAcc) {
                const float4 o = *gp;
                out.x += o.x; out.y += o.y; out.z += o.z; out.w += o.w;
            }
            *gp = out;
            if constexpr (kG16) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(out.x, out.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(out.z, out.w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t*>(&lo);
                pk.y = *reinterpret_cast<uint32_t*>(&hi);
                *reinterpret_cast<uint2*>(g16 + base) = pk;
            }
        } else {
            const float v[4] = {out.x, out.y, out.z, out.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                if (4 * q + w >= d_out) break;
                float x = v[w];
                if constexpr (kAcc) x += g[base + w];
                g[base + w] = x;
                if constexpr (kG16) g16[base + w] = __float2bfloat16_rn(x);
            }
        }
    }
}

template <bool kVec, bool kAcc>
void launch_g16(bool with_g16, dim3 grid, dim3 block, cudaStream_t stream, const float* r, int T, int d_out, int nq,
                const dust_noise& nz, float scale, float* g, __nv_bfloat16* g16) {
    const int nd = static_cast<int>(nz.draw_count);
    if (with_g16)
        layer_estimate_kernel<kVec, kAcc, true><<<grid, block, 0, stream>>>(r, T, d_out, nq, nz.seed, nz.layer,
                                                                            nz.draw_begin, nz.token_begin, nd,
                                                                            scale, g, g16);
    else
        layer_estimate_kernel<kVec, kAcc, false><<<grid, block, 0, stream>>>(r, T, d_out, nq, nz.seed, nz.layer,
                                                                             nz.draw_begin, nz.token_begin, nd,
                                                                             scale, g, g16);
}

}  // namespace

cudaError_t launch_layer_estimate(const float* r, int T, int d_out, const dust_noise& nz, float* g,
                                  void* g_bf16, int accumulate, cudaStream_t stream) {
    const int nq = (d_out + 3) / 4;
    int bx = nq >= 128 ? 128 : ((nq + 31) / 32) * 32;
    const int by = 256 / bx;
    const unsigned gx = static_cast<unsigned>(ceil_div(nq, bx));
    const long long ty = ceil_div(T, by);
    const unsigned gy = static_cast<unsigned>(ty < 65535 ? ty : 65535);
    const float scale = static_cast<float>(-1.0 / (static_cast<double>(nz.K_total) * nz.sigma));
    auto* g16 = static_cast<__nv_bfloat16*>(g_bf16);
    const dim3 grid(gx, gy), block(bx, by);
    const bool vec = (d_out & 3) == 0, acc = accumulate != 0, with_g16 = g16 != nullptr;
    if (vec && !acc) launch_g16<true, false>(with_g16, grid, block, stream, r, T, d_out, nq, nz, scale, g, g16);
    else if (vec) launch_g16<true, true>(with_g16, grid, block, stream, r, T, d_out, nq, nz, scale, g, g16);
    else if (!acc) launch_g16<false, false>(with_g16, grid, block, stream, r, T, d_out, nq, nz, scale, g, g16);
    else launch_g16<false, true>(with_g16, grid, block, stream, r, T, d_out, nq, nz, scale, g, g16);
    return cudaGetLastError();
}

}  // namespace dust
