// estimate.cuh -- one step of the draw reduction (a1 + a5), shared by the
// standalone reduction and the fused reduction + weight-estimate kernel so
// that both produce the same g bit for bit.
//
// cnblogs Dust explainer, section "信用分配：一次前向，两种奖励", error
// equation: g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i).
#pragma once
#include <cstdint>

#include "noise.cuh"

namespace dust {

// acc += r * a for the 4 channels of one Philox call, as two packed lanes:
// xz holds channels (4q, 4q+2), yw channels (4q+1, 4q+3).  r is folded into
// the Box-Muller radius (r * rho once per pair instead of rho * cos and
// rho * sin).
__device__ __forceinline__ void accumulate_quad(float2& xz, float2& yw, float r, uint32_t seed, uint32_t layer,
                                                uint32_t draw, uint32_t token, uint32_t quad) {
    const uint4 x = philox4x32_10(make_uint4(quad, token, draw, 0u), seed, layer);
    const Polar2 p = box_muller_polar2(x.x, x.y, x.z, x.w);
    const float2 rr = __fmul2_rn(splat(r), p.rho);
    xz = __ffma2_rn(rr, p.cos_t, xz);
    yw = __ffma2_rn(rr, p.sin_t, yw);
}

// accumulate_quad from the state after Philox round 1 (philox_round1_state).
__device__ __forceinline__ void accumulate_quad_after_round1(float2& xz, float2& yw, float r, uint4 c1, uint32_t seed,
                                                             uint32_t layer) {
    const uint4 x = philox4x32_10_after_round1(c1, seed, layer);
    const Polar2 p = box_muller_polar2(x.x, x.y, x.z, x.w);
    const float2 rr = __fmul2_rn(splat(r), p.rho);
    xz = __ffma2_rn(rr, p.cos_t, xz);
    yw = __ffma2_rn(rr, p.sin_t, yw);
}

}  // namespace dust
