// common.cuh -- internal helpers shared by the library's translation units.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "dust.h"

namespace dust {

constexpr int kNumSMs = 148;   // B200: 2 dies x 74 SMs (queried at run time where it matters)

__host__ __device__ inline int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }
__host__ __device__ inline long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

// Sequence bounds of sequence q, clamped into [0, T] and made non-decreasing,
// so that malformed offsets cannot send a kernel outside its tensors.
__device__ __forceinline__ int2 seq_bounds(const int32_t* offs, int q, int T) {
    const int s0 = clamp_int(__ldg(offs + q), 0, T);
    int s1 = clamp_int(__ldg(offs + q + 1), 0, T);
    if (s1 < s0) s1 = s0;
    return make_int2(s0, s1);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Status block at the start of every workspace (256 bytes): word 0 is set by a
// kernel whose bounded wait ran out.
constexpr size_t kStatusBytes = 256;
constexpr uint32_t kStatusTimeout = 0x54494D45u;   // "TIME"

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace dust
