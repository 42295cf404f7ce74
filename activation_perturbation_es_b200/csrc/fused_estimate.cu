// fused_estimate.cu -- a1 + a5 + a6 in one kernel: the draw reduction writes
// its bf16 g tile straight into shared memory, where it is the A operand of
// tcgen05.mma; the weight estimate's row block accumulates in TMEM.  g never
// goes to HBM.
//
// cnblogs Dust explainer, section "信用分配：一次前向，两种奖励": error equation
// g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i) and weight equation
// G_W = sum_t g_t x_t^T.
//
// One CTA owns a block of 128 output channels (rows of G_W) and a range of
// tokens; its TMEM holds the whole d_in-wide row block of G_W (fp32, up to 512
// columns), so every g value is produced once.  Tokens go through a ring of
// stages of kTs = 48 tokens:
//   warps 2..25 (producers): thread (warp w, lane q) computes the 4 channels
//     of quad q for the tokens t0 + w and t0 + w + 24 of the stage with the
//     same arithmetic as the standalone reduction (estimate.cuh), scales,
//     rounds to bf16 (RNE) and stores them into the stage's A tile in the
//     MN-major, 128-byte-swizzled layout that TMA would have produced; then a
//     proxy fence and one arrive per warp on the stage's a_full barrier;
//   warp 0, one lane: TMA loads of the stage's X tile (d_in/64 atoms of kTs
//     rows, into this CTA only) onto x_full;
//   warp 1, one lane: allocates TMEM, and per stage issues kTs/16 K steps of
//     tcgen05.mma (M = 128, N <= 256 per instruction) and commits the stage's
//     empty barrier.
// After the last stage the producers drain TMEM into an fp32 partial row
// block for their token split; the split-K reduction sums the splits in a
// fixed order.  Every wait is bounded and gives up when another role aborts.
#include <cuda_bf16.h>

#include "common.cuh"
#include "estimate.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace dust {

namespace {

using namespace tc;

constexpr int kProducerWarps = 24;
constexpr int kTs = 2 * kProducerWarps;              // tokens per stage (a multiple of 16)
constexpr int kFusedThreads = 64 + 32 * kProducerWarps;
constexpr int kRows = 128;                            // output channels per CTA (MMA M)
constexpr int kAtom = kTs * 128;                      // one 64-wide MN atom of kTs K rows, bytes
constexpr int kATile = 2 * kAtom;
constexpr int kMaxStages = 4;
// A stage's A tile fills only when the producers have run all of the call's
// draws for it, so the waits that span a stage's production are bounded in
// time on the GPU's global nanosecond timer, by a budget that grows with the
// draw count: 2 s plus 20 us per draw.  One draw of one stage is 48 tokens x
// 128 channels of noise, about 1.2 us on one SM, so the budget is more than
// ten times the longest legitimate wait.  The host caps a call at
// kFusedMaxDraws draws (23 s).
constexpr uint64_t kProduceBudgetBaseNs = 2000000000ull;
constexpr uint64_t kProduceBudgetPerDrawNs = 20000ull;

struct FusedLayout {
    int d_in, stage_bytes, stages, bytes;
};

__host__ __device__ inline FusedLayout fused_layout(int d_in) {
    FusedLayout L;
    L.d_in = d_in;
    L.stage_bytes = kATile + (d_in / 64) * kAtom;
    L.stages = 1;
    while (L.stages < kMaxStages && (L.stages + 1) * L.stage_bytes + 2048 <= 200 * 1024) ++L.stages;
    L.bytes = L.stages * L.stage_bytes + 1024 /*align*/ + 256 /*barriers*/;
    return L;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                              uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (it > 64) __nanosleep(256);
    }
    return false;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// The same wait, bounded by budget_ns of global-timer time (the poll count is
// capped as well, as a last bound that does not depend on the timer).
__device__ __forceinline__ bool wait_or_abort_ns(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                                 uint64_t budget_ns) {
    const uint64_t start = global_ns();
    for (uint32_t it = 0; it < 0xFFFFFFF0u; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (it > 64) {
            __nanosleep(256);
            if ((it & 255u) == 0u && global_ns() - start > budget_ns) return false;
        }
    }
    return false;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kFusedThreads, 1)
fused_estimate_kernel(const __grid_constant__ CUtensorMap map_x, const float* __restrict__ r, int T, int d_out,
                      int d_in, uint32_t seed, uint32_t layer, uint32_t draw_begin, uint32_t tok0, int nd, float scale,
                      int tokens_per_split, float* __restrict__ partial, float* __restrict__ g_hat,
                      uint32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const FusedLayout L = fused_layout(d_in);
    uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + L.stages * L.stage_bytes);
    uint64_t* x_full = a_full + kMaxStages;
    uint64_t* empty = x_full + kMaxStages;
    uint64_t* acc_full = empty + kMaxStages;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (d_out + kRows - 1) / kRows;
    const int o0 = (blockIdx.x % tiles_m) * kRows;
    const int split = blockIdx.x / tiles_m;
    const int tb = split * tokens_per_split;
    const int te = min(T, tb + tokens_per_split);
    const int n_stages = te > tb ? (te - tb + kTs - 1) / kTs : 0;
    const uint32_t tmem_cols = d_in <= 64 ? 64u : (d_in <= 128 ? 128u : (d_in <= 256 ? 256u : 512u));
    const uint64_t produce_limit = kProduceBudgetBaseNs + kProduceBudgetPerDrawNs * static_cast<uint64_t>(nd);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.stages; ++s) {
            mbar_init(&a_full[s], kProducerWarps);
            mbar_init(&x_full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_slot, tmem_cols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA: X tiles [kTs tokens][d_in] as d_in/64 MN atoms
            int it = 0;
            bool ok = true;
            for (; it < n_stages; ++it) {
                const int s = it % L.stages;
                if (it >= L.stages &&
                    !wait_or_abort_ns(&empty[s], ((it / L.stages) - 1) & 1, abort_flag, produce_limit)) {
                    ok = false;
                    break;
                }
                uint8_t* sb = smem + s * L.stage_bytes + kATile;
                mbar_arrive_expect_tx(&x_full[s], static_cast<uint32_t>((d_in / 64) * kAtom));
                for (int h = 0; h < d_in / 64; ++h) tma_load_2d(sb + h * kAtom, &map_x, &x_full[s], 64 * h, tb + it * kTs);
            }
            if (!ok) {
                atomicExch(status, kStatusTimeout);
                *abort_flag = 1;
            }
            for (int j = it > L.stages ? it - L.stages : 0; j < it; ++j) mbar_wait(&x_full[j % L.stages], (j / L.stages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const int n_chunks = (d_in + 255) / 256;
            bool ok = true;
            for (int it = 0; it < n_stages && ok; ++it) {
                const int s = it % L.stages;
                if (!wait_or_abort_ns(&a_full[s], (it / L.stages) & 1, abort_flag, produce_limit) ||
                    !wait_or_abort(&x_full[s], (it / L.stages) & 1, abort_flag, kWaitLimit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * L.stage_bytes);
                const uint32_t sb = sa + kATile;
#pragma unroll 1
                for (int j = 0; j < kTs / 16; ++j) {
                    // MN-major operands: a 16-deep k step is 16 rows of 128 bytes; the
                    // leading byte offset is the distance between 64-wide MN atoms
                    const uint64_t ad = smem_desc(sa + j * 16 * 128, kAtom, 1024);
                    for (int c = 0; c < n_chunks; ++c) {
                        const int n = min(256, d_in - 256 * c);
                        const uint64_t bd = smem_desc(sb + c * 4 * kAtom + j * 16 * 128, kAtom, 1024);
                        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                               (static_cast<uint32_t>(n >> 3) << 17) |
                                               (static_cast<uint32_t>(kRows >> 4) << 24);
                        tc_mma(tmem + static_cast<uint32_t>(256 * c), ad, bd, idesc, (it > 0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[s]);
            }
            if (!ok) {
                atomicExch(status, kStatusTimeout);
                *abort_flag = 1;
            } else if (n_stages > 0) {
                tc_commit(acc_full);      // arrives once every MMA above has completed
            }
            tc_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ---------------- producers: g tiles into shared memory
        const int pw = warp - 2;                    // 0 .. kProducerWarps - 1
        const uint32_t quad = static_cast<uint32_t>(o0 / 4 + lane);
        const uint2 rq = philox_round1_quad(quad, 0u, layer);
        const int atom = lane >> 4;                 // channels 4q .. 4q+3 lie in MN atom q / 16
        const int chunk = (lane & 15) >> 1;         // 16-byte chunk of the 128-byte row
        const int half8 = (lane & 1) * 8;           // byte offset inside the chunk
        bool ok = true;
        for (int it = 0; it < n_stages; ++it) {
            const int s = it % L.stages;
            if (it >= L.stages &&
                !wait_or_abort_ns(&empty[s], ((it / L.stages) - 1) & 1, abort_flag, produce_limit)) {
                ok = false;
                break;
            }
            uint8_t* sa = smem + s * L.stage_bytes;
            const int row0 = pw, row1 = pw + kProducerWarps;
            const int t0 = tb + it * kTs + row0, t1 = tb + it * kTs + row1;
            const bool v0 = t0 < te, v1 = t1 < te;      // warp-uniform
            float2 xa0 = splat(0.0f), ya0 = splat(0.0f), xa1 = splat(0.0f), ya1 = splat(0.0f);
            float2 xb0 = splat(0.0f), yb0 = splat(0.0f), xb1 = splat(0.0f), yb1 = splat(0.0f);
            if (v0) {
                // the standalone reduction's loop (same draw order and accumulator
                // pairs) on two tokens; when t1 lies past the split it repeats t0
                const int ta = t0, tb_ = v1 ? t1 : t0;
                const float* ra = r + ta;
                const float* rb = r + tb_;
                const uint32_t ua = tok0 + static_cast<uint32_t>(ta), ub = tok0 + static_cast<uint32_t>(tb_);
                DrawProduct dp = draw_product(draw_begin);
                for (int k0 = 0; k0 < nd; k0 += 32) {
                    const int n = nd - k0 < 32 ? nd - k0 : 32;
                    const float rva = lane < n ? __ldg(ra + static_cast<size_t>(k0 + lane) * T) : 0.0f;
                    const float rvb = lane < n ? __ldg(rb + static_cast<size_t>(k0 + lane) * T) : 0.0f;
                    int j = 0;
                    for (; j + 2 <= n; j += 2) {
                        const float a0 = __shfl_sync(0xffffffffu, rva, j), a1 = __shfl_sync(0xffffffffu, rva, j + 1);
                        const float b0 = __shfl_sync(0xffffffffu, rvb, j), b1 = __shfl_sync(0xffffffffu, rvb, j + 1);
                        accumulate_quad_after_round1(xa0, ya0, a0, philox_round1_state(dp, ua, seed, rq), seed, layer);
                        accumulate_quad_after_round1(xb0, yb0, b0, philox_round1_state(dp, ub, seed, rq), seed, layer);
                        next_draw(dp);
                        accumulate_quad_after_round1(xa1, ya1, a1, philox_round1_state(dp, ua, seed, rq), seed, layer);
                        accumulate_quad_after_round1(xb1, yb1, b1, philox_round1_state(dp, ub, seed, rq), seed, layer);
                        next_draw(dp);
                    }
                    if (j < n) {
                        const float a0 = __shfl_sync(0xffffffffu, rva, j), b0 = __shfl_sync(0xffffffffu, rvb, j);
                        accumulate_quad_after_round1(xa0, ya0, a0, philox_round1_state(dp, ua, seed, rq), seed, layer);
                        accumulate_quad_after_round1(xb0, yb0, b0, philox_round1_state(dp, ub, seed, rq), seed, layer);
                        next_draw(dp);
                    }
                }
            }
            // g in the standalone reduction's order: (even draws + odd draws) * scale
            const float4 ga = make_float4((xa0.x + xa1.x) * scale, (ya0.x + ya1.x) * scale,
                                          (xa0.y + xa1.y) * scale, (ya0.y + ya1.y) * scale);
            const float4 gb = make_float4((xb0.x + xb1.x) * scale, (yb0.x + yb1.x) * scale,
                                          (xb0.y + xb1.y) * scale, (yb0.y + yb1.y) * scale);
            const float4 za = v0 ? ga : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 zb = v1 ? gb : make_float4(0.f, 0.f, 0.f, 0.f);
            uint2 pa, pb;
            pa.x = pack_bf16x2(za.x, za.y);
            pa.y = pack_bf16x2(za.z, za.w);
            pb.x = pack_bf16x2(zb.x, zb.y);
            pb.y = pack_bf16x2(zb.z, zb.w);
            // 128-byte swizzle: the 16-byte chunk index is xor-ed with the row's low 3 bits
            *reinterpret_cast<uint2*>(sa + atom * kAtom + row0 * 128 + ((chunk ^ (row0 & 7)) << 4) + half8) = pa;
            *reinterpret_cast<uint2*>(sa + atom * kAtom + row1 * 128 + ((chunk ^ (row1 & 7)) << 4) + half8) = pb;
            if (g_hat != nullptr) {
                const int c0 = 4 * static_cast<int>(quad);
                const float va[4] = {ga.x, ga.y, ga.z, ga.w}, vb[4] = {gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (c0 + w < d_out) {
                        if (v0) g_hat[static_cast<size_t>(t0) * d_out + c0 + w] = va[w];
                        if (v1) g_hat[static_cast<size_t>(t1) * d_out + c0 + w] = vb[w];
                    }
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic stores -> tensor-core reads
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&a_full[s])) : "memory");
        }
        if (!ok) {
            atomicExch(status, kStatusTimeout);
            *abort_flag = 1;
        }
        // ---------------- epilogue: TMEM -> fp32 partial row block of this token split
        bool have = false;
        if (ok && n_stages > 0) {
            have = wait_or_abort_ns(acc_full, 0, abort_flag, produce_limit);
            if (!have) {                               // this split's row block stays unwritten: say so
                atomicExch(status, kStatusTimeout);
                *abort_flag = 1;
            }
        }
        have = __all_sync(0xffffffffu, have);
        const int quarter = warp & 3;                 // the TMEM lane quarter this warp may read
        const int idx = pw >> 2;                      // 0 .. kProducerWarps/4 - 1 within the quarter
        const int row = o0 + quarter * 32 + lane;
        float* dst = partial + (static_cast<size_t>(split) * d_out + row) * d_in;
        if (ok && n_stages == 0 && row < d_out) {     // an empty token split contributes zeros
            for (int c0 = 32 * idx; c0 < d_in; c0 += 32 * (kProducerWarps / 4))
                for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + c0 + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (have) {
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 32 * idx; c0 < d_in; c0 += 32 * (kProducerWarps / 4)) {
                float v[32];
                tmem_ld32(tmem + static_cast<uint32_t>(c0) + (static_cast<uint32_t>(quarter * 32) << 16), v);
                if (row < d_out) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

struct Split {
    int tokens_per_split, n_splits;
};

Split fused_split(int T, int d_out) {
    const int tiles_m = (d_out + kRows - 1) / kRows;
    const int stages_total = (T + kTs - 1) / kTs;
    int want = device_sm_count() / tiles_m;
    if (want < 1) want = 1;
    if (want > stages_total) want = stages_total;
    const int stages_per_split = (stages_total + want - 1) / want;
    Split sp;
    sp.tokens_per_split = stages_per_split * kTs;
    sp.n_splits = (T + sp.tokens_per_split - 1) / sp.tokens_per_split;
    return sp;
}

}  // namespace

bool fused_estimate_supported(int d_in, int d_out) {
    return d_in >= 64 && d_in <= 512 && d_in % 64 == 0 && d_out > 0;
}

size_t fused_estimate_scratch(int T, int d_in, int d_out) {
    if (T <= 0 || !fused_estimate_supported(d_in, d_out)) return 0;
    // the split count depends only on T, d_out and the SM count; bound it by
    // the SM count so the size does not depend on the device queried
    const int tiles_m = (d_out + kRows - 1) / kRows;
    const long long stages_total = (T + kTs - 1) / kTs;
    long long splits = kNumSMs * 2 / tiles_m;
    if (splits < 1) splits = 1;
    if (splits > stages_total) splits = stages_total;
    return sizeof(float) * static_cast<size_t>(splits) * d_out * d_in;
}

cudaError_t launch_fused_estimate(const float* r, int T, int d_out, const void* X, int d_in, const dust_noise& nz,
                                  float* G, int accumulate, float* g_hat, void* scratch, uint32_t* status,
                                  cudaStream_t stream) {
    if (!fused_estimate_supported(d_in, d_out)) return cudaErrorNotSupported;
    const Split sp = fused_split(T, d_out);
    const int tiles_m = (d_out + kRows - 1) / kRows;
    if (sizeof(float) * static_cast<size_t>(sp.n_splits) * d_out * d_in > fused_estimate_scratch(T, d_in, d_out))
        return cudaErrorInvalidValue;
    CUtensorMap mx;
    if (!tma_map_bf16_2d(&mx, X, d_in, T, d_in, kTs)) return cudaErrorInvalidValue;
    const FusedLayout L = fused_layout(d_in);
    static cudaError_t attr_err = [] {
        int most = 0;       // the largest layout over every supported width
        for (int w = 64; w <= 512; w += 64) most = fused_layout(w).bytes > most ? fused_layout(w).bytes : most;
        return cudaFuncSetAttribute(fused_estimate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    }();
    if (attr_err != cudaSuccess) return attr_err;
    const float scale = static_cast<float>(-1.0 / (static_cast<double>(nz.K_total) * nz.sigma));
    auto* partial = static_cast<float*>(scratch);
    fused_estimate_kernel<<<static_cast<unsigned>(tiles_m * sp.n_splits), kFusedThreads, L.bytes, stream>>>(
        mx, r, T, d_out, d_in, nz.seed, nz.layer, nz.draw_begin, nz.token_begin, static_cast<int>(nz.draw_count), scale,
        sp.tokens_per_split, partial, g_hat, status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_splitk_reduce(partial, sp.n_splits, d_out, d_in, G, d_in, accumulate, stream);
}

}  // namespace dust
