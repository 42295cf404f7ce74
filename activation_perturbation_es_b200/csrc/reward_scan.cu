// reward_scan.cu -- a4: discounted reward (reverse segmented gamma-scan).
//
// cnblogs Dust explainer, section "信用分配：一次前向，两种奖励", reward
// equation: r_t = sum_{s >= t} gamma^(s-t) c_s, computed independently for
// every draw and, inside a draw row, for every sequence (causal attention does
// not carry a token's noise into another sequence).
//
// Design (B200): the scan reads c once and writes r once, 8 bytes per
// draw x token, so it is HBM-bound.  One CTA owns one (draw, sequence)
// segment and walks it from its end in chunks of kThreads * 8 tokens.  Each
// thread loads two aligned float4 quads (128-bit loads; elements of the quad
// that belong to a neighbouring segment are masked, never written), composes
// the affine maps x -> c + gamma x of its 8 tokens, and the CTA combines the
// per-thread maps with a warp-shuffle suffix scan plus one shared-memory step
// across warps.  The map of a whole chunk carries r into the previous chunk.
// In place (r == c) is safe, hence no __restrict__ on c and r: a CTA reads a
// chunk completely before writing it, and writes only its own segment.
#include "common.cuh"
#include "kernels.h"

namespace dust {

namespace {

constexpr int kScanThreads = 128;
constexpr int kScanVec = 8;                       // tokens per thread per chunk
constexpr int kScanChunk = kScanThreads * kScanVec;

struct Affine {   // x -> b + a x
    float a, b;
};

// f o g : apply g first (g is the later part of the sequence), then f.
__device__ __forceinline__ Affine compose(Affine f, Affine g) {
    return {f.a * g.a, __fmaf_rn(f.a, g.b, f.b)};
}

__global__ void __launch_bounds__(kScanThreads)
reward_scan_kernel(const float* c, float* r, long long total, int T,
                   const int32_t* __restrict__ offs, int n_seq, float gamma) {
    __shared__ Affine warp_maps[kScanThreads / 32];
    __shared__ float carry_in[kScanThreads / 32];
    __shared__ float next_carry;

    const long long seg = blockIdx.x;
    const int q = static_cast<int>(seg % n_seq);
    const long long row = (seg / n_seq) * static_cast<long long>(T);
    const int2 sb = seq_bounds(offs, q, T);
    if (sb.y <= sb.x) return;
    const long long lo = row + sb.x, hi = row + sb.y;         // flat element range
    const long long qlo = lo >> 2, qhi = (hi + 3) >> 2;        // aligned quads covering it
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    float carry = 0.0f;   // r just after the current chunk (0 past the sequence end)
    for (long long qend = qhi; qend > qlo; qend -= kScanChunk / 4) {
        const long long qbeg = qend - kScanChunk / 4 > qlo ? qend - kScanChunk / 4 : qlo;
        const long long myq = qbeg + 2LL * threadIdx.x;        // first of my two quads
        float v[kScanVec];
        bool ok[kScanVec];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long quad = myq + h;
            const long long e0 = quad * 4;
            if (quad < qend) {
                if (e0 + 4 <= total) {
                    const float4 x = *reinterpret_cast<const float4*>(c + e0);
                    v[4 * h + 0] = x.x; v[4 * h + 1] = x.y; v[4 * h + 2] = x.z; v[4 * h + 3] = x.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[4 * h + e] = (e0 + e < total) ? c[e0 + e] : 0.0f;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) ok[4 * h + e] = (e0 + e >= lo) && (e0 + e < hi);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) { v[4 * h + e] = 0.0f; ok[4 * h + e] = false; }
            }
        }
        // map of my 8 tokens (identity for masked ones), composed right to left
        Affine m = {1.0f, 0.0f};
#pragma unroll
        for (int e = kScanVec - 1; e >= 0; --e)
            if (ok[e]) m = {gamma * m.a, __fmaf_rn(gamma, m.b, v[e])};
        // inclusive suffix scan inside the warp: lane k gets map_k o ... o map_31
        Affine s = m;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            Affine t;
            t.a = __shfl_down_sync(0xffffffffu, s.a, o);
            t.b = __shfl_down_sync(0xffffffffu, s.b, o);
            if (lane + o < 32) s = compose(s, t);
        }
        if (lane == 0) warp_maps[warp] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            // exclusive suffix over warps applied to the carry, from the last warp back
            float x = carry;
            for (int w = kScanThreads / 32 - 1; w >= 0; --w) {
                carry_in[w] = x;
                x = __fmaf_rn(warp_maps[w].a, x, warp_maps[w].b);
            }
            next_carry = x;
        }
        __syncthreads();
        // my input: the suffix map of the lanes after me, applied to the warp's carry
        Affine after;
        after.a = __shfl_down_sync(0xffffffffu, s.a, 1);
        after.b = __shfl_down_sync(0xffffffffu, s.b, 1);
        if (lane == 31) after = {1.0f, 0.0f};
        float x = __fmaf_rn(after.a, carry_in[warp], after.b);
        float out[kScanVec];
#pragma unroll
        for (int e = kScanVec - 1; e >= 0; --e) {
            if (ok[e]) x = __fmaf_rn(gamma, x, v[e]);
            out[e] = x;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long quad = myq + h;
            const long long e0 = quad * 4;
            if (quad >= qend) continue;
            if (ok[4 * h] && ok[4 * h + 1] && ok[4 * h + 2] && ok[4 * h + 3]) {
                *reinterpret_cast<float4*>(r + e0) =
                    make_float4(out[4 * h], out[4 * h + 1], out[4 * h + 2], out[4 * h + 3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (ok[4 * h + e]) r[e0 + e] = out[4 * h + e];
            }
        }
        carry = next_carry;
        __syncthreads();   // warp_maps / carry_in are reused by the next chunk
    }
}

// ---------------------------------------------------------------------------
// Chunked form for few, long sequences.  The token axis of every draw row is
// cut into fixed chunks of kScanChunk tokens, each scanned by its own CTA.
// Element t carries the map x -> c_t + g_t x with g_t = gamma inside a
// sequence and g_t = 0 at a sequence's last token, so sequence boundaries
// inside a chunk need no special case.  Pass 1 composes each chunk's map,
// pass 2 (one thread per draw row) walks the chunk maps from the end of the
// row to get every chunk's incoming carry (r at the next chunk's first
// token), pass 3 rescans each chunk with its carry and writes r.  c is read
// twice (12 bytes per draw x token instead of 8) in exchange for
// parallelism over the whole token axis.

// Index of the first offset greater than t (offsets clamped into [0, T]).
__device__ __forceinline__ int first_offset_above(const int32_t* offs, int n_seq, int T, int t) {
    int lo = 0, hi = n_seq;                       // search offs[0 .. n_seq]
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (clamp_int(__ldg(offs + mid), 0, T) > t) hi = mid;
        else lo = mid + 1;
    }
    return lo;                                    // n_seq + 1 if none
}

template <bool WRITE>
__global__ void __launch_bounds__(kScanThreads)
reward_scan_chunks_kernel(const float* c, float* r, int T, int n_chunks, const int32_t* __restrict__ offs,
                          int n_seq, float gamma, float2* __restrict__ maps, const float* __restrict__ carries) {
    __shared__ Affine warp_maps[kScanThreads / 32];
    __shared__ float carry_in[kScanThreads / 32];
    const long long blk = blockIdx.x;
    const int j = static_cast<int>(blk % n_chunks);
    const long long row = (blk / n_chunks) * static_cast<long long>(T);
    const int t_begin = j * kScanChunk;
    const int t_end = min(T, t_begin + kScanChunk);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // my 8 tokens: t_begin + 8 * tid .. + 7 (within the chunk)
    const int t0 = t_begin + kScanVec * threadIdx.x;
    float v[kScanVec], gm[kScanVec];
    bool ok[kScanVec];
    int idx = first_offset_above(offs, n_seq, T, t0);          // next boundary after t0
#pragma unroll
    for (int e = 0; e < kScanVec; ++e) {
        const int t = t0 + e;
        ok[e] = t < t_end;
        v[e] = ok[e] ? c[row + t] : 0.0f;
        // t is the last token of its sequence iff some offset equals t + 1
        while (idx <= n_seq && clamp_int(__ldg(offs + idx), 0, T) <= t) ++idx;
        const bool last = idx <= n_seq && clamp_int(__ldg(offs + idx), 0, T) == t + 1;
        gm[e] = last ? 0.0f : gamma;
    }
    Affine m = {1.0f, 0.0f};
#pragma unroll
    for (int e = kScanVec - 1; e >= 0; --e)
        if (ok[e]) m = {gm[e] * m.a, __fmaf_rn(gm[e], m.b, v[e])};
    Affine s = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        Affine t;
        t.a = __shfl_down_sync(0xffffffffu, s.a, o);
        t.b = __shfl_down_sync(0xffffffffu, s.b, o);
        if (lane + o < 32) s = compose(s, t);
    }
    if (lane == 0) warp_maps[warp] = s;
    __syncthreads();
    const float carry = WRITE ? carries[blk] : 0.0f;
    if (threadIdx.x == 0) {
        float x = carry;
        Affine total = {1.0f, 0.0f};
        for (int w = kScanThreads / 32 - 1; w >= 0; --w) {
            carry_in[w] = x;
            x = __fmaf_rn(warp_maps[w].a, x, warp_maps[w].b);
            total = compose(warp_maps[w], total);
        }
        if (!WRITE) maps[blk] = make_float2(total.a, total.b);
    }
    if (!WRITE) return;
    __syncthreads();
    Affine after;
    after.a = __shfl_down_sync(0xffffffffu, s.a, 1);
    after.b = __shfl_down_sync(0xffffffffu, s.b, 1);
    if (lane == 31) after = {1.0f, 0.0f};
    float x = __fmaf_rn(after.a, carry_in[warp], after.b);
#pragma unroll
    for (int e = kScanVec - 1; e >= 0; --e) {
        if (!ok[e]) continue;
        x = __fmaf_rn(gm[e], x, v[e]);
        r[row + t0 + e] = x;
    }
}

// One thread per draw row: carries[row][j] = r at the first token of chunk j + 1.
__global__ void reward_scan_carries_kernel(const float2* __restrict__ maps, int K, int n_chunks,
                                           float* __restrict__ carries) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= K) return;
    float x = 0.0f;
    for (int j = n_chunks - 1; j >= 0; --j) {
        const size_t k = static_cast<size_t>(i) * n_chunks + j;
        carries[k] = x;
        const float2 mj = maps[k];
        x = __fmaf_rn(mj.x, x, mj.y);
    }
}

}  // namespace

size_t reward_scan_chunks_workspace(int K, int T) {
    const size_t n = static_cast<size_t>(K) * static_cast<size_t>(ceil_div(T, kScanChunk));
    return n * (sizeof(float2) + sizeof(float));
}

bool reward_scan_prefers_chunks(int K, int T, int n_seq) {
    // the per-sequence kernel has K * n_seq CTAs; prefer chunks when that
    // leaves the SMs idle and sequences span several chunks
    return static_cast<long long>(K) * n_seq < 4LL * kNumSMs && T / n_seq > kScanChunk;
}

cudaError_t launch_reward_scan_chunks(const float* c, float* r, int K, int T, const int32_t* offs, int n_seq,
                                      float gamma, void* scratch, cudaStream_t stream) {
    if (K == 0 || T == 0) return cudaSuccess;
    if (gamma == 0.0f) {
        if (r == c) return cudaSuccess;
        return cudaMemcpyAsync(r, c, sizeof(float) * static_cast<size_t>(K) * T, cudaMemcpyDeviceToDevice, stream);
    }
    const int n_chunks = static_cast<int>(ceil_div(T, kScanChunk));
    const long long blocks = static_cast<long long>(K) * n_chunks;
    auto* maps = static_cast<float2*>(scratch);
    float* carries = reinterpret_cast<float*>(maps + blocks);
    reward_scan_chunks_kernel<false><<<static_cast<unsigned>(blocks), kScanThreads, 0, stream>>>(
        c, r, T, n_chunks, offs, n_seq, gamma, maps, carries);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    reward_scan_carries_kernel<<<static_cast<unsigned>(ceil_div(K, 128)), 128, 0, stream>>>(maps, K, n_chunks, carries);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    reward_scan_chunks_kernel<true><<<static_cast<unsigned>(blocks), kScanThreads, 0, stream>>>(
        c, r, T, n_chunks, offs, n_seq, gamma, maps, carries);
    return cudaGetLastError();
}

cudaError_t launch_reward_scan(const float* c, float* r, int K, int T, const int32_t* offs,
                               int n_seq, float gamma, cudaStream_t stream) {
    if (K == 0 || T == 0) return cudaSuccess;
    if (gamma == 0.0f) {   // 0^0 = 1: r = c bit for bit
        if (r == c) return cudaSuccess;
        return cudaMemcpyAsync(r, c, sizeof(float) * static_cast<size_t>(K) * T,
                               cudaMemcpyDeviceToDevice, stream);
    }
    const long long segs = static_cast<long long>(K) * n_seq;
    const long long total = static_cast<long long>(K) * T;
    // gridDim.x allows 2^31 - 1 blocks
    reward_scan_kernel<<<static_cast<unsigned>(segs), kScanThreads, 0, stream>>>(c, r, total, T, offs,
                                                                                  n_seq, gamma);
    return cudaGetLastError();
}

}  // namespace dust
