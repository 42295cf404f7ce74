// toy_suffix.cu -- harness: a small causal suffix that scores the draws of a
// perturbed hidden linear layer (produces the per-token losses behind c_s).
//
// cnblogs Dust explainer, section "真正的工作量：压住干扰", first measure: the
// draws of a block rerun the network from that block on, on top of the cached
// clean forward.  The pages give no model; this library's reading is the
// smallest suffix in which a token's noise reaches later tokens:
//   y~ = Y + sigma a,  q,k,v = y~ W{q,k,v}^T,  o_t = causal softmax attention
//   inside the sequence (scores / sqrt(dh)),  h = y~ + o Wo^T,  z = h Wout^T,
//   loss_t = logsumexp(z_t) - z_t[target_t].
// fp32 on CUDA cores, batched over draws; not part of the graded hot path.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "noise.cuh"

namespace dust {

namespace {

// rows [b][t][j]: Y + sigma a(draw_of[b], tok0 + t, j), or Y for the clean row
__global__ void perturb_kernel(const float* __restrict__ Y, int T, int d, uint32_t seed, uint32_t layer,
                               uint32_t tok0, uint32_t first_draw, int clean_first, int nb, float sigma,
                               float* __restrict__ out) {
    const int nq = d / 4;
    const long long total = static_cast<long long>(nb) * T * nq;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int q = static_cast<int>(idx % nq);
        const long long rest = idx / nq;
        const int t = static_cast<int>(rest % T);
        const int b = static_cast<int>(rest / T);
        float4 y = __ldg(reinterpret_cast<const float4*>(Y + static_cast<size_t>(t) * d) + q);
        if (!(clean_first && b == 0)) {
            const uint32_t draw = first_draw + static_cast<uint32_t>(b - clean_first);
            const float4 a = gauss4(seed, layer, draw, tok0 + static_cast<uint32_t>(t), static_cast<uint32_t>(q), 0);
            y.x += sigma * a.x; y.y += sigma * a.y; y.z += sigma * a.z; y.w += sigma * a.w;
        }
        reinterpret_cast<float4*>(out + static_cast<size_t>(b * static_cast<long long>(T) + t) * d)[q] = y;
    }
}

// One warp per (batch row, token): online softmax over the token's causal
// prefix inside its sequence, in chunks of 32 keys (one key per lane).
// q, k, v are [nb][T][dh] with a batch stride each (0: shared by the batch).
__global__ void __launch_bounds__(256)
causal_attention_kernel(const float* __restrict__ qa, const float* __restrict__ ka, const float* __restrict__ va,
                        long long q_bs, long long k_bs, long long v_bs, int nb, int T, int dh,
                        const int32_t* __restrict__ offs, int n_seq, float scale, float* __restrict__ o) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.x * 8LL + warp;
    if (row >= static_cast<long long>(nb) * T) return;
    const int t = static_cast<int>(row % T);
    const long long b = row / T;
    const float* q = qa + b * q_bs;
    const float* k = ka + b * k_bs;
    const float* v = va + b * v_bs;
    // sequence of t (offsets clamped; linear search is fine for a harness)
    int s0 = 0;
    for (int sq = 0; sq < n_seq; ++sq) {
        const int2 sb = seq_bounds(offs, sq, T);
        if (t >= sb.x && t < sb.y) { s0 = sb.x; break; }
    }
    const float* qt = q + static_cast<long long>(t) * dh;
    float m = -INFINITY, l = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};   // channels lane + 32 e, dh <= 128
    for (int u0 = s0; u0 <= t; u0 += 32) {
        const int u = u0 + lane;
        float sc = -INFINITY;
        if (u <= t) {
            const float* ku = k + static_cast<long long>(u) * dh;
            float s = 0.0f;
            for (int e = 0; e < dh; ++e) s = fmaf(__ldg(qt + e), __ldg(ku + e), s);
            sc = s * scale;
        }
        const float mc = warp_max(sc);
        const float mn = fmaxf(m, mc);
        const float corr = m == -INFINITY ? 0.0f : expf(m - mn);
        const float p = u <= t ? expf(sc - mn) : 0.0f;
        l = l * corr + warp_sum(p);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] *= corr;
        const int n_keys = min(32, t - u0 + 1);
        for (int j = 0; j < n_keys; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
            const float* vu = v + static_cast<long long>(u0 + j) * dh;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (lane + 32 * e < dh) acc[e] = fmaf(pj, __ldg(vu + lane + 32 * e), acc[e]);
        }
        m = mn;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if (lane + 32 * e < dh) o[row * dh + lane + 32 * e] = acc[e] / l;
}

__global__ void ce_rows_kernel(const float* __restrict__ z, const int32_t* __restrict__ targets, long long rows,
                               int T, int V, float* __restrict__ loss) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.x * 8LL + warp;
    if (row >= rows) return;
    const float* zr = z + row * V;
    float m = -INFINITY;
    for (int c = lane; c < V; c += 32) m = fmaxf(m, __ldg(zr + c));
    m = warp_max(m);
    float s = 0.0f;
    for (int c = lane; c < V; c += 32) s += expf(__ldg(zr + c) - m);
    s = warp_sum(s);
    if (lane == 0) {
        const int t = static_cast<int>(row % T);
        loss[row] = m + logf(s) - zr[clamp_int(targets[t], 0, V - 1)];
    }
}

__global__ void diff_kernel(const float* __restrict__ loss, long long n, int T, float* __restrict__ c) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        c[i] = loss[T + i] - loss[i % T];
}

}  // namespace

cudaError_t launch_causal_attention(const float* q, const float* k, const float* v, long long q_bs, long long k_bs,
                                    long long v_bs, int nb, int T, int dh, const int32_t* offs, int n_seq,
                                    float* o, cudaStream_t stream) {
    const long long rows = static_cast<long long>(nb) * T;
    causal_attention_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, stream>>>(
        q, k, v, q_bs, k_bs, v_bs, nb, T, dh, offs, n_seq, 1.0f / std::sqrt(static_cast<float>(dh)), o);
    return cudaGetLastError();
}

namespace {

unsigned blocks_for(long long n, int per) {
    const long long b = ceil_div(n, per);
    return static_cast<unsigned>(b < 16 * 1184 ? b : 16 * 1184);
}

}  // namespace

namespace {

int toy_suffix_batch(int draw_count) { return draw_count + 1 < 16 ? draw_count + 1 : 16; }

struct ToyLayout {
    size_t yt, q, k, v, o, z, part, total;
    int nb;
};

ToyLayout toy_layout(int draw_count, int T, int d, int dh, int V) {
    ToyLayout L{};
    L.nb = toy_suffix_batch(draw_count);
    const size_t rows = static_cast<size_t>(L.nb) * T;
    size_t off = kStatusBytes;
    auto add = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 256); return o; };
    L.yt = add(sizeof(float) * rows * d);
    L.q = add(sizeof(float) * rows * dh);
    L.k = add(sizeof(float) * rows * dh);
    L.v = add(sizeof(float) * rows * dh);
    L.o = add(sizeof(float) * rows * dh);
    L.z = add(sizeof(float) * rows * V);
    const int M = static_cast<int>(rows);
    size_t part = 0;
    const int shapes[4][3] = {{M, dh, d}, {M, d, dh}, {M, V, d}, {M, dh, d}};
    for (auto& s : shapes) {
        const int sp = gemm_simt_splits(s[0], s[1], s[2]);
        if (sp > 1) part = std::max(part, sizeof(float) * static_cast<size_t>(sp) * s[0] * s[1]);
    }
    L.part = add(part);
    L.total = off;
    return L;
}

}  // namespace

size_t toy_suffix_workspace_bytes(int draw_count, int T, int d, int dh, int V) {
    return toy_layout(draw_count, T, d, dh, V).total;
}

cudaError_t run_toy_suffix(const float* Y, int T, int d, const int32_t* offs, int n_seq, const float* Wq,
                           const float* Wk, const float* Wv, const float* Wo, int dh, const float* Wout, int V,
                           const int32_t* targets, const dust_noise& nz, float* loss, float* c, void* ws,
                           cudaStream_t st) {
    const ToyLayout L = toy_layout(static_cast<int>(nz.draw_count), T, d, dh, V);
    auto* base = static_cast<uint8_t*>(ws);
    float* yt = reinterpret_cast<float*>(base + L.yt);
    float* q = reinterpret_cast<float*>(base + L.q);
    float* k = reinterpret_cast<float*>(base + L.k);
    float* v = reinterpret_cast<float*>(base + L.v);
    float* o = reinterpret_cast<float*>(base + L.o);
    float* z = reinterpret_cast<float*>(base + L.z);
    float* part = reinterpret_cast<float*>(base + L.part);
    const int rows_total = static_cast<int>(nz.draw_count) + 1;   // clean + draws
    cudaError_t e = cudaSuccess;
    for (int r0 = 0; r0 < rows_total && e == cudaSuccess; r0 += L.nb) {
        const int nb = std::min(L.nb, rows_total - r0);
        const int clean_first = r0 == 0 ? 1 : 0;
        const uint32_t first_draw = nz.draw_begin + static_cast<uint32_t>(r0 == 0 ? 0 : r0 - 1);
        const long long rows = static_cast<long long>(nb) * T;
        const int M = static_cast<int>(rows);
        perturb_kernel<<<blocks_for(rows * (d / 4), 256), 256, 0, st>>>(Y, T, d, nz.seed, nz.layer, nz.token_begin,
                                                                          first_draw, clean_first, nb, nz.sigma, yt);
        if ((e = cudaGetLastError()) != cudaSuccess) break;
        const float* Ws[3] = {Wq, Wk, Wv};
        float* outs[3] = {q, k, v};
        for (int w = 0; w < 3 && e == cudaSuccess; ++w)
            e = launch_gemm_simt(yt, true, d, Ws[w], true, d, DUST_F32, M, dh, d, outs[w], dh, 0, part,
                                 gemm_simt_splits(M, dh, d), st);
        if (e != cudaSuccess) break;
        const long long bs = static_cast<long long>(T) * dh;
        if ((e = launch_causal_attention(q, k, v, bs, bs, bs, nb, T, dh, offs, n_seq, o, st)) != cudaSuccess) break;
        // h = y~ + o Wo^T, in place over y~
        e = launch_gemm_simt(o, true, dh, Wo, true, dh, DUST_F32, M, d, dh, yt, d, 1, part,
                             gemm_simt_splits(M, d, dh), st);
        if (e != cudaSuccess) break;
        e = launch_gemm_simt(yt, true, d, Wout, true, d, DUST_F32, M, V, d, z, V, 0, part,
                             gemm_simt_splits(M, V, d), st);
        if (e != cudaSuccess) break;
        ce_rows_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, st>>>(
            z, targets, rows, T, V, loss + static_cast<size_t>(r0) * T);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && c != nullptr) {
        const long long n = static_cast<long long>(nz.draw_count) * T;
        diff_kernel<<<blocks_for(n, 256), 256, 0, st>>>(loss, n, T, c);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace dust
