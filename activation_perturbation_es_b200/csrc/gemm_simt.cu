// gemm_simt.cu -- fp32 CUDA-core GEMM for the small fp32 workloads, plus the
// fixed-order split-K reduction and the fp32 -> bf16 conversion shared by the
// GEMM paths.
//
// Used for a6 (G_W = g^T X, cnblogs Dust explainer, credit-assignment section,
// weight equation) and a2 (clean logits Z = X W^T) when the operands are fp32.
// 64 x 64 output tiles, 16-deep k steps staged in shared memory, 4 x 4 outputs
// per thread; optional split over k with partial tiles reduced in a fixed
// order, so the result does not depend on the launch.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dust {

namespace {

constexpr int kTile = 64, kStep = 16;

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_as_float<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

// A and B may differ in type (fp32 or bf16): every element is widened to fp32
// exactly before the fp32 products.
template <typename TA, typename TB, bool AK, bool BK>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const TA* __restrict__ A, int lda, const TB* __restrict__ B, int ldb, int M, int N,
                 int K, int k_per_split, float* __restrict__ C, int ldc, int accumulate,
                 float* __restrict__ partial) {
    __shared__ float As[kStep][kTile + 4];
    __shared__ float Bs[kStep][kTile + 4];
    const int m0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
    const int kb = blockIdx.z * k_per_split;
    const int ke = min(K, kb + k_per_split);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = kb; k0 < ke; k0 += kStep) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = threadIdx.x + 256 * i;
            int m, k;
            if (AK) { m = e / kStep; k = e % kStep; } else { m = e % kTile; k = e / kTile; }
            const int gm = m0 + m, gk = k0 + k;
            float v = 0.0f;
            if (gm < M && gk < ke) v = load_as_float(AK ? A + static_cast<size_t>(gm) * lda + gk
                                                         : A + static_cast<size_t>(gk) * lda + gm);
            As[k][m] = v;
            int n, kk;
            if (BK) { n = e / kStep; kk = e % kStep; } else { n = e % kTile; kk = e / kTile; }
            const int gn = n0 + n, gk2 = k0 + kk;
            float w = 0.0f;
            if (gn < N && gk2 < ke) w = load_as_float(BK ? B + static_cast<size_t>(gn) * ldb + gk2
                                                          : B + static_cast<size_t>(gk2) * ldb + gn);
            Bs[kk][n] = w;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kStep; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = As[k][ty * 4 + i]; b[i] = Bs[k][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gm = m0 + ty * 4 + i;
        if (gm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gn = n0 + tx * 4 + j;
            if (gn >= N) continue;
            if (partial) {
                partial[(static_cast<size_t>(blockIdx.z) * M + gm) * N + gn] = acc[i][j];
            } else {
                float* cp = C + static_cast<size_t>(gm) * ldc + gn;
                *cp = accumulate ? *cp + acc[i][j] : acc[i][j];
            }
        }
    }
}

__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N,
                                     float* __restrict__ C, int ldc, int accumulate) {
    const long long total = static_cast<long long>(M) * N;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        float s = 0.0f;
        for (int p = 0; p < splits; ++p) s += partial[static_cast<size_t>(p) * total + idx];
        const int m = static_cast<int>(idx / N), n = static_cast<int>(idx % N);
        float* cp = C + static_cast<size_t>(m) * ldc + n;
        *cp = accumulate ? *cp + s : s;
    }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

template <typename TA, typename TB>
cudaError_t launch_typed(const TA* A, bool ak, int lda, const TB* B, bool bk, int ldb, int M, int N, int K,
                         float* C, int ldc, int accumulate, float* partial, int splits, cudaStream_t st) {
    const int kps = static_cast<int>(ceil_div(ceil_div(K, splits), kStep) * kStep);
    const dim3 grid(static_cast<unsigned>(ceil_div(N, kTile)), static_cast<unsigned>(ceil_div(M, kTile)),
                    static_cast<unsigned>(splits));
    float* part = splits > 1 ? partial : nullptr;
#define DUST_SIMT_LAUNCH(AKV, BKV) \
    gemm_simt_kernel<TA, TB, AKV, BKV><<<grid, 256, 0, st>>>(A, lda, B, ldb, M, N, K, kps, C, ldc, accumulate, part)
    if (ak && bk) DUST_SIMT_LAUNCH(true, true);
    else if (ak && !bk) DUST_SIMT_LAUNCH(true, false);
    else if (!ak && bk) DUST_SIMT_LAUNCH(false, true);
    else DUST_SIMT_LAUNCH(false, false);
#undef DUST_SIMT_LAUNCH
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || splits == 1) return e;
    return launch_splitk_reduce(partial, splits, M, N, C, ldc, accumulate, st);
}

}  // namespace

int gemm_simt_splits(int M, int N, int K) {
    const long long tiles = ceil_div(M, kTile) * ceil_div(N, kTile);
    long long s = ceil_div(2 * kNumSMs, tiles);
    const long long kmax = ceil_div(K, 256);       // at least 256 k per slice
    if (s > kmax) s = kmax;
    if (s < 1) s = 1;
    if (s > 64) s = 64;
    return static_cast<int>(s);
}

cudaError_t launch_gemm_simt(const void* A, bool a_kmajor, int lda, const void* B, bool b_kmajor, int ldb,
                             dust_dtype dt, int M, int N, int K, float* C, int ldc, int accumulate,
                             float* partial, int splits, cudaStream_t stream) {
    return launch_gemm_simt_mixed(A, dt, a_kmajor, lda, B, dt, b_kmajor, ldb, M, N, K, C, ldc, accumulate, partial,
                                  splits, stream);
}

cudaError_t launch_gemm_simt_mixed(const void* A, dust_dtype a_dt, bool a_kmajor, int lda, const void* B,
                                   dust_dtype b_dt, bool b_kmajor, int ldb, int M, int N, int K, float* C, int ldc,
                                   int accumulate, float* partial, int splits, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const auto* af = static_cast<const float*>(A);
    const auto* ab = static_cast<const bf*>(A);
    const auto* bf32 = static_cast<const float*>(B);
    const auto* bb = static_cast<const bf*>(B);
    if (a_dt == DUST_F32 && b_dt == DUST_F32)
        return launch_typed(af, a_kmajor, lda, bf32, b_kmajor, ldb, M, N, K, C, ldc, accumulate, partial, splits,
                            stream);
    if (a_dt == DUST_F32)
        return launch_typed(af, a_kmajor, lda, bb, b_kmajor, ldb, M, N, K, C, ldc, accumulate, partial, splits,
                            stream);
    if (b_dt == DUST_F32)
        return launch_typed(ab, a_kmajor, lda, bf32, b_kmajor, ldb, M, N, K, C, ldc, accumulate, partial, splits,
                            stream);
    return launch_typed(ab, a_kmajor, lda, bb, b_kmajor, ldb, M, N, K, C, ldc, accumulate, partial, splits, stream);
}

cudaError_t launch_splitk_reduce(const float* partial, int splits, int M, int N, float* C, int ldc,
                                 int accumulate, cudaStream_t stream) {
    const long long total = static_cast<long long>(M) * N;
    const long long blocks = ceil_div(total, 256);
    splitk_reduce_kernel<<<static_cast<unsigned>(blocks < 4 * 1184 ? blocks : 4 * 1184), 256, 0, stream>>>(
        partial, splits, M, N, C, ldc, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float* src, void* dst, size_t n, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n + 255) / 256;
    to_bf16_kernel<<<static_cast<unsigned>(blocks < 8 * 1184 ? blocks : 8 * 1184), 256, 0, stream>>>(
        src, static_cast<__nv_bfloat16*>(dst), n);
    return cudaGetLastError();
}

}  // namespace dust
