// tuner.cu -- support for choosing sigma by the cosine criterion.
//
// cnblogs Dust explainer, section "真正的工作量：压住干扰" (last paragraph): the
// cheap way to set the hyper-parameters is to maximise, on a single batch, the
// cosine similarity between the Dust estimate and the backprop gradient;
// section "梯度是"长"出来的": that cosine follows cos(K) = c_max/sqrt(1 + c/K).
// For the LM head the backprop gradient has a closed form,
//   grad_W sum_t l_t = sum_t (softmax(z_t) - e_{y_t}) x_t^T,
// so the comparator runs in this library too: a kernel forms
// D = softmax(Z) - onehot(y) (bf16 or fp32, as the GEMM wants) and the weight-
// estimate GEMM forms D^T X.  The cosine is a fixed-order two-pass reduction
// in double.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace dust {

namespace {

template <bool BF16>
__global__ void softmax_minus_onehot_kernel(const float* __restrict__ Z, const float* __restrict__ lse,
                                            const int32_t* __restrict__ targets, int T, int V, void* __restrict__ D) {
    const long long total = static_cast<long long>(T) * V;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / V), v = static_cast<int>(i % V);
        float d = expf(__ldg(Z + i) - __ldg(lse + t));
        if (v == clamp_int(__ldg(targets + t), 0, V - 1)) d -= 1.0f;
        if (BF16) static_cast<__nv_bfloat16*>(D)[i] = __float2bfloat16_rn(d);
        else static_cast<float*>(D)[i] = d;
    }
}

constexpr int kCosThreads = 256;
constexpr int kCosBlocks = 4 * 148;

__global__ void __launch_bounds__(kCosThreads)
cosine_partial_kernel(const float* __restrict__ a, const float* __restrict__ b, long long n, double* __restrict__ part) {
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const double x = __ldg(a + i), y = __ldg(b + i);
        ab += x * y;
        aa += x * x;
        bb += y * y;
    }
    __shared__ double s[3][kCosThreads];
    s[0][threadIdx.x] = ab;
    s[1][threadIdx.x] = aa;
    s[2][threadIdx.x] = bb;
    __syncthreads();
    for (int w = kCosThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            for (int k = 0; k < 3; ++k) s[k][threadIdx.x] += s[k][threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x < 3) part[blockIdx.x * 3 + threadIdx.x] = s[threadIdx.x][0];
}

__global__ void cosine_final_kernel(const double* __restrict__ part, int nblocks, double* __restrict__ out) {
    if (threadIdx.x != 0) return;
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (int i = 0; i < nblocks; ++i) {
        ab += part[3 * i];
        aa += part[3 * i + 1];
        bb += part[3 * i + 2];
    }
    out[0] = ab;
    out[1] = aa;
    out[2] = bb;
    out[3] = (aa > 0.0 && bb > 0.0) ? ab / (sqrt(aa) * sqrt(bb)) : 0.0;
}

}  // namespace

cudaError_t launch_softmax_minus_onehot(const float* Z, const float* lse, const int32_t* targets, int T, int V,
                                        void* D, bool bf16, cudaStream_t stream) {
    const long long total = static_cast<long long>(T) * V;
    const long long blocks = ceil_div(total, 256);
    const unsigned g = static_cast<unsigned>(blocks < 8 * 1184 ? blocks : 8 * 1184);
    if (bf16) softmax_minus_onehot_kernel<true><<<g, 256, 0, stream>>>(Z, lse, targets, T, V, D);
    else softmax_minus_onehot_kernel<false><<<g, 256, 0, stream>>>(Z, lse, targets, T, V, D);
    return cudaGetLastError();
}

size_t cosine_partial_bytes() { return sizeof(double) * 3 * kCosBlocks; }

cudaError_t launch_cosine(const float* a, const float* b, long long n, double* part, double* out,
                          cudaStream_t stream) {
    cosine_partial_kernel<<<kCosBlocks, kCosThreads, 0, stream>>>(a, b, n, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cosine_final_kernel<<<1, 32, 0, stream>>>(part, kCosBlocks, out);
    return cudaGetLastError();
}

}  // namespace dust
