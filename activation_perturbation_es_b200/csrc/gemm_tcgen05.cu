// gemm_tcgen05.cu -- bf16 x bf16 -> fp32 GEMM on the 5th-generation tensor
// cores (tcgen05.mma, accumulator in TMEM), operands staged by TMA.
//
// Serves a6, the weight estimate G_W = g^T X (cnblogs Dust explainer, credit-
// assignment section, weight equation: the same outer product with the same
// input as backprop), and a2, the clean head logits Z = X W^T.
//   a6: C[d_out][d_in] = sum_t g[t][o] X[t][i]: both operands are MN-major
//       (the reduction index t is the row index of both tensors);
//   a2: C[T][V] = sum_k X[t][k] W[v][k]: both operands are K-major.
//
// Tile 128 x BN (BN in {64, 128, 256}), 64-deep k blocks in a 4-stage ring.
// The kernel is persistent: one CTA of 10 warps per SM walks the work units
// (output tile, k slice) in a grid-stride loop, and the roles are split by warp:
//   warp 0, one lane: TMA producer (cp.async.bulk.tensor, 128-byte swizzle,
//           each CTA loads its own tiles into its own shared memory), one
//           mbarrier per stage with the expected bytes;
//   warp 1, one lane: MMA issuer, 4 x tcgen05.mma (M = 128, N = BN, K = 16)
//           per stage, tcgen05.commit frees the stage; warp 1 also allocates
//           and frees TMEM: two BN-column fp32 accumulators (2 BN columns), so
//           that unit i's epilogue overlaps unit i+1's main loop;
//   warps 2-9: epilogue, two warps per TMEM lane quarter taking alternate
//           32-column blocks: tcgen05.ld of the warp's 32 TMEM lanes (rows)
//           into registers, then the block into shared memory in the TMA's
//           128-byte-swizzled layout (eight conflict-free 16-byte stores per
//           lane) and one TMA store of the 32 x 32 block (C, or the split's
//           partial slab through a 3-D map); the tensor map clips ragged edges.
//           When C is accumulated into, the TMA adds the block into C (one
//           fp32 addition per element, as C + x).  When C's row pitch is not a
//           multiple of 16 bytes, the block goes through an xor-swizzled shared
//           transpose to row-segment fp32 stores instead.  The warps release the accumulator
//           buffer once its columns are in registers.
// Split over k writes fp32 partial tiles that a second kernel sums in a fixed
// order (deterministic).  Every mbarrier wait is bounded: when a bound runs
// out the role records the workspace status word, raises the CTA's abort flag
// (which ends the other roles' waits), drains its own copies and MMAs
// (bounded too), frees TMEM and returns.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace dust {

namespace {

using namespace tc;

constexpr int kBM = 128;
constexpr int kBK = 64;          // bf16 elements = 128 bytes = one swizzle row
constexpr int kStages = 4;
// Instruction descriptor, kind::f16: fp32 accumulator (bits [4,6) = 1), A and
// B bf16 (bits [7,10) = 1, [10,13) = 1), A/B major (bit 15/16: 1 = MN-major),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t instr_desc(int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(kBM >> 4) << 24);
}

template <int BN>
struct Smem {
    static constexpr int kABytes = kBM * kBK * 2;   // 16 KB
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kEpiBytes = 8 * 32 * 32 * 4;   // per epilogue warp: a 32 x 32 fp32 tile (xor-swizzled)
    static constexpr int kBytes = kStages * kStageBytes + kEpiBytes + 1024 /*align*/ + 256 /*barriers*/;
};

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag) {
    for (uint32_t it = 0; it < kWaitLimit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (it > 64) __nanosleep(256);
    }
    return false;
}

struct Unit {       // one output tile and k slice
    int m0, n0, kb, nk;
};

__device__ __forceinline__ Unit unit_of(int u, int tiles_m, int tiles_n, int BN, int K, int k_per_split) {
    Unit w;
    const int n_t = u % tiles_n;
    const int rest = u / tiles_n;
    const int m_t = rest % tiles_m;
    const int split = rest / tiles_m;
    w.m0 = m_t * kBM;
    w.n0 = n_t * BN;
    w.kb = split * k_per_split;
    const int ke = min(K, w.kb + k_per_split);
    w.nk = ke > w.kb ? (ke - w.kb + kBK - 1) / kBK : 0;
    return w;
}

constexpr int kEpiWarps = 8;                          // two per TMEM lane quarter
// how the epilogue writes a 32 x 32 block: generic stores after a shared
// transpose; a TMA store into C ([M][N], 2-D map); a TMA store into the
// split's partial slab ([splits][M][N], 3-D map); a TMA reduce-add into C
constexpr int kStoreGeneric = 0, kStoreC = 1, kStorePartial = 2, kAddC = 3;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;     // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue

// Persistent, warp-specialised: every CTA walks the work units (tile, k
// slice) u = blockIdx.x, blockIdx.x + gridDim.x, ...  Two TMEM accumulators
// of BN columns let the epilogue of one unit overlap the mainloop of the
// next.  A: K-major (rows m, 128-byte K rows) or MN-major (two 64-wide MN
// atoms of 64 K rows each); B likewise with BN rows / BN/64 atoms.
template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, int store_mode, int M, int N, int K, int k_per_split,
               int splits, float* __restrict__ C, int ldc, int accumulate, float* __restrict__ partial,
               uint32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using S = Smem<BN>;
    float* epi = reinterpret_cast<float*>(smem + kStages * S::kStageBytes);   // [8 warps][32][32]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * S::kStageBytes + S::kEpiBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;       // [2] accumulator ready for the epilogue
    uint64_t* tempty = tfull + 2;            // [2] accumulator drained by the epilogue
    uint64_t* drain = tempty + 2;            // MMAs in flight at an abort
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + kBM - 1) / kBM, tiles_n = (N + BN - 1) / BN;
    const int units = tiles_m * tiles_n * splits;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_slot, 2 * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const Unit w = unit_of(u, tiles_m, tiles_n, BN, K, k_per_split);
                for (int kk = 0; kk < w.nk; ++kk, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait_or_abort(&empty[s], ((it / kStages) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + s * S::kStageBytes;
                    uint8_t* sb = sa + S::kABytes;
                    mbar_arrive_expect_tx(&full[s], S::kStageBytes);
                    const int k0 = w.kb + kk * kBK;
                    if (A_MN) {
                        tma_load_2d(sa, &map_a, &full[s], w.m0, k0);
                        tma_load_2d(sa + 64 * kBK * 2, &map_a, &full[s], w.m0 + 64, k0);
                    } else {
                        tma_load_2d(sa, &map_a, &full[s], k0, w.m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int h = 0; h < BN / 64; ++h)
                            tma_load_2d(sb + h * 64 * kBK * 2, &map_b, &full[s], w.n0 + 64 * h, k0);
                    } else {
                        tma_load_2d(sb, &map_b, &full[s], k0, w.n0);
                    }
                }
            }
            if (!ok) {
                atomicExch(status, kStatusTimeout);
                *abort_flag = 1;
            }
            // the last (up to kStages) loads must land before the CTA exits
            for (int j = it > kStages ? it - kStages : 0; j < it; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            constexpr uint32_t idesc = instr_desc(BN, A_MN, B_MN);
            int it = 0, tcount = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tcount) {
                const Unit w = unit_of(u, tiles_m, tiles_n, BN, K, k_per_split);
                const int buf = tcount & 1;
                if (tcount >= 2 && !mbar_wait_or_abort(&tempty[buf], ((tcount >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + static_cast<uint32_t>(buf * BN);
                for (int kk = 0; kk < w.nk; ++kk, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait_or_abort(&full[s], (it / kStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * S::kStageBytes);
                    const uint32_t sb = sa + S::kABytes;
#pragma unroll
                    for (int j = 0; j < kBK / 16; ++j) {
                        // K-major: a 16-element k step is 32 bytes along the swizzled row;
                        // MN-major: it is 16 rows of 128 bytes.
                        const uint64_t ad = A_MN ? smem_desc(sa + j * 16 * 128, 64 * kBK * 2, 1024)
                                                 : smem_desc(sa + j * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc(sb + j * 16 * 128, 64 * kBK * 2, 1024)
                                                 : smem_desc(sb + j * 32, 16, 1024);
                        tc_mma(acc, ad, bd, idesc, (kk > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(&tfull[buf]);   // arrives once this unit's MMAs have completed
            }
            if (!ok) {
                atomicExch(status, kStatusTimeout);
                *abort_flag = 1;
            }
            tc_commit(drain);             // every MMA issued above has completed when this arrives
            mbar_wait(drain, 0);
        }
    } else {
        // ---------------- epilogue: TMEM -> registers -> global (warps 2-9)
        const int quarter = warp & 3;     // the TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2; // the two warps of a quarter take alternate 32-column blocks
        int tcount = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++tcount) {
            const Unit w = unit_of(u, tiles_m, tiles_n, BN, K, k_per_split);
            const int buf = tcount & 1;
            bool have = mbar_wait_or_abort(&tfull[buf], (tcount >> 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, have)) {
                // this unit's tile stays unwritten: record it (another role may
                // have done so already; the word and the flag only ever get set)
                if (lane == 0) {
                    atomicExch(status, kStatusTimeout);
                    *abort_flag = 1;
                }
                break;
            }
            tc_fence_after();
            have = w.nk > 0;
            const int split = u / (tiles_m * tiles_n);
            // Each 32 x 32 block (this warp's 32 rows x 32 columns) goes through the
            // warp's 4 KB shared buffer: in the TMA's swizzled layout for a bulk
            // store, or xor-swizzled and transposed (lane l then holds column
            // c0 + l of every row) for row-segment stores.
            float* tile = epi + (warp - 2) * (32 * 32);
            const int row0 = w.m0 + quarter * 32;
            float* base = partial != nullptr ? partial + static_cast<size_t>(split) * M * N : C;
            const int ld = partial != nullptr ? N : ldc;
            const bool add = partial == nullptr && accumulate;
#pragma unroll 1
            for (int c0 = 32 * half; c0 < BN; c0 += 64) {
                float v[32];
                if (have) {
                    tmem_ld32(tmem + static_cast<uint32_t>(buf * BN + c0) + (static_cast<uint32_t>(quarter * 32) << 16), v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
                }
                if (store_mode != kStoreGeneric) {
                    // the previous block's store has finished reading the buffer
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    // row `lane` of the block: 16-byte chunk g at chunk position g ^ (row mod 8)
                    float4* rowp = reinterpret_cast<float4*>(tile + lane * 32);
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        rowp[g ^ (lane & 7)] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                    fence_proxy_async_shared();
                    __syncwarp();
                    const int col0 = w.n0 + c0;
                    if (lane == 0 && row0 < M && col0 < N) {
                        if (store_mode == kStoreC) tma_store_2d(&map_c, tile, col0, row0);
                        else if (store_mode == kAddC) tma_reduce_add_2d(&map_c, tile, col0, row0);
                        else tma_store_3d(&map_c, tile, col0, row0, split);
                        bulk_commit();
                    }
                    continue;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) tile[lane * 32 + (i ^ lane)] = v[i];
                __syncwarp();
                const int col = w.n0 + c0 + lane;
                if (col < N) {
#pragma unroll 4
                    for (int r = 0; r < 32; ++r) {
                        const int row = row0 + r;
                        if (row >= M) break;
                        float* dst = base + static_cast<size_t>(row) * ld + col;
                        const float x = tile[r * 32 + (lane ^ r)];
                        *dst = add ? *dst + x : x;
                    }
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&tempty[buf])) : "memory");
        }
        // the block stores this warp issued have completed before the CTA's
        // shared memory goes away
        if (store_mode != kStoreGeneric && lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 2 * BN);
}

// One thread waits, with the pipeline's bounded-wait code, on an mbarrier that
// nothing ever completes, so the wait runs out and the status word is set.
__global__ void bounded_wait_selftest_kernel(uint32_t* status, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (!mbar_wait(&bar, 0, polls)) atomicExch(status, kStatusTimeout);
    }
}

// ------------------------------------------------------------------ host side
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// 2-D bf16 tensor [outer][inner] with row pitch `ld` elements, box {64, box_outer}, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int inner, int outer, int ld, int box_outer) {
    EncodeTiled enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_outer)};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 output of the epilogue's TMA stores: [outer2][outer1][inner] with row
// pitch `ld` floats (outer2 = 1 gives the 2-D map of C), box {32, 32, 1},
// 128-byte swizzle (one 32-float row is one 128-byte swizzle row).
bool make_store_map(CUtensorMap* map, float* base, int inner, int outer1, int ld, int outer2) {
    EncodeTiled enc = encode_fn();
    if (enc == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (ld & 3) != 0) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer1),
                                static_cast<cuuint64_t>(outer2)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 4,
                                   static_cast<cuuint64_t>(ld) * 4 * static_cast<cuuint64_t>(outer1)};
    const cuuint32_t box[3] = {32u, 32u, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const cuuint32_t rank = outer2 > 1 ? 3u : 2u;
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank, base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int pick_bn(int N) { return N >= 256 ? 256 : (N > 64 ? 128 : 64); }

int sm_count() {
    static int n = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = kNumSMs;
    });
    return n;
}

template <int BN, bool A_MN, bool B_MN>
cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, int store_mode, int M,
                     int N, int K, int kps, int splits, float* C, int ldc, int accumulate, float* partial,
                     uint32_t* status, cudaStream_t st) {
    auto kern = gemm_tc_kernel<BN, A_MN, B_MN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<BN>::kBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const long long units = ceil_div(N, BN) * ceil_div(M, kBM) * splits;
    const int per_sm = Smem<BN>::kBytes * 2 <= 227 * 1024 ? 2 : 1;   // TMEM: 2 x 2 BN <= 512 columns for BN <= 128
    const long long grid = units < static_cast<long long>(sm_count()) * per_sm ? units : sm_count() * per_sm;
    kern<<<static_cast<unsigned>(grid), kGemmThreads, Smem<BN>::kBytes, st>>>(
        ma, mb, mc, store_mode, M, N, K, kps, splits, C, ldc, accumulate, splits > 1 ? partial : nullptr, status);
    return cudaGetLastError();
}

template <bool A_MN, bool B_MN>
cudaError_t launch_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, int store_mode,
                      int M, int N, int K, int kps, int splits, float* C, int ldc, int accumulate, float* partial,
                      uint32_t* status, cudaStream_t st) {
#define DUST_GEMM_BN(BN_)                                                                                        \
    launch_t<BN_, A_MN, B_MN>(ma, mb, mc, store_mode, M, N, K, kps, splits, C, ldc, accumulate, partial, status, st)
    switch (bn) {
        case 256: return DUST_GEMM_BN(256);
        case 128: return DUST_GEMM_BN(128);
        default: return DUST_GEMM_BN(64);
    }
#undef DUST_GEMM_BN
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(uint32_t* status, uint32_t polls, cudaStream_t stream) {
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, polls);
    return cudaGetLastError();
}

bool tma_map_bf16_2d(CUtensorMap* map, const void* base, int inner, int outer, int ld, int box_outer) {
    return make_map(map, base, inner, outer, ld, box_outer);
}

int device_sm_count() { return sm_count(); }

bool gemm_tc_supported(int M, int N, int K, bool a_kmajor, bool b_kmajor) {
    if (M <= 0 || N <= 0 || K <= 0) return false;
    if (encode_fn() == nullptr) return false;
    // TMA: global row pitch a multiple of 16 bytes -> contiguous extent a multiple of 8
    const bool a_ok = a_kmajor ? (K % 8 == 0) : (M % 8 == 0);
    const bool b_ok = b_kmajor ? (K % 8 == 0) : (N % 8 == 0);
    return a_ok && b_ok;
}

int gemm_tc_splits(int M, int N, int K) {
    // Work units are (tile, k slice); the persistent grid (one CTA per SM)
    // walks them in rounds.  Pick the split of k that keeps the most SMs busy
    // over all rounds, keeping slices of at least 16 k blocks; on a tie the
    // smaller split wins (partial tiles cost HBM traffic and a reduction).
    const long long tiles = ceil_div(M, kBM) * ceil_div(N, pick_bn(N));
    const long long kblocks = ceil_div(K, kBK);
    const long long grid = kNumSMs;
    long long best_s = 1;
    double best_u = 0.0;
    for (long long s = 1; s <= 32 && (s == 1 || kblocks / s >= 16); s *= 2) {
        const long long units = tiles * s;
        const double util = static_cast<double>(units) / static_cast<double>(ceil_div(units, grid) * grid);
        if (util > best_u + 1e-3) {
            best_u = util;
            best_s = s;
        }
    }
    return static_cast<int>(best_s);
}

cudaError_t launch_gemm_tc(const void* A, bool a_kmajor, int lda, const void* B, bool b_kmajor, int ldb, int M, int N,
                           int K, float* C, int ldc, int accumulate, float* partial, int splits, uint32_t* status,
                           cudaStream_t stream) {
    if (!gemm_tc_supported(M, N, K, a_kmajor, b_kmajor)) return cudaErrorNotSupported;
    const int bn = pick_bn(N);
    CUtensorMap ma, mb;
    // A: K-major [M][K] -> box {64 k, 128 rows}; MN-major [K][M] -> box {64 m, 64 k rows}
    const bool okA = a_kmajor ? make_map(&ma, A, K, M, lda, kBM) : make_map(&ma, A, M, K, lda, kBK);
    const bool okB = b_kmajor ? make_map(&mb, B, K, N, ldb, bn) : make_map(&mb, B, N, K, ldb, kBK);
    if (!okA || !okB) return cudaErrorInvalidValue;
    const int kps = static_cast<int>(ceil_div(ceil_div(K, splits), kBK) * kBK);
    // the epilogue's store: TMA into the split-K slabs, or into C (a store, or
    // a reduce-add when C is accumulated into) where the tensor map can
    // describe them; generic stores otherwise
    CUtensorMap mc;
    std::memset(&mc, 0, sizeof(mc));
    int store_mode = kStoreGeneric;
    if (splits > 1) {
        if (make_store_map(&mc, partial, N, M, N, splits)) store_mode = kStorePartial;
    } else if (make_store_map(&mc, C, N, M, ldc, 1)) {
        store_mode = accumulate ? kAddC : kStoreC;
    }
    cudaError_t e;
#define DUST_GEMM_MAJOR(AMN_, BMN_)                                                                              \
    launch_bn<AMN_, BMN_>(bn, ma, mb, mc, store_mode, M, N, K, kps, splits, C, ldc, accumulate, partial, status, stream)
    if (!a_kmajor && !b_kmajor)
        e = DUST_GEMM_MAJOR(true, true);
    else if (a_kmajor && b_kmajor)
        e = DUST_GEMM_MAJOR(false, false);
    else if (a_kmajor)
        e = DUST_GEMM_MAJOR(false, true);
    else
        e = DUST_GEMM_MAJOR(true, false);
#undef DUST_GEMM_MAJOR
    if (e != cudaSuccess || splits == 1) return e;
    return launch_splitk_reduce(partial, splits, M, N, C, ldc, accumulate, stream);
}

}  // namespace dust
