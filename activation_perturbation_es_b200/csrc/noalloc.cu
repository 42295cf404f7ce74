// noalloc.cu -- dust_layer_estimate_noalloc: the hidden-layer error estimate
// for callers that cannot allocate device memory.
//
// Some callers never get to call cudaMalloc: a plugin inside a host framework
// that owns every byte of device memory and hands the plugin only the device
// pointers of its inputs and outputs, or a caller whose memory pool is fully
// reserved and may not grow.  dust_layer_estimate needs a caller-provided
// workspace for the rewards r when it runs the reward scan itself; this entry
// point keeps that scratch instead in a file-scope device array of fixed size
// that is part of the library image, so the caller passes only inputs and
// outputs.
//
// Costs and limits of the static array:
//   - every GPU on which the library is loaded holds kNoAllocScratchBytes
//     (16 MiB for the rewards, plus 64 KiB for the chunk maps of the chunked
//     scan) for it until the process exits;
//   - the reward scan takes the same path as dust_layer_estimate's (per
//     sequence, or over 1024-token chunks for few long sequences), so both
//     entry points return the same bits;
//   - draw_count * T must not exceed kNoAllocScratchFloats (4 Mi) when the
//     scan is needed (gamma > 0); split the draws over several calls with
//     accumulate = 1 otherwise (the estimate is linear in the draws);
//   - all calls share the one array: two calls whose kernels overlap on the
//     GPU (different streams, or several host threads) race on it, so
//     serialise them (one stream, or events);
//   - the array keeps the previous call's rewards; nothing here needs it to
//     start at zero, because the scan overwrites every element of
//     [draw_count][T] that the reduction then reads (seq_offsets cover [0, T)).
//
// Host code must not pass the array's name to a kernel: on the host it is a
// stand-in symbol, not a device address.  The device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first
// call made on that device; make that first call before any stream capture.
// The address is cached for the life of the process: after cudaDeviceReset of
// a device it is stale, and this entry point must not be used on that device
// again.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dust {

namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 22;           // the rewards r: 16 MiB
// The chunked scan runs only when draws x sequences < 4 x 148 (so draw_count
// < 592), and then needs 12 bytes per (draw, 1024-token chunk): at most
// (4 Mi / 1024 + 592) x 12 bytes < 64 KiB within the rewards' limit.
constexpr size_t kNoAllocChunkFloats = size_t(1) << 14;             // 64 KiB
constexpr size_t kNoAllocScratchBytes = (kNoAllocScratchFloats + kNoAllocChunkFloats) * sizeof(float);
static_assert(kNoAllocScratchFloats * sizeof(float) == (size_t(16) << 20), "16 MiB of static scratch for r");

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats + kNoAllocChunkFloats];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_address(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

dust_status reject(dust_status s, const char* fmt, long long a = 0, long long b = 0) {
    char msg[256];
    std::snprintf(msg, sizeof msg, fmt, a, b);
    return record_error(s, msg);
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

}  // namespace dust

extern "C" dust_status dust_layer_estimate_noalloc(const float* c, int T, int d_out, const int32_t* seq_offsets,
                                                   int n_seq, float gamma, dust_noise nz, float* g_hat,
                                                   void* g_hat_bf16, int accumulate, void* stream) {
    using namespace dust;
    if (nz.draw_count == 0 || nz.K_total == 0 || !(nz.sigma > 0.0f) || !(nz.sigma < INFINITY))
        return reject(DUST_ERR_INVALID_ARG, "noise: draw_count and K_total must be > 0, sigma finite and > 0");
    if (static_cast<unsigned long long>(nz.draw_begin) + nz.draw_count > (1ull << 32))
        return reject(DUST_ERR_INVALID_ARG, "draw_begin + draw_count exceeds 2^32");
    if (nz.token_begin > 0x7FFFFFFFu) return reject(DUST_ERR_INVALID_ARG, "token_begin must be < 2^31");
    if (T <= 0 || d_out <= 0) return reject(DUST_ERR_INVALID_ARG, "T and d_out must be > 0 (T=%lld, d_out=%lld)", T, d_out);
    if (!(gamma >= 0.0f && gamma <= 1.0f)) return reject(DUST_ERR_INVALID_ARG, "gamma must be in [0, 1]");
    if (c == nullptr || g_hat == nullptr) return reject(DUST_ERR_INVALID_ARG, "c and g_hat must not be NULL");
    if (misaligned(c) || misaligned(g_hat) || misaligned(g_hat_bf16))
        return reject(DUST_ERR_ALIGNMENT, "c, g_hat and g_hat_bf16 must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float* r = c;
    if (gamma != 0.0f) {   // gamma = 0: r = c, no scratch needed
        if (seq_offsets == nullptr || n_seq < 1) return reject(DUST_ERR_INVALID_ARG, "seq_offsets and n_seq >= 1 are required");
        if (misaligned(seq_offsets)) return reject(DUST_ERR_ALIGNMENT, "seq_offsets must be 16-byte aligned");
        const unsigned long long need = static_cast<unsigned long long>(nz.draw_count) * static_cast<unsigned long long>(T);
        if (need > kNoAllocScratchFloats)
            return reject(DUST_ERR_WORKSPACE,
                          "draw_count x T = %lld exceeds the static scratch of %lld floats (16 MiB); split the "
                          "draws over several calls with accumulate = 1, or use dust_layer_estimate",
                          static_cast<long long>(need), static_cast<long long>(kNoAllocScratchFloats));
        if (static_cast<long long>(nz.draw_count) * n_seq >= (1ll << 31))
            return reject(DUST_ERR_INVALID_ARG, "draws x sequences must be < 2^31");
        float* scratch = nullptr;
        cudaError_t e = scratch_address(&scratch);
        const int K = static_cast<int>(nz.draw_count);
        // the scan dust_layer_estimate would run (same bits); the chunk maps live
        // behind the rewards (their size always fits, see kNoAllocChunkFloats)
        const bool chunks = reward_scan_prefers_chunks(K, T, n_seq) &&
                            reward_scan_chunks_workspace(K, T) <= kNoAllocChunkFloats * sizeof(float);
        if (e == cudaSuccess)
            e = chunks ? launch_reward_scan_chunks(c, scratch, K, T, seq_offsets, n_seq, gamma,
                                                   scratch + kNoAllocScratchFloats, st)
                       : launch_reward_scan(c, scratch, K, T, seq_offsets, n_seq, gamma, st);
        if (e != cudaSuccess) return record_error(DUST_ERR_CUDA, cudaGetErrorString(e));
        r = scratch;
    }
    const cudaError_t e = launch_layer_estimate(r, T, d_out, nz, g_hat, g_hat_bf16, accumulate, st);
    if (e != cudaSuccess) return record_error(DUST_ERR_CUDA, cudaGetErrorString(e));
    return DUST_OK;
}
