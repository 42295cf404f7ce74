// gemm_tcgen05.cu -- placeholder until the tcgen05 kernel lands.
#include "common.cuh"
#include "kernels.h"

namespace dust {
bool gemm_tc_supported(int, int, int, bool, bool) { return false; }
int gemm_tc_splits(int, int, int) { return 1; }
cudaError_t launch_gemm_tc(const void*, bool, int, const void*, bool, int, int, int, int, float*, int, int, float*,
                           int, uint32_t*, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace dust
