// gemm_fp8.cu -- grouped expert GEMMs with FP8 e4m3 operands and 128x128
// block scales (placeholder launchers until the kernels land).
#include "common.cuh"
#include "launch.h"

namespace moe {

cudaError_t launch_gateup_fp8(const GroupedGemmArgs&, const uint8_t*, const float*, const uint8_t*,
                              const float*, const uint8_t*, const float*, uint8_t*, float*,
                              cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t launch_down_fp8(const GroupedGemmArgs&, const uint8_t*, const float*, const uint8_t*,
                            const float*, const uint8_t*, const float*, float*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace moe
