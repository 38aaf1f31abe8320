// gemm_tc.cu -- prefill path (M > 8 tokens): tensor-core GEMM.
#include "common.cuh"

namespace bitnet {

bool gemm_available() { return false; }

cudaError_t launch_gemm(const int8_t *, const float *, int64_t, const bitnet_tw *, float *, int32_t *, int32_t *,
                        cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace bitnet
