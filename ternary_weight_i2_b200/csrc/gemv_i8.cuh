// gemv_i8.cuh -- host-side description of one I8_S linear handed to the
// grouped decode launch (gemv_i8.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/bitnet.h"

namespace bitnet {

// One linear of a grouped call: weights, the quantised activations of all m
// tokens, the outputs of all m tokens and the optional epilogue.
struct I8Job {
    const int8_t *w;        // [n, 32*ceil(k/32)]
    int64_t n, k;
    float s_w;
    const int8_t *q;        // [m, kpad]
    const float *s_act;     // [m]
    float *y;               // [m, n]
    int32_t *acc;           // [m, n] or null
    const bitnet_epilogue *epi;
};

// Runs `count` (<= BITNET_I8_GROUP_MAX) linears sharing the token count m,
// one launch per slice of at most 8 tokens.
cudaError_t launch_gemv_i8_group(const I8Job *jobs, int count, int64_t m, int sm_count, cudaStream_t st);

}  // namespace bitnet
