// gated_rmsnorm.h -- the gated RMSNorm after the scan as api.cu sees it.
#pragma once

#include "internal.cuh"

namespace ssd {

struct NormParams {
    int64_t rows, channels, group;
    float eps;
    const void* y;          // [rows, channels]
    const void* z;          // [rows, channels]; may be null (no gate)
    const float* weight;    // [channels]
    void* out;              // [rows, channels]; may equal y
};

cudaError_t launch_gated_rmsnorm(const NormParams& p, bool bf16, cudaStream_t s);

}  // namespace ssd
