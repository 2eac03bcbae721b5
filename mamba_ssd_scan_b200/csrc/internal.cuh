// internal.cuh -- shared declarations of the SSD scan kernels (not part of the
// public ABI; see include/ssd.h for the operation and the layouts).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// Sizes and pointers of one forward call, as the kernels see them.
struct FwdParams {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nchunks;
    int64_t heads_per_group;
    int32_t flags;         // SSD_FLAG_* of the call
    const void* x;
    const void* dt_raw;
    const float* A;
    const void* B;
    const void* C;
    const float* D;        // may be null
    const float* dt_bias;  // may be null
    const float* init_state;  // may be null
    void* y;
    float* final_state;    // may be null
    // intermediates (workspace)
    float* dt;      // [b, H, nc, Q]
    float* cumA;    // [b, H, nc, Q]
    void* states;   // [b, nc, H, P, N] in the input dtype (local states, then states entering each chunk)
    int* status;    // device status word (SSD_ERR_TIMEOUT on a timed-out wait); may be null
};

struct DecodeParams {
    int64_t batch, nheads, headdim, dstate, ngroups, heads_per_group;
    float* state;
    const void* x;
    const void* dt_raw;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    void* y;
};

// Element loads/stores for the two supported input types.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// softplus(u) = log(1 + e^u) without overflow.
__device__ __forceinline__ float softplus_f32(float u) {
    return fmaxf(u, 0.0f) + log1pf(expf(-fabsf(u)));
}

// Launchers (one per kernel family).  Each returns cudaGetLastError().
template <typename T> cudaError_t launch_chunk_cumsum(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_chunk_state_ffma(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_state_passing(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_chunk_scan_ffma(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_state_update(const DecodeParams& p, cudaStream_t s);

// Tensor-core (tcgen05) variants for bf16 inputs, with their shape ranges.
bool chunk_state_tc_supported(const FwdParams& p);
cudaError_t launch_chunk_state_tc(const FwdParams& p, cudaStream_t s);
bool chunk_scan_tc_supported(const FwdParams& p);
cudaError_t launch_chunk_scan_tc(const FwdParams& p, cudaStream_t s);

}  // namespace ssd
