// bwd_tc.h -- the backward pass's tensor-core kernels as bwd.cu sees them.
#pragma once

#include "internal.cuh"

namespace ssd {

// The chunk-local adjoint dS_c = sum_t e^{cumA_t} dy_t C_t^T on the tensor
// cores (same shapes as launch_bwd_tc), fp32 into BwdParams::dstates.
cudaError_t launch_bwd_tc_dstate(const BwdParams& p, cudaStream_t s);

}  // namespace ssd
