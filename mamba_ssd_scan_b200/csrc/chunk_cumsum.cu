// chunk_cumsum.cu -- step 1 of the chunked SSD forward: dt = softplus(dt_raw +
// dt_bias) (no clamp) and the inclusive cumulative sum of dt * A_h inside each
// chunk ("MAMBA-2 Reference Implementations Comparison", section 3.2: the
// softplus discretisation of dt and the exp(A dt) decay whose exponents this
// sum accumulates; "MAMBA-2 Implementation Gaps", Gap 1: the per-chunk
// processing).
//
// One warp per (chunk, head) (chunk_cumsum_warp in internal.cuh, which the
// tensor-core chunk_state also runs when it forms dt and cumA itself); the
// eight warps of a CTA take eight consecutive heads of one chunk, so their
// strided dt reads share sectors.
#include "internal.cuh"

namespace ssd {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) chunk_cumsum_kernel(FwdParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t H = p.nheads, nc = p.nchunks;
    const int64_t b = blockIdx.y;
    grid_dep_wait();    // dt / cumA may still be read by earlier work on the stream
    grid_dep_launch();
    if (blockIdx.x == 0 && b == 0 && threadIdx.x == 0 && p.status) *p.status = 0;  // a new call
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    if (item >= nc * H) return;  // whole warps only
    const int64_t c = item / H, h = item % H;
    const int64_t off = ((b * H + h) * nc + c) * p.chunk;
    chunk_cumsum_warp<T>(p, b, c, h, p.dt + off, p.cumA + off, lane);
}

}  // namespace

template <typename T>
cudaError_t launch_chunk_cumsum(const FwdParams& p, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((p.nchunks * p.nheads + 7) / 8), static_cast<unsigned>(p.batch));
    return launch_kernel(chunk_cumsum_kernel<T>, grid, dim3(256), 0, s, p.pdl != 0, p);
}

template cudaError_t launch_chunk_cumsum<float>(const FwdParams&, cudaStream_t);
template cudaError_t launch_chunk_cumsum<__nv_bfloat16>(const FwdParams&, cudaStream_t);

}  // namespace ssd
