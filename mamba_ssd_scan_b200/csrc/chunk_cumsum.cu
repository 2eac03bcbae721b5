// chunk_cumsum.cu -- step 1 of the chunked SSD forward: dt = softplus(dt_raw +
// dt_bias) (no clamp) and the inclusive cumulative sum of dt * A_h inside each
// chunk ("MAMBA-2 Reference Implementations Comparison", section 3.2: the
// softplus discretisation of dt and the exp(A dt) decay whose exponents this
// sum accumulates; "MAMBA-2 Implementation Gaps", Gap 1: the per-chunk
// processing).
//
// One warp per (chunk, head); the eight warps of a CTA take eight consecutive
// heads of one chunk, so their strided dt reads share sectors.  Each lane
// loads its tokens of every 32-token segment first, then the warp scans the
// segments in order with warp shuffles and a running carry.  Entries past the
// end of a short last chunk hold dt = 0 and the last cumulative value, so
// cumA[.., Q-1] is always the chunk's total log-decay.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int MAXSEG = 8;  // chunk <= 256 tokens

template <typename T>
__global__ void __launch_bounds__(256) chunk_cumsum_kernel(FwdParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Q = p.chunk, H = p.nheads, L = p.seqlen, nc = p.nchunks;
    const int64_t b = blockIdx.y;
    if (blockIdx.x == 0 && b == 0 && threadIdx.x == 0 && p.status) *p.status = 0;  // a new call
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    if (item >= nc * H) return;  // whole warps only
    const int64_t c = item / H, h = item % H;
    const int64_t t0 = c * Q;
    const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
    const int nseg = static_cast<int>((Q + 31) / 32);
    const T* dtr = static_cast<const T*>(p.dt_raw) + (b * L + t0) * H + h;
    const float A = p.A[h];
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
    float u[MAXSEG];
#pragma unroll
    for (int s = 0; s < MAXSEG; ++s) {
        const int64_t l = s * 32 + lane;
        u[s] = (s < nseg && l < Lc) ? to_f32(dtr[l * H]) : 0.0f;
    }
    float* dto = p.dt + ((b * H + h) * nc + c) * Q;
    float* cso = p.cumA + ((b * H + h) * nc + c) * Q;
    float carry = 0.0f;
#pragma unroll
    for (int s = 0; s < MAXSEG; ++s) {
        if (s >= nseg) break;
        const int64_t l = s * 32 + lane;
        float dt = 0.0f, v = 0.0f;
        if (l < Lc) {
            dt = softplus_f32(u[s] + bias);
            v = dt * A;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        v += carry;
        if (l < Q) {
            dto[l] = dt;
            cso[l] = v;
        }
        carry = __shfl_sync(0xffffffffu, v, 31);
    }
}

}  // namespace

template <typename T>
cudaError_t launch_chunk_cumsum(const FwdParams& p, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((p.nchunks * p.nheads + 7) / 8), static_cast<unsigned>(p.batch));
    chunk_cumsum_kernel<T><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

template cudaError_t launch_chunk_cumsum<float>(const FwdParams&, cudaStream_t);
template cudaError_t launch_chunk_cumsum<__nv_bfloat16>(const FwdParams&, cudaStream_t);

}  // namespace ssd
