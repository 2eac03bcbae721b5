// chunk_state_ffma.cu -- step 2 of the chunked SSD forward on CUDA cores
// (fp32 FFMA): every chunk's local state, as if the chunk started from zero,
//   S_c[p,n] = sum_{l in c} exp(cumA[last] - cumA[l]) dt[l] x[l,p] B[l,n]
// (the "diagonal block: local state" of "MAMBA-2 Implementation Gaps", Gap 1),
// accumulated in fp32 and stored in the input dtype.
//
// This is the exact-fp32 path (fp32 inputs need 1e-4 agreement, beyond what
// TF32 tensor cores give) and the fallback for shapes outside the tensor-core
// kernel's range.  One CTA computes a 64(p) x 64(n) tile of one (b, c, h);
// tokens are staged 32 at a time in shared memory, the decay weight folded
// into x while staging.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int TP = 64, TN = 64, TK = 32;

template <typename T>
__global__ void __launch_bounds__(256) chunk_state_ffma_kernel(FwdParams p) {
    grid_dep_wait();  // dt and cumA come from step 1
    grid_dep_launch();
    const int64_t H = p.nheads, P = p.headdim, N = p.dstate, G = p.ngroups;
    const int64_t L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int64_t ntile_n = (N + TN - 1) / TN;
    const int64_t p0 = (blockIdx.y / ntile_n) * TP, n0 = (blockIdx.y % ntile_n) * TN;
    const int64_t c = blockIdx.x / H, h = blockIdx.x % H, b = blockIdx.z;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const float cs_last = csc[Q - 1];
    const T* x = static_cast<const T*>(p.x);
    const T* Bm = static_cast<const T*>(p.B);

    __shared__ float xs[TK][TP];
    __shared__ float bs[TK][TN];
    __shared__ float ws[TK];

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < Lc; k0 += TK) {
        if (tid < TK) {
            const int64_t l = k0 + tid;
            ws[tid] = (l < Lc) ? expf(cs_last - csc[l]) * dtc[l] : 0.0f;
        }
        __syncthreads();
        for (int i = tid; i < TK * TP; i += 256) {
            const int kk = i / TP, pp = i % TP;
            const int64_t l = k0 + kk;
            float v = 0.0f;
            if (l < Lc && p0 + pp < P) v = to_f32(x[((b * L + t0 + l) * H + h) * P + p0 + pp]);
            xs[kk][pp] = v * ws[kk];
        }
        for (int i = tid; i < TK * TN; i += 256) {
            const int kk = i / TN, nn = i % TN;
            const int64_t l = k0 + kk;
            float v = 0.0f;
            if (l < Lc && n0 + nn < N) v = to_f32(Bm[((b * L + t0 + l) * G + g) * N + n0 + nn]);
            bs[kk][nn] = v;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int64_t sbase = ((b * nc + c) * H + h) * P * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t pi = p0 + ty * 4 + i, nj = n0 + tx * 4;
        if (pi < P && nj < N) {
            if (p.states_f32) {
                float* out = static_cast<float*>(p.states) + sbase;
#pragma unroll
                for (int j = 0; j < 4; ++j) out[pi * N + nj + j] = acc[i][j];
            } else {
                T* out = static_cast<T*>(p.states) + sbase;
#pragma unroll
                for (int j = 0; j < 4; ++j) out[pi * N + nj + j] = from_f32<T>(acc[i][j]);
            }
        }
    }
}

}  // namespace

template <typename T>
cudaError_t launch_chunk_state_ffma(const FwdParams& p, cudaStream_t s) {
    const unsigned tiles = (unsigned)(((p.headdim + TP - 1) / TP) * ((p.dstate + TN - 1) / TN));
    dim3 grid((unsigned)(p.nchunks * p.nheads), tiles, (unsigned)p.batch);
    return launch_kernel(chunk_state_ffma_kernel<T>, grid, dim3(256), 0, s, p.pdl != 0, p);
}

template cudaError_t launch_chunk_state_ffma<float>(const FwdParams&, cudaStream_t);
template cudaError_t launch_chunk_state_ffma<__nv_bfloat16>(const FwdParams&, cudaStream_t);

}  // namespace ssd
