// chunk_scan_ffma.cu -- step 4 of the chunked SSD forward on CUDA cores (fp32
// FFMA): each chunk's output from its own tokens and the state entering it,
//
//   y[l,p] = sum_{j<=l, j in chunk} exp(cumA[l]-cumA[j]) (C_l.B_j) dt[j] x[j,p]
//          + exp(cumA[l]) sum_n C_l[n] H_in[p,n]  +  D x[l,p]
//
// The first sum is the masked-attention (quadratic) dual form of SSD applied
// inside the chunk ("MAMBA-2 Reference Implementations Comparison", section
// 2.2: Y = diag(p) M diag(q) X with M 1-semiseparable); the second is the
// off-diagonal contribution of the carried state ("MAMBA-2 Implementation
// Gaps", Gap 1); the third is the D skip (Gap 4).
//
// Exact-fp32 path and fallback for shapes the tensor-core kernel does not
// take.  One CTA produces a 64(l) x 64(p) output tile of one (b, c, h): the
// C rows of the tile stay in shared memory; the state term runs over 32-wide
// dstate slabs of H_in; the intra-chunk term walks 32-token slabs of the chunk
// up to the tile's last row (causal: later tokens are skipped), forming the
// masked C.B^T slab in shared memory before multiplying it into x.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int TL = 64, TPP = 64, TJ = 32;

__host__ __device__ inline int64_t cs_stride(int64_t N) { return N + 4; }  // padded rows

template <typename T>
__global__ void __launch_bounds__(256) chunk_scan_ffma_kernel(FwdParams p) {
    grid_dep_wait();  // dt, cumA and the carried states come from steps 1-3
    const int64_t H = p.nheads, P = p.headdim, N = p.dstate, G = p.ngroups;
    const int64_t L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int64_t ntile_p = (P + TPP - 1) / TPP;
    const int64_t l0 = (blockIdx.y / ntile_p) * TL, p0 = (blockIdx.y % ntile_p) * TPP;
    const int64_t c = blockIdx.x / H, h = blockIdx.x % H, b = blockIdx.z;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
    if (l0 >= Lc) return;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const T* x = static_cast<const T*>(p.x);
    const T* Bm = static_cast<const T*>(p.B);
    const T* Cm = static_cast<const T*>(p.C);
    // the state entering the chunk, fp32 or in the input dtype
    const int64_t sbase = ((b * nc + c) * H + h) * P * N;
    const float* Hin32 = static_cast<const float*>(p.states) + sbase;
    const T* HinT = static_cast<const T*>(p.states) + sbase;
    auto hin = [&](int64_t i) { return p.states_f32 ? Hin32[i] : to_f32(HinT[i]); };
    const int64_t SN = cs_stride(N);

    extern __shared__ float smem[];
    float* Cs = smem;                    // [TL][SN]
    float* Bs = Cs + TL * SN;            // [TJ][SN]
    float* Ms = Bs + TJ * SN;            // [TL][TJ + 1]
    float* Xs = Ms + TL * (TJ + 1);      // [TJ][TPP]  (also H_in slab [TJ][TPP])
    float* cl = Xs + TJ * TPP;           // [TL] cumA of the tile's rows
    float* cj = cl + TL;                 // [TJ] cumA of the slab's tokens
    float* dj = cj + TJ;                 // [TJ] dt of the slab's tokens

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    for (int64_t i = tid; i < TL * N; i += 256) {
        const int64_t r = i / N, n = i % N, l = l0 + r;
        Cs[r * SN + n] = (l < Lc) ? to_f32(Cm[((b * L + t0 + l) * G + g) * N + n]) : 0.0f;
    }
    if (tid < TL) cl[tid] = (l0 + tid < Lc) ? csc[l0 + tid] : 0.0f;
    __syncthreads();

    // state term: acc = C_tile . H_in^T over dstate slabs of 32
    float acc[4][4] = {};
    for (int64_t n0 = 0; n0 < N; n0 += TJ) {
        for (int i = tid; i < TJ * TPP; i += 256) {
            const int kk = i / TPP, pp = i % TPP;
            const int64_t n = n0 + kk, pi = p0 + pp;
            Xs[kk * TPP + pp] = (n < N && pi < P) ? hin(pi * N + n) : 0.0f;
        }
        __syncthreads();
        const int64_t kmax = (N - n0 < TJ) ? (N - n0) : TJ;
        for (int kk = 0; kk < kmax; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Cs[(ty * 4 + i) * SN + n0 + kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Xs[kk * TPP + tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float sc = expf(cl[ty * 4 + i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] *= sc;
    }

    // intra-chunk term over token slabs up to the tile's last row
    const int64_t jend = (l0 + TL < Lc) ? (l0 + TL) : Lc;
    for (int64_t j0 = 0; j0 < jend; j0 += TJ) {
        for (int64_t i = tid; i < TJ * N; i += 256) {
            const int64_t r = i / N, n = i % N, j = j0 + r;
            Bs[r * SN + n] = (j < Lc) ? to_f32(Bm[((b * L + t0 + j) * G + g) * N + n]) : 0.0f;
        }
        for (int i = tid; i < TJ * TPP; i += 256) {
            const int kk = i / TPP, pp = i % TPP;
            const int64_t j = j0 + kk, pi = p0 + pp;
            Xs[kk * TPP + pp] =
                (j < Lc && pi < P) ? to_f32(x[((b * L + t0 + j) * H + h) * P + pi]) : 0.0f;
        }
        if (tid < TJ) {
            const int64_t j = j0 + tid;
            cj[tid] = (j < Lc) ? csc[j] : 0.0f;
            dj[tid] = (j < Lc) ? dtc[j] : 0.0f;
        }
        __syncthreads();
        // masked C.B^T slab: thread -> row r = tid/4, 8 columns
        {
            const int r = tid >> 2, jc = (tid & 3) * 8;
            const int64_t l = l0 + r;
            float cb[8] = {};
            for (int64_t n = 0; n < N; ++n) {
                const float cv = Cs[r * SN + n];
#pragma unroll
                for (int q = 0; q < 8; ++q) cb[q] = fmaf(cv, Bs[(jc + q) * SN + n], cb[q]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t j = j0 + jc + q;
                float m = 0.0f;
                if (j <= l && l < Lc) m = expf(cl[r] - cj[jc + q]) * cb[q] * dj[jc + q];
                Ms[r * (TJ + 1) + jc + q] = m;
            }
        }
        __syncthreads();
        for (int kk = 0; kk < TJ; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Ms[(ty * 4 + i) * (TJ + 1) + kk];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Xs[kk * TPP + tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }

    // epilogue: + D x, the optional output gate, round to the output type
    const float Dh = p.D ? p.D[h] : 0.0f;
    T* y = static_cast<T*>(p.y);
    const T* zg = static_cast<const T*>(p.z);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t l = l0 + ty * 4 + i;
        if (l >= Lc) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t pi = p0 + tx * 4 + j;
            if (pi >= P) continue;
            const int64_t o = ((b * L + t0 + l) * H + h) * P + pi;
            const float v = acc[i][j] + Dh * to_f32(x[o]);
            y[o] = from_f32<T>(zg ? v * silu_f32(to_f32(zg[o])) : v);
        }
    }
}

size_t scan_smem_bytes(int64_t N) {
    const int64_t SN = cs_stride(N);
    return sizeof(float) * (size_t)(TL * SN + TJ * SN + TL * (TJ + 1) + TJ * TPP + TL + 2 * TJ);
}

}  // namespace

template <typename T>
cudaError_t launch_chunk_scan_ffma(const FwdParams& p, cudaStream_t s) {
    const size_t smem = scan_smem_bytes(p.dstate);
    cudaError_t e = cudaFuncSetAttribute(chunk_scan_ffma_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned tiles = (unsigned)(((p.chunk + TL - 1) / TL) * ((p.headdim + TPP - 1) / TPP));
    dim3 grid((unsigned)(p.nchunks * p.nheads), tiles, (unsigned)p.batch);
    return launch_kernel(chunk_scan_ffma_kernel<T>, grid, dim3(256), smem, s, p.pdl != 0, p);
}

template cudaError_t launch_chunk_scan_ffma<float>(const FwdParams&, cudaStream_t);
template cudaError_t launch_chunk_scan_ffma<__nv_bfloat16>(const FwdParams&, cudaStream_t);

}  // namespace ssd
