// bwd.cu -- the backward pass of the chunked SSD scan: gradients of
//   J = sum_t dy_t . y_t + d_final : h_L
// with respect to x, the raw dt, A, B, C, D, dt_bias and the initial state.
// The page "Agent 230: Comprehensive MAMBA-2 Implementation Comparison",
// section 6 (Gradient Computation), takes the gradients of A, B, C and delta
// (dt) after its backward pass; it gives no formulas.  Theirs and the other
// inputs' follow from the chain rule on the chunked forward ("MAMBA-2 Reference Implementations Comparison", section
// 2.2; "MAMBA-2 Implementation Gaps", Gap 1).  Per (batch, head), with cumA
// the in-chunk cumulative log decay, H_c the state entering chunk c and dH_c
// the gradient with respect to the state leaving chunk c:
//
//   dH_{nc-1} = d_final,  dH_{c-1} = e^{cumA_c[last]} dH_c + sum_{l in c} e^{cumA_l} dy_l C_l^T
//   d_init    = dH_{-1}
//   dxs_s = sum_{t>=s} e^{cumA_t - cumA_s} (C_t . B_s) dy_t + e^{cumA_last - cumA_s} dH_c B_s
//   dx_s  = D dy_s + dt_s dxs_s
//   dB_s  = dt_s [ sum_{t>=s} e^{cumA_t - cumA_s} (dy_t . x_s) C_t + e^{cumA_last - cumA_s} dH_c^T x_s ]
//   dC_t  = sum_{s<=t} e^{cumA_t - cumA_s} dt_s (dy_t . x_s) B_s + e^{cumA_t} H_c^T dy_t
//   da_t  = e^{a_t} <g_t, h_{t-1}>  (the gradient of the log decay a_t = dt_t A,
//           g_t = dJ/dh_t), taken apart at the chunk boundary into sums over
//           one chunk (bwd_dt_kernel)
//   ddt_t = x_t . dxs_t + A da_t,   ddt_raw_t = ddt_t sigmoid(dt_raw_t + dt_bias)
//   dA = sum dt_t da_t,  dD = sum dy_t . x_t,  ddt_bias = sum ddt_raw_t
// da_t is not formed as a reverse cumulative sum over the whole sequence of
// the per-token gradients of the cumulative decay: that sum runs over up to L
// large, mostly cancelling terms and loses the precision the chunk-local form
// keeps.
//
// The forward's own kernels first recompute dt, cumA and H_c into the
// workspace.  Then, all on CUDA cores in fp32: the local adjoint of each chunk
// (bwd_dstate_kernel), the reverse carry (bwd_state_passing_kernel), two
// per-chunk kernels over 64-token blocks (A: per source block s, dx and dB;
// B: per target block t, dC; both also leave the per-token pieces of da), one
// warp per (batch, head) for da and the dt gradients, and a finishing kernel that sums over batch
// rows and over the heads of a group in a fixed order (no atomics: the result
// is bitwise reproducible).
#include "internal.cuh"
#include "bwd_tc.h"

namespace ssd {
namespace {

constexpr int BR = 64;    // tokens per block of the per-chunk kernels
constexpr int NT = 256;   // threads of the per-chunk kernels (16 x 16, 4 x 4 outputs each)

// ---------------------------------------------------------------------------
// Local adjoint of each chunk, dS_c[p,n] = sum_{l in c} e^{cumA_l} dy_l[p] C_l[n]
// (fp32); one CTA per 64(p) x 64(n) tile of one (b, c, h), tokens staged 32 at a
// time with the decay folded into dy.
constexpr int DP = 64, DN = 64, DK = 32;

template <typename T>
__global__ void __launch_bounds__(256) bwd_dstate_kernel(BwdParams bp) {
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, P = p.headdim, N = p.dstate, G = p.ngroups;
    const int64_t L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int64_t ntile_n = (N + DN - 1) / DN;
    const int64_t p0 = (blockIdx.y / ntile_n) * DP, n0 = (blockIdx.y % ntile_n) * DN;
    const int64_t c = blockIdx.x / H, h = blockIdx.x % H, b = blockIdx.z;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const T* dy = static_cast<const T*>(bp.dy);
    const T* Cm = static_cast<const T*>(p.C);

    __shared__ float ys[DK][DP];
    __shared__ float cs[DK][DN];
    __shared__ float ws[DK];

    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < Lc; k0 += DK) {
        if (tid < DK) {
            const int64_t l = k0 + tid;
            ws[tid] = (l < Lc) ? expf(csc[l]) : 0.0f;
        }
        __syncthreads();
        for (int i = tid; i < DK * DP; i += 256) {
            const int kk = i / DP, pp = i % DP;
            const int64_t l = k0 + kk;
            float v = 0.0f;
            if (l < Lc && p0 + pp < P) v = to_f32(dy[((b * L + t0 + l) * H + h) * P + p0 + pp]);
            ys[kk][pp] = v * ws[kk];
        }
        for (int i = tid; i < DK * DN; i += 256) {
            const int kk = i / DN, nn = i % DN;
            const int64_t l = k0 + kk;
            float v = 0.0f;
            if (l < Lc && n0 + nn < N) v = to_f32(Cm[((b * L + t0 + l) * G + g) * N + n0 + nn]);
            cs[kk][nn] = v;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < DK; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = ys[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = cs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = bp.dstates + ((b * nc + c) * H + h) * P * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t pi = p0 + ty * 4 + i, nj = n0 + tx * 4;
        if (pi < P && nj < N) {
#pragma unroll
            for (int j = 0; j < 4; ++j) out[pi * N + nj + j] = acc[i][j];
        }
    }
}

// ---------------------------------------------------------------------------
// Reverse carry over chunks, one thread per 4 state elements of one (b, h):
//   carry = d_final;  for c = nc-1 .. 0: slot c <- carry;  carry = e^{cumA_c[last]} carry + dS_c
// in place over dstates (slot c then holds the gradient with respect to the
// state leaving chunk c); d_init = the carry after chunk 0.
__global__ void __launch_bounds__(256) bwd_state_passing_kernel(BwdParams bp) {
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, nc = p.nchunks, Q = p.chunk;
    const int64_t vecs_per_head = p.headdim * p.dstate / 4;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= p.batch * H * vecs_per_head) return;
    const int64_t bh = e / vecs_per_head, off = e % vecs_per_head;
    const int64_t b = bh / H, h = bh % H;
    float4 carry = bp.d_final ? reinterpret_cast<const float4*>(bp.d_final)[e]
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float4* base = reinterpret_cast<float4*>(bp.dstates) + (b * nc * H + h) * vecs_per_head + off;
    const int64_t cstride = H * vecs_per_head;
    const float* cs = p.cumA + (b * H + h) * nc * Q + (Q - 1);
    for (int64_t c = nc - 1; c >= 0; --c) {
        const float4 s = base[c * cstride];
        const float a = expf(cs[c * Q]);
        base[c * cstride] = carry;
        carry.x = fmaf(a, carry.x, s.x);
        carry.y = fmaf(a, carry.y, s.y);
        carry.z = fmaf(a, carry.z, s.z);
        carry.w = fmaf(a, carry.w, s.w);
    }
    if (bp.d_init) reinterpret_cast<float4*>(bp.d_init)[e] = carry;
}

// ---------------------------------------------------------------------------
// Per-chunk kernels.  Shared-memory operands are fp32; "transposed" copies
// ([column][token], row stride BRP = 68 floats: 16-byte aligned rows, 4-way
// bank conflicts at most when they are filled) serve the products whose
// reduction runs over channels, row-major copies those that reduce over tokens.
constexpr int BRP = BR + 4;

__host__ __device__ inline int64_t smem_a_floats(int64_t P, int64_t N, int64_t Q) {
    const int64_t tblk = N * BRP + BR * N + P * BRP + BR * P;
    const int64_t uni = tblk > 2 * N * P ? tblk : 2 * N * P;
    return N * BRP + P * BRP + uni + 2 * BR * BR + 2 * Q + 16 * BR;
}
__host__ __device__ inline int64_t smem_b_floats(int64_t P, int64_t N, int64_t Q) {
    const int64_t sblk = P * BRP + BR * N + BR * BR;
    const int64_t uni = sblk > P * N ? sblk : P * N;
    return P * BRP + uni + 2 * Q;
}

// rows r0 .. r0+BR-1 of a [rows][width] matrix (row stride `stride` elements,
// zero at and after row `lim`) into dst[col * BRP + r] (transposed) or
// dst[r * width + col] (row-major), widened to fp32
template <typename T>
__device__ __forceinline__ void stage(float* dst, bool transposed, const T* src, int64_t stride,
                                      int width, int r0, int lim) {
    for (int i = threadIdx.x; i < BR * width; i += NT) {
        const int r = i / width, col = i % width;
        const float v = (r0 + r < lim) ? to_f32(src[static_cast<int64_t>(r0 + r) * stride + col]) : 0.0f;
        if (transposed) dst[col * BRP + r] = v;
        else dst[r * width + col] = v;
    }
}

__device__ __forceinline__ void outer4(float (&acc)[4][4], float4 a, float4 b) {
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// the sum of v over the 16 threads of a half-warp (one row group of the 16 x 16 layout)
__device__ __forceinline__ float sum16(float v) {
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Kernel A: one CTA per (b, c, h, source block s).  Rows of its outputs are the
// block's tokens s; it loops over the target blocks t >= s.
template <typename T>
__global__ void __launch_bounds__(NT) bwd_chunk_a_kernel(BwdParams bp) {
    extern __shared__ __align__(16) float sm[];
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int P = static_cast<int>(p.headdim), N = static_cast<int>(p.dstate);
    const int NB = static_cast<int>(Q / BR);
    const int64_t h = blockIdx.x / NB;
    const int ib = blockIdx.x % NB;
    const int64_t c = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int s0 = ib * BR;
    if (s0 >= Lc) return;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

    const int64_t tblk = static_cast<int64_t>(N) * BRP + BR * N + P * BRP + BR * P;
    const int64_t uni = tblk > 2 * N * P ? tblk : 2 * static_cast<int64_t>(N) * P;
    float* sBT = sm;                  // [N][BRP]  B of the source block
    float* sXT = sBT + N * BRP;       // [P][BRP]  x of the source block
    float* sU = sXT + P * BRP;
    float* sCT = sU;                  // [N][BRP]  C of the target block
    float* sC = sCT + N * BRP;        // [BR][N]
    float* sDYT = sC + BR * N;        // [P][BRP]  dy of the target block
    float* sDY = sDYT + P * BRP;      // [BR][P]
    float* sdHT = sU;                 // [N][P]    dH (after the target loop)
    float* sdH = sU + N * P;          // [P][N]
    float* sT1 = sU + uni;            // [BR][BR]  e^{cumA_t - cumA_s} C_t . B_s
    float* sT2 = sT1 + BR * BR;       // [BR][BR]  e^{cumA_t - cumA_s} dy_t . x_s
    float* scs = sT2 + BR * BR;       // [Q] cumA of the chunk
    float* sdt = scs + Q;             // [Q] dt of the chunk
    float* scol = sdt + Q;            // [16][BR] column sums of W, one row per thread row group

    const T* xb = static_cast<const T*>(p.x) + ((b * L + t0) * H + h) * P;
    const T* dyb = static_cast<const T*>(bp.dy) + ((b * L + t0) * H + h) * P;
    const T* Bb = static_cast<const T*>(p.B) + ((b * L + t0) * G + g) * N;
    const T* Cb = static_cast<const T*>(p.C) + ((b * L + t0) * G + g) * N;
    const int64_t xs = H * P, bs = G * N;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;
    for (int i = tid; i < Q; i += NT) {
        scs[i] = csc[i];
        sdt[i] = dtc[i];
    }
    stage(sBT, true, Bb, bs, N, s0, Lc);
    stage(sXT, true, xb, xs, P, s0, Lc);

    float ax[2][4][4] = {}, ab[2][4][4] = {};
    float colacc = 0.0f;  // thread tid < BR: sum over later targets of W[t, s0 + tid]
    for (int jb = ib; jb < NB; ++jb) {
        const int r0 = jb * BR;
        if (r0 >= Lc) break;
        __syncthreads();  // the previous block's readers are done
        stage(sCT, true, Cb, bs, N, r0, Lc);
        stage(sC, false, Cb, bs, N, r0, Lc);
        stage(sDYT, true, dyb, xs, P, r0, Lc);
        stage(sDY, false, dyb, xs, P, r0, Lc);
        __syncthreads();
        float t1[4][4] = {}, t2[4][4] = {};
        for (int n = 0; n < N; ++n) outer4(t1, ld4(sCT + n * BRP + ty * 4), ld4(sBT + n * BRP + tx * 4));
        for (int q = 0; q < P; ++q) outer4(t2, ld4(sDYT + q * BRP + ty * 4), ld4(sXT + q * BRP + tx * 4));
        // W[t, s] = e^{cumA_t - cumA_s} dt_s (dy_t . x_s)(C_t . B_s) for t > s: its row
        // sums (over this block's sources) and column sums (over this block's targets)
        float colp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tl = r0 + ty * 4 + i;
            float rowp = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int sl = s0 + tx * 4 + j;
                const float w = (tl >= sl && tl < Lc) ? expf(scs[tl] - scs[sl]) : 0.0f;
                t1[i][j] *= w;
                const float wst = (tl > sl) ? t1[i][j] * t2[i][j] * sdt[sl] : 0.0f;
                rowp += wst;
                colp[j] += wst;
                t2[i][j] *= w;
            }
            *reinterpret_cast<float4*>(sT1 + (ty * 4 + i) * BR + tx * 4) =
                make_float4(t1[i][0], t1[i][1], t1[i][2], t1[i][3]);
            *reinterpret_cast<float4*>(sT2 + (ty * 4 + i) * BR + tx * 4) =
                make_float4(t2[i][0], t2[i][1], t2[i][2], t2[i][3]);
            rowp = sum16(rowp);
            if (tx == 0 && tl < Lc)
                bp.roww[(((b * H + h) * NB + ib) * L) + t0 + tl] = rowp;
        }
        *reinterpret_cast<float4*>(scol + ty * BR + tx * 4) = make_float4(colp[0], colp[1], colp[2], colp[3]);
        __syncthreads();
        if (tid < BR) {
            float cs = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) cs += scol[k * BR + tid];
            colacc += cs;
        }
        const int tmax = (Lc - r0 < BR) ? Lc - r0 : BR;
        for (int t = 0; t < tmax; ++t) {
            const float4 a1 = ld4(sT1 + t * BR + ty * 4);
            const float4 a2 = ld4(sT2 + t * BR + ty * 4);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int col = 64 * k + tx * 4;
                if (col < P) outer4(ax[k], a1, ld4(sDY + t * P + col));
                if (col < N) outer4(ab[k], a2, ld4(sC + t * N + col));
            }
        }
    }
    __syncthreads();
    // the state terms, through dH = dJ/d(state leaving chunk c)
    const float* dHg = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(P) * N;
    for (int i = tid; i < P * N; i += NT) {
        const int q = i / N, n = i % N;
        const float v = dHg[i];
        sdH[q * N + n] = v;
        sdHT[n * P + q] = v;
    }
    __syncthreads();
    float wsr[4], pms[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int sl = s0 + ty * 4 + i;
        wsr[i] = (sl < Lc) ? expf(scs[Q - 1] - scs[sl]) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int col = 64 * k + tx * 4;
        if (col < P) {
            float tmp[4][4] = {};
            for (int n = 0; n < N; ++n) outer4(tmp, ld4(sBT + n * BRP + ty * 4), ld4(sdHT + n * P + col));
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float v = wsr[i] * tmp[i][j];
                    ax[k][i][j] += v;
                    pms[i] = fmaf(sXT[(col + j) * BRP + ty * 4 + i], v, pms[i]);
                }
        }
        if (col < N) {
            float tmp[4][4] = {};
            for (int q = 0; q < P; ++q) outer4(tmp, ld4(sXT + q * BRP + ty * 4), ld4(sdH + q * N + col));
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) ab[k][i][j] = fmaf(wsr[i], tmp[i][j], ab[k][i][j]);
        }
    }
    // outputs of the source rows
    const float Dh = p.D ? p.D[h] : 0.0f;
    T* dxo = static_cast<T*>(bp.dx) + ((b * L + t0) * H + h) * P;
    const int64_t tok = (b * H + h) * L + t0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i, sl = s0 + r;
        const bool valid = sl < Lc;
        const float dts = valid ? sdt[sl] : 0.0f;
        float pxd = 0.0f, pyx = 0.0f;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = 64 * k + tx * 4 + j;
                if (valid && col < P) {
                    const float dyv = to_f32(dyb[sl * xs + col]);
                    const float xv = sXT[col * BRP + r];
                    const float d = ax[k][i][j];
                    dxo[sl * xs + col] = from_f32<T>(fmaf(dts, d, Dh * dyv));
                    pxd = fmaf(xv, d, pxd);
                    pyx = fmaf(dyv, xv, pyx);
                }
                if (valid && col < N) {
                    const float v = dts * ab[k][i][j];
                    if (bp.dB_h) bp.dB_h[((b * L + t0 + sl) * H + h) * N + col] = v;
                    else static_cast<T*>(bp.dB)[((b * L + t0 + sl) * G + g) * N + col] = from_f32<T>(v);
                }
            }
        }
        pxd = sum16(pxd);
        pyx = sum16(pyx);
        const float pm = sum16(pms[i]);
        if (tx == 0 && valid) {
            bp.xdxs[tok + sl] = pxd;
            bp.dyx[tok + sl] = pyx;
            bp.mterm[tok + sl] = dts * pm;
        }
    }
    if (tid < BR && s0 + tid < Lc) bp.colw[tok + s0 + tid] = colacc;
}

// Kernel B: one CTA per (b, c, h, target block t); loops over the source
// blocks s <= t.
template <typename T>
__global__ void __launch_bounds__(NT) bwd_chunk_b_kernel(BwdParams bp) {
    extern __shared__ __align__(16) float sm[];
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int P = static_cast<int>(p.headdim), N = static_cast<int>(p.dstate);
    const int NB = static_cast<int>(Q / BR);
    const int64_t h = blockIdx.x / NB;
    const int jb = blockIdx.x % NB;
    const int64_t c = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int r0 = jb * BR;
    if (r0 >= Lc) return;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

    const int64_t sblk = static_cast<int64_t>(P) * BRP + BR * N + BR * BR;
    const int64_t uni = sblk > static_cast<int64_t>(P) * N ? sblk : static_cast<int64_t>(P) * N;
    float* sDYT = sm;                 // [P][BRP]  dy of the target block
    float* sU = sDYT + P * BRP;
    float* sXT = sU;                  // [P][BRP]  x of the source block
    float* sB = sXT + P * BRP;        // [BR][N]   B of the source block
    float* sT2T = sB + BR * N;        // [BR(s)][BR(t)] e^{cumA_t - cumA_s} dt_s dy_t . x_s
    float* sHin = sU;                 // [P][N]    state entering the chunk (after the loop)
    float* scs = sU + uni;            // [Q]
    float* sdt = scs + Q;             // [Q]

    const T* xb = static_cast<const T*>(p.x) + ((b * L + t0) * H + h) * P;
    const T* dyb = static_cast<const T*>(bp.dy) + ((b * L + t0) * H + h) * P;
    const T* Bb = static_cast<const T*>(p.B) + ((b * L + t0) * G + g) * N;
    const T* Cb = static_cast<const T*>(p.C) + ((b * L + t0) * G + g) * N;
    const int64_t xs = H * P, bs = G * N;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;
    for (int i = tid; i < Q; i += NT) {
        scs[i] = csc[i];
        sdt[i] = dtc[i];
    }
    stage(sDYT, true, dyb, xs, P, r0, Lc);

    float ac[2][4][4] = {};
    for (int ib = 0; ib <= jb; ++ib) {
        const int s0 = ib * BR;
        __syncthreads();
        stage(sXT, true, xb, xs, P, s0, Lc);
        stage(sB, false, Bb, bs, N, s0, Lc);
        __syncthreads();
        float t2[4][4] = {};
        for (int q = 0; q < P; ++q) outer4(t2, ld4(sDYT + q * BRP + ty * 4), ld4(sXT + q * BRP + tx * 4));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int sl = s0 + tx * 4 + j;
            float col[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tl = r0 + ty * 4 + i;
                const float w = (tl >= sl && tl < Lc) ? expf(scs[tl] - scs[sl]) * sdt[sl] : 0.0f;
                col[i] = t2[i][j] * w;
            }
            *reinterpret_cast<float4*>(sT2T + (tx * 4 + j) * BR + ty * 4) =
                make_float4(col[0], col[1], col[2], col[3]);
        }
        __syncthreads();
        const int smax = (Lc - s0 < BR) ? Lc - s0 : BR;
        for (int s = 0; s < smax; ++s) {
            const float4 a = ld4(sT2T + s * BR + ty * 4);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int col = 64 * k + tx * 4;
                if (col < N) outer4(ac[k], a, ld4(sB + s * N + col));
            }
        }
    }
    __syncthreads();
    // the state term e^{cumA_t} H_c^T dy_t, H_c = the state entering chunk c
    const T* Hg = static_cast<const T*>(p.states) + ((b * nc + c) * H + h) * static_cast<int64_t>(P) * N;
    for (int i = tid; i < P * N; i += NT) sHin[i] = to_f32(Hg[i]);
    __syncthreads();
    float wt[4], pq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tl = r0 + ty * 4 + i;
        wt[i] = (tl < Lc) ? expf(scs[tl]) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int col = 64 * k + tx * 4;
        if (col < N) {
            float tmp[4][4] = {};
            for (int q = 0; q < P; ++q) outer4(tmp, ld4(sDYT + q * BRP + ty * 4), ld4(sHin + q * N + col));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tl = r0 + ty * 4 + i;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float v = wt[i] * tmp[i][j];
                    ac[k][i][j] += v;
                    if (tl < Lc) pq[i] = fmaf(to_f32(Cb[tl * bs + col + j]), v, pq[i]);
                }
            }
        }
    }
    const int64_t tok = (b * H + h) * L + t0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tl = r0 + ty * 4 + i;
        const bool valid = tl < Lc;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = 64 * k + tx * 4 + j;
                if (valid && col < N) {
                    const float v = ac[k][i][j];
                    if (bp.dC_h) bp.dC_h[((b * L + t0 + tl) * H + h) * N + col] = v;
                    else static_cast<T*>(bp.dC)[((b * L + t0 + tl) * G + g) * N + col] = from_f32<T>(v);
                }
            }
        }
        const float qv = sum16(pq[i]);
        if (tx == 0 && valid) bp.qterm[tok + tl] = qv;
    }
    if (jb == 0) {
        // e^{cumA_last} <dH_c, H_c>, reduced in a fixed order
        const float* dHg = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(P) * N;
        float v = 0.0f;
        for (int i = tid; i < P * N; i += NT) v = fmaf(dHg[i], sHin[i], v);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        __shared__ float wsum[NT / 32];
        if ((tid & 31) == 0) wsum[tid >> 5] = v;
        __syncthreads();
        if (tid == 0) {
            float tot = 0.0f;
#pragma unroll
            for (int k = 0; k < NT / 32; ++k) tot += wsum[k];
            bp.k4[(b * H + h) * nc + c] = expf(scs[Q - 1]) * tot;
        }
    }
}

// ---------------------------------------------------------------------------
// The gradient of the log decay a_t, one chunk per warp:
//   da_t = e^{a_t} <g_t, h_{t-1}>
//        = k4_c + sum_{s in c, s>=t} q_s + sum_{r in c, r<t} (m_r + colw_r - roww_r)
// (g_t = dJ/dh_t; splitting g_t and h_{t-1} at the chunk's boundary gives the
// dH_c . H_c constant, the H_c . dy_s C_s^T terms q, the dH_c . x_r B_r^T terms
// m, and the pairs r < t <= s inside the chunk, W[s, r], whose sum over the
// pairs straddling t is the prefix of column-minus-row sums of W), then ddt_t,
// ddt_raw_t and the chunk's sums of dt da, dy.x and ddt_raw.  All sums run over
// one chunk at most.
constexpr int DTW = 8;  // warps per CTA of bwd_dt_kernel

// One warp per (b, h, chunk): the chunk-local pieces make chunks independent.
template <typename T>
__global__ void __launch_bounds__(DTW * 32) bwd_dt_kernel(BwdParams bp) {
    __shared__ float spre[DTW][256];  // exclusive prefix of m + colw - roww over the chunk
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int RB = bp.rblk, NB = static_cast<int>(Q / RB);
    const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * DTW + wi;  // (b * H + h) * nc + c
    if (w >= p.batch * H * nc) return;
    const int64_t bh = w / nc, c = w % nc, b = bh / H, h = bh % H;
    const float* xd = bp.xdxs + bh * L;
    const float* yx = bp.dyx + bh * L;
    const float* mt = bp.mterm + bh * L;
    const float* qt = bp.qterm + bh * L;
    const float* cw = bp.colw + bh * L;
    const float* rw = bp.roww + bh * NB * L;
    const float* dtw = p.dt + bh * nc * Q;
    const float Ah = p.A[h], bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
    const T* dtr = static_cast<const T*>(p.dt_raw);
    T* ddt = static_cast<T*>(bp.ddt);
    float* pre = spre[wi];
    float sA = 0.0f, sD = 0.0f, sb = 0.0f;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    float carry = 0.0f;
    for (int l0 = 0; l0 < Lc; l0 += 32) {
        const int l = l0 + lane;
        float v = 0.0f;
        if (l < Lc) {
            const int64_t t = t0 + l;
            float rsum = 0.0f;
            for (int i = 0; i <= l / RB; ++i) rsum += rw[i * L + t];
            v = mt[t] + cw[t] - rsum;
        }
        float incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (l < Lc) pre[l] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    const float k4 = bp.k4[w];
    carry = 0.0f;
    for (int l0 = ((Lc - 1) / 32) * 32; l0 >= 0; l0 -= 32) {
        const int l = l0 + lane;
        const int64_t t = t0 + l;
        float v = (l < Lc) ? qt[t] : 0.0f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_down_sync(0xffffffffu, v, off);
            if (lane + off < 32) v += o;
        }
        if (l < Lc) {
            const float da = k4 + carry + v + pre[l];
            const float dtv = dtw[c * Q + l];
            const float ddtv = fmaf(Ah, da, xd[t]);
            const float u = to_f32(dtr[(b * L + t) * H + h]) + bias;
            const float dr = ddtv / (1.0f + expf(-u));
            ddt[(b * L + t) * H + h] = from_f32<T>(dr);
            sA = fmaf(dtv, da, sA);
            sD += yx[t];
            sb += dr;
        }
        carry += __shfl_sync(0xffffffffu, v, 0);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sA += __shfl_xor_sync(0xffffffffu, sA, off);
        sD += __shfl_xor_sync(0xffffffffu, sD, off);
        sb += __shfl_xor_sync(0xffffffffu, sb, off);
    }
    if (lane == 0) {
        bp.partial[w * 3 + 0] = sA;
        bp.partial[w * 3 + 1] = sD;
        bp.partial[w * 3 + 2] = sb;
    }
}

// Sums over batch rows (dA, dD, ddt_bias) and, when heads share groups, over
// the heads of each group (dB, dC), in a fixed order.
template <typename T>
__global__ void __launch_bounds__(256) bwd_finish_kernel(BwdParams bp) {
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, N = p.dstate, L = p.seqlen;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < H) {
        float sA = 0.0f, sD = 0.0f, sb = 0.0f;
        const int64_t nc = p.nchunks;
        for (int64_t b = 0; b < p.batch; ++b)
            for (int64_t c = 0; c < nc; ++c) {
                const float* pp = bp.partial + ((b * H + i) * nc + c) * 3;
                sA += pp[0];
                sD += pp[1];
                sb += pp[2];
            }
        bp.dA[i] = sA;
        if (bp.dD) bp.dD[i] = sD;
        if (bp.ddt_bias) bp.ddt_bias[i] = sb;
    }
    if (!bp.dB_h) return;
    const int64_t hpg = p.heads_per_group;
    const int64_t total = p.batch * L * G * N;
    for (int64_t e = i; e < total; e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t n = e % N, bg = e / N, g = bg % G, bt = bg / G;  // bt = b * L + t
        const int64_t base = (bt * H + g * hpg) * N + n;
        float sbv = 0.0f, scv = 0.0f;
        for (int64_t k = 0; k < hpg; ++k) {
            sbv += bp.dB_h[base + k * N];
            scv += bp.dC_h[base + k * N];
        }
        static_cast<T*>(bp.dB)[e] = from_f32<T>(sbv);
        static_cast<T*>(bp.dC)[e] = from_f32<T>(scv);
    }
}

}  // namespace

// Shared memory the per-chunk kernels need for this shape (bytes).
size_t bwd_smem_bytes(int64_t headdim, int64_t dstate, int64_t chunk) {
    const int64_t a = smem_a_floats(headdim, dstate, chunk), b = smem_b_floats(headdim, dstate, chunk);
    return static_cast<size_t>(a > b ? a : b) * sizeof(float);
}

template <typename T>
cudaError_t launch_ssd_bwd(const BwdParams& bp, cudaStream_t s) {
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, P = p.headdim, N = p.dstate, nc = p.nchunks;
    cudaError_t e;
    if (bp.rblk == 128) {
        if ((e = launch_bwd_tc_dstate(bp, s)) != cudaSuccess) return e;
    } else {
        const unsigned tiles = static_cast<unsigned>(((P + DP - 1) / DP) * ((N + DN - 1) / DN));
        dim3 grid(static_cast<unsigned>(nc * H), tiles, static_cast<unsigned>(p.batch));
        bwd_dstate_kernel<T><<<grid, 256, 0, s>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int64_t n = p.batch * H * P * N / 4;
        bwd_state_passing_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (bp.rblk == 128) {
        if ((e = launch_bwd_tc(bp, s)) != cudaSuccess) return e;
    } else {
        const size_t sa = static_cast<size_t>(smem_a_floats(P, N, p.chunk)) * sizeof(float);
        const size_t sb = static_cast<size_t>(smem_b_floats(P, N, p.chunk)) * sizeof(float);
        if ((e = cudaFuncSetAttribute(bwd_chunk_a_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(sa))) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(bwd_chunk_b_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(sb))) != cudaSuccess)
            return e;
        dim3 grid(static_cast<unsigned>(H * (p.chunk / BR)), static_cast<unsigned>(nc),
                  static_cast<unsigned>(p.batch));
        bwd_chunk_a_kernel<T><<<grid, NT, sa, s>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        bwd_chunk_b_kernel<T><<<grid, NT, sb, s>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int64_t warps = p.batch * H * nc;
        bwd_dt_kernel<T><<<static_cast<unsigned>((warps + DTW - 1) / DTW), DTW * 32, 0, s>>>(bp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        int64_t n = bp.dB_h ? p.batch * p.seqlen * p.ngroups * N : H;
        if (n < H) n = H;
        int64_t blocks = (n + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        bwd_finish_kernel<T><<<static_cast<unsigned>(blocks), 256, 0, s>>>(bp);
        e = cudaGetLastError();
    }
    return e;
}

template cudaError_t launch_ssd_bwd<float>(const BwdParams&, cudaStream_t);
template cudaError_t launch_ssd_bwd<__nv_bfloat16>(const BwdParams&, cudaStream_t);

}  // namespace ssd
