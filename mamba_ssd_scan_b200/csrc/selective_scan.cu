// selective_scan.cu -- the selective scan with a diagonal A per channel and
// state (the Mamba-1 form the page "MAMBA-2 Reference Implementations
// Comparison" sets beside SSD in section 2.3; A_log [d_inner, d_state] in the
// block parameter list of section 1.3; dt per channel and B * dt as the input
// term in "MAMBA-2 Implementation Gaps", Gap 3):
//
//   dt_t[d]  = softplus(dt_raw_t[d] + dt_bias[d])
//   h_t[d,n] = exp(dt_t[d] A[d,n]) h_{t-1}[d,n] + dt_t[d] B_t[n] x_t[d]
//   y_t[d]   = sum_n C_t[n] h_t[d,n] + D[d] x_t[d]
//
// A differs per state, so there is no matrix form for the tensor cores: the
// work is one exponential and two multiply-adds per (token, channel, state),
// streamed.  The sequence is cut into chunks for parallelism, in three
// kernels: each chunk's local state from zero (sel_local_kernel), the carry
// across chunks (sel_carry_kernel; a chunk's decay is exp(A[d,n] * sum of its
// dt), so one dt sum per channel and chunk is all it needs), and the outputs,
// each chunk replayed from the state entering it (sel_output_kernel).  One
// thread per channel, its N states in registers; the chunk's B and C rows
// (shared by every channel) are staged in shared memory and read as
// broadcasts.  The decode step (sel_update_kernel) applies the recurrence
// once to a carried state [b, channels, N].
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int CT = 128;  // threads (channels) per CTA

__device__ __forceinline__ float ex2f(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int N>
__global__ void __launch_bounds__(CT) sel_local_kernel(SelParams p) {
    extern __shared__ __align__(16) float sb[];  // [chunk][N] B rows of the chunk
    const int64_t L = p.seqlen, Dc = p.channels, Q = p.chunk, nc = p.nchunks;
    const int64_t c = blockIdx.y, b = blockIdx.z, t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int64_t d = static_cast<int64_t>(blockIdx.x) * CT + threadIdx.x;
    const T* Bg = static_cast<const T*>(p.B) + (b * L + t0) * N;
    for (int i = threadIdx.x; i < Lc * N; i += CT) sb[i] = to_f32(Bg[i]);
    __syncthreads();
    if (d >= Dc) return;
    float a2[N], h[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        a2[n] = p.A[d * N + n] * kLog2e;
        h[n] = 0.0f;
    }
    const float bias = p.dt_bias ? p.dt_bias[d] : 0.0f;
    const T* xg = static_cast<const T*>(p.x) + (b * L + t0) * Dc + d;
    const T* dg = static_cast<const T*>(p.dt_raw) + (b * L + t0) * Dc + d;
    float sdt = 0.0f;
    for (int t = 0; t < Lc; ++t) {
        const float dt = softplus_f32(to_f32(dg[t * Dc]) + bias);
        const float dx = dt * to_f32(xg[t * Dc]);
        sdt += dt;
        const float* bt = sb + t * N;
#pragma unroll
        for (int n = 0; n < N; ++n) h[n] = fmaf(ex2f(dt * a2[n]), h[n], dx * bt[n]);
    }
    float4* out = reinterpret_cast<float4*>(p.S + ((b * nc + c) * Dc + d) * N);
#pragma unroll
    for (int n = 0; n < N; n += 4) out[n / 4] = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
    p.sdt[(b * nc + c) * Dc + d] = sdt;
}

// One thread per 4 states of one (b, d): H_{c} (entering chunk c) in place of
// the local state S_c, the final state after the last chunk.
__global__ void __launch_bounds__(256) sel_carry_kernel(SelParams p) {
    const int64_t Dc = p.channels, N = p.dstate, nc = p.nchunks;
    const int64_t nv = N / 4;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= p.batch * Dc * nv) return;
    const int64_t bd = e / nv, q = e % nv, b = bd / Dc, d = bd % Dc;
    float4 carry = p.init_state ? reinterpret_cast<const float4*>(p.init_state)[e]
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float4 a = reinterpret_cast<const float4*>(p.A + d * N)[q];
    for (int64_t c = 0; c < nc; ++c) {
        float4* sp = reinterpret_cast<float4*>(p.S + ((b * nc + c) * Dc + d) * N) + q;
        const float4 s = *sp;
        const float st = p.sdt[(b * nc + c) * Dc + d];
        *sp = carry;
        carry.x = fmaf(expf(a.x * st), carry.x, s.x);
        carry.y = fmaf(expf(a.y * st), carry.y, s.y);
        carry.z = fmaf(expf(a.z * st), carry.z, s.z);
        carry.w = fmaf(expf(a.w * st), carry.w, s.w);
    }
    if (p.final_state) reinterpret_cast<float4*>(p.final_state)[e] = carry;
}

template <typename T, int N>
__global__ void __launch_bounds__(CT) sel_output_kernel(SelParams p) {
    extern __shared__ __align__(16) float sbc[];  // [chunk][N] B rows, then [chunk][N] C rows
    const int64_t L = p.seqlen, Dc = p.channels, Q = p.chunk, nc = p.nchunks;
    const int64_t c = blockIdx.y, b = blockIdx.z, t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int64_t d = static_cast<int64_t>(blockIdx.x) * CT + threadIdx.x;
    float* sb = sbc;
    float* sc = sbc + Q * N;
    const T* Bg = static_cast<const T*>(p.B) + (b * L + t0) * N;
    const T* Cg = static_cast<const T*>(p.C) + (b * L + t0) * N;
    for (int i = threadIdx.x; i < Lc * N; i += CT) {
        sb[i] = to_f32(Bg[i]);
        sc[i] = to_f32(Cg[i]);
    }
    __syncthreads();
    if (d >= Dc) return;
    float a2[N], h[N];
    const float4* hin = reinterpret_cast<const float4*>(p.S + ((b * nc + c) * Dc + d) * N);
#pragma unroll
    for (int n = 0; n < N; n += 4) {
        const float4 v = hin[n / 4];
        h[n] = v.x; h[n + 1] = v.y; h[n + 2] = v.z; h[n + 3] = v.w;
    }
#pragma unroll
    for (int n = 0; n < N; ++n) a2[n] = p.A[d * N + n] * kLog2e;
    const float bias = p.dt_bias ? p.dt_bias[d] : 0.0f;
    const float Dd = p.D ? p.D[d] : 0.0f;
    const T* xg = static_cast<const T*>(p.x) + (b * L + t0) * Dc + d;
    const T* dg = static_cast<const T*>(p.dt_raw) + (b * L + t0) * Dc + d;
    T* yg = static_cast<T*>(p.y) + (b * L + t0) * Dc + d;
    for (int t = 0; t < Lc; ++t) {
        const float xv = to_f32(xg[t * Dc]);
        const float dt = softplus_f32(to_f32(dg[t * Dc]) + bias);
        const float dx = dt * xv;
        const float* bt = sb + t * N;
        const float* ct = sc + t * N;
        float acc = 0.0f;
#pragma unroll
        for (int n = 0; n < N; ++n) {
            h[n] = fmaf(ex2f(dt * a2[n]), h[n], dx * bt[n]);
            acc = fmaf(ct[n], h[n], acc);
        }
        yg[t * Dc] = from_f32<T>(fmaf(Dd, xv, acc));
    }
}

// Decode: one thread per (b, d), its N states moved as 16-byte vectors.
template <typename T, int N>
__global__ void __launch_bounds__(256) sel_update_kernel(SelParams p) {
    const int64_t Dc = p.channels;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= p.batch * Dc) return;
    const int64_t b = e / Dc, d = e % Dc;
    float4* sp = reinterpret_cast<float4*>(p.S + e * N);
    float h[N];
#pragma unroll
    for (int n = 0; n < N; n += 4) {
        const float4 v = sp[n / 4];
        h[n] = v.x; h[n + 1] = v.y; h[n + 2] = v.z; h[n + 3] = v.w;
    }
    const float xv = to_f32(static_cast<const T*>(p.x)[e]);
    const float dt = softplus_f32(to_f32(static_cast<const T*>(p.dt_raw)[e]) +
                                  (p.dt_bias ? p.dt_bias[d] : 0.0f));
    const float dx = dt * xv;
    const T* Bg = static_cast<const T*>(p.B) + b * N;
    const T* Cg = static_cast<const T*>(p.C) + b * N;
    float acc = 0.0f;
#pragma unroll
    for (int n = 0; n < N; ++n) {
        h[n] = fmaf(ex2f(dt * p.A[d * N + n] * kLog2e), h[n], dx * to_f32(Bg[n]));
        acc = fmaf(to_f32(Cg[n]), h[n], acc);
    }
#pragma unroll
    for (int n = 0; n < N; n += 4) sp[n / 4] = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
    static_cast<T*>(p.y)[e] = from_f32<T>(fmaf(p.D ? p.D[d] : 0.0f, xv, acc));
}

template <typename T, int N>
cudaError_t launch_n(const SelParams& p, bool update, cudaStream_t s) {
    if (update) {
        const int64_t n = p.batch * p.channels;
        sel_update_kernel<T, N><<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    const dim3 grid(static_cast<unsigned>((p.channels + CT - 1) / CT),
                    static_cast<unsigned>(p.nchunks), static_cast<unsigned>(p.batch));
    const size_t sm1 = static_cast<size_t>(p.chunk) * N * sizeof(float);
    sel_local_kernel<T, N><<<grid, CT, sm1, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t nv = p.batch * p.channels * N / 4;
    sel_carry_kernel<<<static_cast<unsigned>((nv + 255) / 256), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    sel_output_kernel<T, N><<<grid, CT, 2 * sm1, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_selective_scan(const SelParams& p, bool update, cudaStream_t s) {
    switch (p.dstate) {
        case 4: return launch_n<T, 4>(p, update, s);
        case 8: return launch_n<T, 8>(p, update, s);
        case 12: return launch_n<T, 12>(p, update, s);
        case 16: return launch_n<T, 16>(p, update, s);
        case 20: return launch_n<T, 20>(p, update, s);
        case 24: return launch_n<T, 24>(p, update, s);
        case 28: return launch_n<T, 28>(p, update, s);
        case 32: return launch_n<T, 32>(p, update, s);
        default: return cudaErrorInvalidValue;
    }
}

template cudaError_t launch_selective_scan<float>(const SelParams&, bool, cudaStream_t);
template cudaError_t launch_selective_scan<__nv_bfloat16>(const SelParams&, bool, cudaStream_t);

}  // namespace ssd
