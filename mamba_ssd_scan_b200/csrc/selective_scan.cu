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
// broadcasts.  The decode step (sel_update_split_kernel for N = 8, 16, 32,
// sel_update_kernel otherwise) applies the recurrence once to a carried state
// [b, channels, N].
#include "internal.cuh"

namespace ssd {
namespace {

// threads (channels) per CTA; with dstate <= 16 at most 80 registers each keeps 6
// CTAs (24 warps) per SM, which measured faster than fewer, larger-register CTAs
constexpr int CT = 128;

__device__ __forceinline__ float ex2f(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr int TU = 4;  // tokens whose x and dt loads are in flight together

// x and dt of one channel for TU tokens at a time: the next group's loads go
// out when the current group is taken, so they overlap its arithmetic.
template <typename T>
struct TokenQueue {
    const T* x;
    const T* dt;
    int64_t stride;
    int n;
    float nx[TU], nd[TU];
    __device__ __forceinline__ TokenQueue(const T* x_, const T* dt_, int64_t stride_, int n_)
        : x(x_), dt(dt_), stride(stride_), n(n_) {
        load(0);
    }
    __device__ __forceinline__ void load(int t0) {
#pragma unroll
        for (int u = 0; u < TU; ++u) {
            const bool ok = t0 + u < n;
            nx[u] = ok ? to_f32(x[(t0 + u) * stride]) : 0.0f;
            nd[u] = ok ? to_f32(dt[(t0 + u) * stride]) : 0.0f;
        }
    }
    __device__ __forceinline__ void take(int t0, float (&xv)[TU], float (&dv)[TU]) {
#pragma unroll
        for (int u = 0; u < TU; ++u) {
            xv[u] = nx[u];
            dv[u] = nd[u];
        }
        if (t0 + TU < n) load(t0 + TU);
    }
};

template <typename T, int N>
__global__ void __launch_bounds__(CT, N <= 16 ? 6 : 3) sel_local_kernel(SelParams p) {
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
    TokenQueue<T> qx(xg, dg, Dc, Lc);
    for (int t0g = 0; t0g < Lc; t0g += TU) {
        float xv[TU], dv[TU];
        qx.take(t0g, xv, dv);
#pragma unroll
        for (int u = 0; u < TU; ++u) {
            const int t = t0g + u;
            if (t < Lc) {
                const float dt = softplus_f32(dv[u] + bias);
                const float dx = dt * xv[u];
                sdt += dt;
                const float* bt = sb + t * N;
#pragma unroll
                for (int n = 0; n < N; ++n) h[n] = fmaf(ex2f(dt * a2[n]), h[n], dx * bt[n]);
            }
        }
    }
    float4* out = reinterpret_cast<float4*>(p.S + ((b * nc + c) * Dc + d) * N);
#pragma unroll
    for (int n = 0; n < N; n += 4) out[n / 4] = make_float4(h[n], h[n + 1], h[n + 2], h[n + 3]);
    p.sdt[(b * nc + c) * Dc + d] = sdt;
}

// One thread per 4 states of one (b, d): H_{c} (entering chunk c) in place of
// the local state S_c, the final state after the last chunk.  The loads of
// CU chunks (independent of the carry) go out before their multiply-adds.
constexpr int CU = 8;

__global__ void __launch_bounds__(256) sel_carry_kernel(SelParams p) {
    const int64_t Dc = p.channels, N = p.dstate, nc = p.nchunks;
    const int64_t nv = N / 4;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= p.batch * Dc * nv) return;
    const int64_t bd = e / nv, q = e % nv, b = bd / Dc, d = bd % Dc;
    float4 carry = p.init_state ? reinterpret_cast<const float4*>(p.init_state)[e]
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float4 a = reinterpret_cast<const float4*>(p.A + d * N)[q];
    float4* sbase = reinterpret_cast<float4*>(p.S + (b * nc * Dc + d) * N) + q;
    const int64_t cstride = Dc * nv;  // float4s between consecutive chunks
    const float* sdt = p.sdt + b * nc * Dc + d;
    for (int64_t c0 = 0; c0 < nc; c0 += CU) {
        float4 sv[CU];
        float st[CU];
#pragma unroll
        for (int u = 0; u < CU; ++u) {
            if (c0 + u < nc) {
                sv[u] = sbase[(c0 + u) * cstride];
                st[u] = sdt[(c0 + u) * Dc];
            }
        }
#pragma unroll
        for (int u = 0; u < CU; ++u) {
            if (c0 + u < nc) {
                sbase[(c0 + u) * cstride] = carry;
                carry.x = fmaf(expf(a.x * st[u]), carry.x, sv[u].x);
                carry.y = fmaf(expf(a.y * st[u]), carry.y, sv[u].y);
                carry.z = fmaf(expf(a.z * st[u]), carry.z, sv[u].z);
                carry.w = fmaf(expf(a.w * st[u]), carry.w, sv[u].w);
            }
        }
    }
    if (p.final_state) reinterpret_cast<float4*>(p.final_state)[e] = carry;
}

template <typename T, int N>
__global__ void __launch_bounds__(CT, N <= 16 ? 6 : 3) sel_output_kernel(SelParams p) {
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
    TokenQueue<T> qx(xg, dg, Dc, Lc);
    for (int t0g = 0; t0g < Lc; t0g += TU) {
        float xv[TU], dv[TU];
        qx.take(t0g, xv, dv);
#pragma unroll
        for (int u = 0; u < TU; ++u) {
            const int t = t0g + u;
            if (t < Lc) {
                const float dt = softplus_f32(dv[u] + bias);
                const float dx = dt * xv[u];
                const float* bt = sb + t * N;
                const float* ct = sc + t * N;
                float acc = 0.0f;
#pragma unroll
                for (int n = 0; n < N; ++n) {
                    h[n] = fmaf(ex2f(dt * a2[n]), h[n], dx * bt[n]);
                    acc = fmaf(ct[n], h[n], acc);
                }
                yg[t * Dc] = from_f32<T>(fmaf(Dd, xv[u], acc));
            }
        }
    }
}

// Decode: one thread per (b, d), its N states and A row moved as 16-byte
// vectors, B and C of the batch row as 4-element vectors.  Consecutive steps
// go out with programmatic dependent launch (wait for the previous step's
// state, then let the next step's CTAs in).
template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float* p) {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
};

template <typename T, int N>
__global__ void __launch_bounds__(256) sel_update_kernel(SelParams p) {
    const int64_t Dc = p.channels;
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= p.batch * Dc) return;
    const int64_t b = e / Dc, d = e % Dc;
    grid_dep_wait();
    grid_dep_launch();
    float4* sp = reinterpret_cast<float4*>(p.S + e * N);
    const float4* ap = reinterpret_cast<const float4*>(p.A + d * N);
    const T* Bg = static_cast<const T*>(p.B) + b * N;
    const T* Cg = static_cast<const T*>(p.C) + b * N;
    // every load first (the stores below could alias them for the compiler),
    // then the arithmetic, then the stores
    float4 hv[N / 4], av[N / 4], bv[N / 4], cv[N / 4];
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
        hv[q] = sp[q];
        av[q] = __ldg(ap + q);
        bv[q] = Vec4<T>::load(Bg + 4 * q);
        cv[q] = Vec4<T>::load(Cg + 4 * q);
    }
    const float xv = to_f32(static_cast<const T*>(p.x)[e]);
    const float dt = softplus_f32(to_f32(static_cast<const T*>(p.dt_raw)[e]) +
                                  (p.dt_bias ? p.dt_bias[d] : 0.0f));
    const float Dd = p.D ? p.D[d] : 0.0f;
    const float dx = dt * xv, dl = dt * kLog2e;
    float acc = 0.0f;
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
        float4& h = hv[q];
        h.x = fmaf(ex2f(dl * av[q].x), h.x, dx * bv[q].x);
        h.y = fmaf(ex2f(dl * av[q].y), h.y, dx * bv[q].y);
        h.z = fmaf(ex2f(dl * av[q].z), h.z, dx * bv[q].z);
        h.w = fmaf(ex2f(dl * av[q].w), h.w, dx * bv[q].w);
        acc = fmaf(cv[q].x, h.x, acc);
        acc = fmaf(cv[q].y, h.y, acc);
        acc = fmaf(cv[q].z, h.z, acc);
        acc = fmaf(cv[q].w, h.w, acc);
    }
#pragma unroll
    for (int q = 0; q < N / 4; ++q) sp[q] = hv[q];
    static_cast<T*>(p.y)[e] = from_f32<T>(fmaf(Dd, xv, acc));
}

// The decode step with a (batch, channel)'s N states split over N / 4 lanes
// (N = 8, 16 or 32), one float4 of state each, so that a warp's state loads and
// stores are contiguous and a step has N / 4 times as many threads to hide
// their latency; the lanes' parts of C . h are summed by a shuffle.  Every
// lane takes part in the shuffle; only live lanes load and store.
template <typename T, int N>
__global__ void __launch_bounds__(256) sel_update_split_kernel(SelParams p) {
    constexpr int TPE = N / 4;                       // lanes per (batch, channel)
    static_assert(TPE == 2 || TPE == 4 || TPE == 8, "power-of-two split");
    const int64_t Dc = p.channels, n = p.batch * Dc;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t e = tid / TPE;
    const int j = static_cast<int>(tid % TPE);
    const bool live = e < n;
    const int64_t b = live ? e / Dc : 0, d = live ? e % Dc : 0;
    grid_dep_wait();
    grid_dep_launch();
    float4* sp = reinterpret_cast<float4*>(p.S) + e * TPE + j;
    float4 hv = make_float4(0.0f, 0.0f, 0.0f, 0.0f), av = hv, bv = hv, cv = hv;
    float xv = 0.0f, dr = 0.0f, bias = 0.0f, Dd = 0.0f;
    if (live) {
        hv = *sp;
        av = __ldg(reinterpret_cast<const float4*>(p.A + d * N) + j);
        bv = Vec4<T>::load(static_cast<const T*>(p.B) + b * N + 4 * j);
        cv = Vec4<T>::load(static_cast<const T*>(p.C) + b * N + 4 * j);
        xv = to_f32(static_cast<const T*>(p.x)[e]);
        dr = to_f32(static_cast<const T*>(p.dt_raw)[e]);
        bias = p.dt_bias ? p.dt_bias[d] : 0.0f;
        Dd = p.D ? p.D[d] : 0.0f;
    }
    const float dt = softplus_f32(dr + bias);
    const float dx = dt * xv, dl = dt * kLog2e;
    hv.x = fmaf(ex2f(dl * av.x), hv.x, dx * bv.x);
    hv.y = fmaf(ex2f(dl * av.y), hv.y, dx * bv.y);
    hv.z = fmaf(ex2f(dl * av.z), hv.z, dx * bv.z);
    hv.w = fmaf(ex2f(dl * av.w), hv.w, dx * bv.w);
    float acc = fmaf(cv.x, hv.x, fmaf(cv.y, hv.y, fmaf(cv.z, hv.z, cv.w * hv.w)));
#pragma unroll
    for (int o = TPE / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (live) {
        *sp = hv;
        if (j == 0) static_cast<T*>(p.y)[e] = from_f32<T>(fmaf(Dd, xv, acc));
    }
}

template <typename T, int N>
cudaError_t launch_n(const SelParams& p, bool update, cudaStream_t s) {
    if (update) {
        const int64_t n = p.batch * p.channels;
        if constexpr (N == 8 || N == 16 || N == 32) {
            const int64_t threads = n * (N / 4);
            return launch_kernel(sel_update_split_kernel<T, N>,
                                 dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, s,
                                 true, p);
        }
        return launch_kernel(sel_update_kernel<T, N>, dim3(static_cast<unsigned>((n + 255) / 256)),
                             dim3(256), 0, s, true, p);
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
