// state_update.cu -- the single-token decode step against a carried fp32
// state (the SSM half of the Mamba2Cache of "MAMBA-2 Reference
// Implementations Comparison", section 1.3; the recurrence of section 3.2
// applied to one token):
//
//   dt = softplus(dt_raw + dt_bias_h);  a = exp(dt A_h)
//   h[p,n] <- a h[p,n] + dt x[p] B[n];   y[p] = sum_n h[p,n] C[n] + D_h x[p]
//
// Bandwidth-bound: the state is read once and written once, in place.  One
// CTA of four warps owns one (batch, head) state tile [P x N]; a state row is
// spread over TPR lanes holding 4 V consecutive floats each, a warp covers
// RPW rows per pass, and every thread issues the 16-byte loads of MAXPASS
// passes before their arithmetic.  Four passes keep the kernel at 55
// registers, so many small CTAs share an SM and one CTA's loads overlap
// another's stores (measured: 4 passes x 128 threads streams at the copy
// bandwidth; 8 passes x 256 threads, at 86 registers, reached 74% of it).
// The state stream is marked evict-first (ld/st .cs) so it does not push
// B/C/x out of L2.  dt, the decay and B/C are computed or loaded once per
// thread, and the C-dot of each row is reduced with xor shuffles inside its
// lane group.
#include "internal.cuh"

namespace ssd {
namespace {

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ void load(const float* p, float v[4]) {
        const float4 q = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float v[4]) {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
};

constexpr int MAXPASS = 4;
constexpr int NTHREADS = 128;

template <typename T, int N>
__global__ void __launch_bounds__(NTHREADS) state_update_kernel(DecodeParams p) {
    constexpr int TPR = (N / 4 < 32) ? N / 4 : 32;  // threads per state row
    constexpr int V = N / (4 * TPR);                // float4s per thread per row
    constexpr int RPW = 32 / TPR;                   // rows per warp per pass
    constexpr int RPP = (NTHREADS / 32) * RPW;      // rows per CTA pass
    static_assert(TPR * V * 4 == N && RPW * TPR == 32, "bad tiling");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / TPR, tl = lane % TPR;
    const int64_t bh = blockIdx.x, H = p.nheads, P = p.headdim;
    const int64_t b = bh / H, h = bh % H, g = h / p.heads_per_group;

    const float dt = softplus_f32(to_f32(static_cast<const T*>(p.dt_raw)[bh]) +
                                  (p.dt_bias ? p.dt_bias[h] : 0.0f));
    const float a = expf(dt * p.A[h]);
    const float Dh = p.D ? p.D[h] : 0.0f;
    float bv[V][4], cv[V][4];
    const T* Bp = static_cast<const T*>(p.B) + (b * p.ngroups + g) * N + tl * 4 * V;
    const T* Cp = static_cast<const T*>(p.C) + (b * p.ngroups + g) * N + tl * 4 * V;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        Vec4<T>::load(Bp + 4 * v, bv[v]);
        Vec4<T>::load(Cp + 4 * v, cv[v]);
    }
    const T* xg = static_cast<const T*>(p.x) + bh * P;
    T* yg = static_cast<T*>(p.y) + bh * P;
    const T* zg = p.z ? static_cast<const T*>(p.z) + bh * P : nullptr;  // output gate
    float* st = p.state + bh * P * N;

    for (int64_t p0 = 0; p0 < P; p0 += MAXPASS * RPP) {
        float4 s[MAXPASS][V];
        float xv[MAXPASS];
#pragma unroll
        for (int ps = 0; ps < MAXPASS; ++ps) {
            const int64_t row = p0 + ps * RPP + warp * RPW + sub;
            if (row < P) {
                const float4* sp = reinterpret_cast<const float4*>(st + row * N) + tl * V;
#pragma unroll
                for (int v = 0; v < V; ++v) s[ps][v] = __ldcs(sp + v);
                xv[ps] = to_f32(xg[row]);
            }
        }
#pragma unroll
        for (int ps = 0; ps < MAXPASS; ++ps) {
            const int64_t row = p0 + ps * RPP + warp * RPW + sub;
            const bool valid = row < P;
            const float xdt = valid ? dt * xv[ps] : 0.0f;
            float acc = 0.0f;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float4& q = s[ps][v];
                q.x = fmaf(a, q.x, xdt * bv[v][0]);
                q.y = fmaf(a, q.y, xdt * bv[v][1]);
                q.z = fmaf(a, q.z, xdt * bv[v][2]);
                q.w = fmaf(a, q.w, xdt * bv[v][3]);
                acc = fmaf(q.x, cv[v][0], acc);
                acc = fmaf(q.y, cv[v][1], acc);
                acc = fmaf(q.z, cv[v][2], acc);
                acc = fmaf(q.w, cv[v][3], acc);
            }
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (valid) {
                float4* sp = reinterpret_cast<float4*>(st + row * N) + tl * V;
#pragma unroll
                for (int v = 0; v < V; ++v) __stcs(sp + v, s[ps][v]);
                if (tl == 0) {
                    const float v = acc + Dh * xv[ps];
                    yg[row] = from_f32<T>(zg ? v * silu_f32(to_f32(zg[row])) : v);
                }
            }
        }
    }
}

template <typename T, int N>
cudaError_t launch_n(const DecodeParams& p, cudaStream_t s) {
    state_update_kernel<T, N><<<static_cast<unsigned>(p.batch * p.nheads), NTHREADS, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_state_update(const DecodeParams& p, cudaStream_t s) {
    switch (p.dstate) {
        case 16: return launch_n<T, 16>(p, s);
        case 32: return launch_n<T, 32>(p, s);
        case 64: return launch_n<T, 64>(p, s);
        case 128: return launch_n<T, 128>(p, s);
        case 256: return launch_n<T, 256>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

template cudaError_t launch_state_update<float>(const DecodeParams&, cudaStream_t);
template cudaError_t launch_state_update<__nv_bfloat16>(const DecodeParams&, cudaStream_t);

}  // namespace ssd
