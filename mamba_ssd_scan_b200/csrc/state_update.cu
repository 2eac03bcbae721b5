// state_update.cu -- the single-token decode step against a carried fp32
// state (the SSM half of the Mamba2Cache of "MAMBA-2 Reference
// Implementations Comparison", section 1.3; the recurrence of section 3.2
// applied to one token):
//
//   dt = softplus(dt_raw + dt_bias_h);  a = exp(dt A_h)
//   h[p,n] <- a h[p,n] + dt x[p] B[n];   y[p] = sum_n h[p,n] C[n] + D_h x[p]
//
// Bandwidth-bound: the state is read once and written once, in place, with
// 16-byte vector accesses marked streaming (evict-first) so the state stream
// does not push the small, reused B/C/x lines out of L2.  A state row (one p,
// all n) is spread over TPR = N/VEC consecutive lanes holding VEC floats each;
// the C-dot is reduced with xor shuffles inside the lane group.  Every warp
// takes ROWS rows per pass with all loads issued before any math, so each SM
// keeps ~64 KB of state reads in flight.
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
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
        const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
};

template <typename T, int N>
__global__ void __launch_bounds__(256) state_update_kernel(DecodeParams p) {
    constexpr int VEC = (N > 128) ? N / 32 : 4;  // floats per thread
    constexpr int TPR = N / VEC;                  // threads per state row
    constexpr int RPW = 32 / TPR;                 // rows per warp per sub-pass
    constexpr int ROWS = 2;                       // sub-passes in flight per warp
    static_assert(VEC % 4 == 0 && TPR * VEC == N && RPW * TPR == 32, "bad tiling");

    const int lane = threadIdx.x & 31, sub = lane / TPR, tl = lane % TPR;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nrows = p.batch * p.nheads * p.headdim;
    const int64_t H = p.nheads, P = p.headdim;
    const T* xg = static_cast<const T*>(p.x);
    const T* dtg = static_cast<const T*>(p.dt_raw);
    const T* Bg = static_cast<const T*>(p.B);
    const T* Cg = static_cast<const T*>(p.C);

    float4 s[ROWS][VEC / 4];
    int64_t row[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        row[r] = (warp * ROWS + r) * RPW + sub;
#pragma unroll
        for (int v = 0; v < VEC / 4; ++v) s[r][v] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row[r] < nrows) {
            const float4* sp = reinterpret_cast<const float4*>(p.state + row[r] * N) + tl * (VEC / 4);
#pragma unroll
            for (int v = 0; v < VEC / 4; ++v) s[r][v] = __ldcs(sp + v);
        }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const bool valid = row[r] < nrows;
        const int64_t rr = valid ? row[r] : 0;
        const int64_t bh = rr / P, b = bh / H, h = bh % H;
        const int64_t g = h / p.heads_per_group;
        const float dt = softplus_f32(to_f32(dtg[bh]) + (p.dt_bias ? p.dt_bias[h] : 0.0f));
        const float a = expf(dt * p.A[h]);
        const float xv = to_f32(xg[rr]);
        const float xdt = dt * xv;
        const T* Bp = Bg + (b * p.ngroups + g) * N + tl * VEC;
        const T* Cp = Cg + (b * p.ngroups + g) * N + tl * VEC;
        float acc = 0.0f;
#pragma unroll
        for (int v = 0; v < VEC / 4; ++v) {
            float bv[4], cv[4];
            Vec4<T>::load(Bp + v * 4, bv);
            Vec4<T>::load(Cp + v * 4, cv);
            float4& q = s[r][v];
            q.x = fmaf(a, q.x, xdt * bv[0]);
            q.y = fmaf(a, q.y, xdt * bv[1]);
            q.z = fmaf(a, q.z, xdt * bv[2]);
            q.w = fmaf(a, q.w, xdt * bv[3]);
            acc = fmaf(q.x, cv[0], acc);
            acc = fmaf(q.y, cv[1], acc);
            acc = fmaf(q.z, cv[2], acc);
            acc = fmaf(q.w, cv[3], acc);
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (valid) {
            float4* sp = reinterpret_cast<float4*>(p.state + rr * N) + tl * (VEC / 4);
#pragma unroll
            for (int v = 0; v < VEC / 4; ++v) __stcs(sp + v, s[r][v]);
            if (tl == 0) {
                const float Dh = p.D ? p.D[h] : 0.0f;
                static_cast<T*>(p.y)[rr] = from_f32<T>(acc + Dh * xv);
            }
        }
    }
}

template <typename T, int N>
cudaError_t launch_n(const DecodeParams& p, cudaStream_t s) {
    constexpr int VEC = (N > 128) ? N / 32 : 4;
    constexpr int RPW = 32 / (N / VEC);
    const int64_t nrows = p.batch * p.nheads * p.headdim;
    const int64_t rows_per_block = 8 * RPW * 2;  // 8 warps x RPW x ROWS
    const int64_t blocks = (nrows + rows_per_block - 1) / rows_per_block;
    state_update_kernel<T, N><<<(unsigned)blocks, 256, 0, s>>>(p);
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
