// gated_rmsnorm.cu -- the RMSNorm after the scan, with the output gate inside
// it ("MAMBA-2 Implementation Gaps", section 7.3, items 9 and 11: the output
// gating y * silu(z) and an RMSNorm before the final projection).  For each
// row (token) and each group of `group` consecutive channels:
//
//   g = y * silu(z)            (g = y without z)
//   out = g / sqrt(mean_group(g^2) + eps) * weight
//
// Bandwidth-bound: y and z are read once and out written once.  The group's
// mean spans heads that different chunk-scan CTAs produce, so the norm is its
// own pass over y rather than a chunk-scan epilogue.
//
// A unit is one (row, group) pair; its `group` elements are contiguous at
// unit * group.  A unit is spread over LPU lanes (a power of two up to the
// CTA's 256 threads, the smallest that leaves each lane at most MAXV
// vectors), lane l taking vectors l, l + LPU, ... of the unit, so the lanes of
// a unit read consecutive 16-byte pieces; the last round may be ragged.  Up to MAXV vectors per lane are kept in registers between the sum
// of squares and the scaling; a longer unit re-reads its y and z (from L2) in
// the second pass.  The sum of squares is a shuffle reduction over the unit's
// lanes, plus a shared-memory step when the unit spans several warps.
#include "gated_rmsnorm.h"

namespace ssd {
namespace {

constexpr int TPB = 256;
constexpr int MAXV = 4;   // 16-byte vectors per lane kept in registers

// Eight (bf16) or four (fp32) consecutive elements, widened to fp32.  Plain
// (coherent) loads: out may be y itself.
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void load(const float* p, float* v) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* v) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* v) {
        const uint4 a = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// g = y * silu(z) for one vector (y alone when there is no gate).
template <typename T>
__device__ __forceinline__ void gated(const T* y, const T* z, int64_t off, float* g) {
    constexpr int N = Vec<T>::N;
    Vec<T>::load(y + off, g);
    if (z) {
        float zv[N];
        Vec<T>::load(z + off, zv);
#pragma unroll
        for (int i = 0; i < N; ++i) g[i] *= silu_f32(zv[i]);
    }
}

// N consecutive fp32 weights (16-byte aligned: N and the offset are multiples
// of 4).
template <int N> __device__ __forceinline__ void weights(const float* p, float* w) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p + i));
        w[i] = a.x; w[i + 1] = a.y; w[i + 2] = a.z; w[i + 3] = a.w;
    }
}

template <typename T>
__global__ void __launch_bounds__(TPB) gated_rmsnorm_kernel(NormParams p, int lpu, int nvec, int vecs) {
    constexpr int N = Vec<T>::N;
    __shared__ float red[TPB / 32];
    const T* y = static_cast<const T*>(p.y);
    const T* z = static_cast<const T*>(p.z);
    T* out = static_cast<T*>(p.out);
    const int upc = TPB / lpu;                       // units per CTA pass
    const int lane_in_unit = threadIdx.x & (lpu - 1);
    const int unit_in_cta = threadIdx.x / lpu;
    const int64_t units = p.rows * (p.channels / p.group);
    const int64_t ngroups = p.channels / p.group;
    const float inv_group = 1.0f / static_cast<float>(p.group);

    for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * upc; u0 < units;
         u0 += static_cast<int64_t>(gridDim.x) * upc) {
        const int64_t u = u0 + unit_in_cta;
        const bool live = u < units;
        const int64_t base = u * p.group;
        const int64_t wbase = (u % ngroups) * p.group;

        // pass 1: g and the sum of its squares
        float g[MAXV][N];
        float ss = 0.0f;
        if (live) {
#pragma unroll
            for (int j = 0; j < MAXV; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (j < nvec && v < vecs) {
                    gated(y, z, base + static_cast<int64_t>(v) * N, g[j]);
#pragma unroll
                    for (int i = 0; i < N; ++i) ss = fmaf(g[j][i], g[j][i], ss);
                }
            }
            for (int j = MAXV; j < nvec; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (v >= vecs) break;
                float t[N];
                gated(y, z, base + static_cast<int64_t>(v) * N, t);
#pragma unroll
                for (int i = 0; i < N; ++i) ss = fmaf(t[i], t[i], ss);
            }
        }
        // the unit's sum: within the warp, then across the unit's warps
        for (int o = (lpu < 32 ? lpu : 32) / 2; o > 0; o >>= 1)
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lpu > 32) {
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
            __syncthreads();
            const int w0 = (unit_in_cta * lpu) >> 5;
            ss = 0.0f;
            for (int w = 0; w < (lpu >> 5); ++w) ss += red[w0 + w];
            __syncthreads();
        }
        const float inv = rsqrtf(ss * inv_group + p.eps);

        // pass 2: scale by inv and the weight, round, store
        if (live) {
#pragma unroll
            for (int j = 0; j < MAXV; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (j < nvec && v < vecs) {
                    const int64_t c = static_cast<int64_t>(v) * N;
                    float w[N];
                    weights<N>(p.weight + wbase + c, w);
#pragma unroll
                    for (int i = 0; i < N; ++i) w[i] *= g[j][i] * inv;
                    Vec<T>::store(out + base + c, w);
                }
            }
            for (int j = MAXV; j < nvec; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (v >= vecs) break;
                const int64_t c = static_cast<int64_t>(v) * N;
                float t[N], w[N];
                gated(y, z, base + c, t);
                weights<N>(p.weight + wbase + c, w);
#pragma unroll
                for (int i = 0; i < N; ++i) w[i] *= t[i] * inv;
                Vec<T>::store(out + base + c, w);
            }
        }
    }
}

int device_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

template <typename T> cudaError_t launch(const NormParams& p, cudaStream_t s) {
    constexpr int N = Vec<T>::N;
    const int64_t vecs = p.group / N;                // 16-byte vectors per unit
    // lanes per unit: the smallest power of two (at most a CTA) that leaves
    // each lane at most MAXV vectors, so that a lane keeps as many bytes in
    // flight as its registers hold; the last round of a unit may be ragged
    if (vecs > (int64_t{1} << 30)) return cudaErrorInvalidValue;
    int lpu = 1;
    while (lpu < TPB && static_cast<int64_t>(lpu) * MAXV < vecs) lpu *= 2;
    const int64_t nvec = (vecs + lpu - 1) / lpu;
    const int64_t units = p.rows * (p.channels / p.group);
    const int64_t upc = TPB / lpu;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gated_rmsnorm_kernel<T>, TPB, 0) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t want = (units + upc - 1) / upc;
    const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    gated_rmsnorm_kernel<T><<<grid, TPB, 0, s>>>(p, lpu, static_cast<int>(nvec),
                                                 static_cast<int>(vecs));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const NormParams& p, bool bf16, cudaStream_t s) {
    return bf16 ? launch<__nv_bfloat16>(p, s) : launch<float>(p, s);
}

}  // namespace ssd
