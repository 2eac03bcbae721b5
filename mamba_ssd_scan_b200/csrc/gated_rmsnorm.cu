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
// a unit read consecutive 16-byte pieces; the last round may be ragged.  Up
// to MAXV vectors per lane are kept in registers between the sum of squares
// and the scaling; a longer unit re-reads its y and z (from L2) in the second
// pass.  The sum of squares is a shuffle reduction over the unit's lanes,
// plus a shared-memory step when the unit spans several warps.
#include "gated_rmsnorm.h"

namespace ssd {
namespace {

constexpr int TPB = 256;
constexpr int MAXV = 4;   // 16-byte vectors per lane kept in registers

// Eight (bf16) or four (fp32) consecutive elements as one 16-byte word, widened
// to fp32.  Plain (coherent) loads: out may be y itself.
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void widen(uint4 a, float* v) {
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
        v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    }
    static __device__ __forceinline__ void store(float* p, const float* v) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void widen(uint4 a, float* v) {
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

template <typename T> __device__ __forceinline__ uint4 ld16(const T* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// g = y * silu(z) from the raw words (y alone without the gate).
template <typename T, bool GATED>
__device__ __forceinline__ void gate_vec(uint4 ry, uint4 rz, float* g) {
    constexpr int N = Vec<T>::N;
    Vec<T>::widen(ry, g);
    if constexpr (GATED) {
        float zv[N];
        Vec<T>::widen(rz, zv);
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

// NV: vectors per lane held in registers (1..MAXV); a lane's vectors past
// NV (nvec > NV) are re-read in the second pass.
template <typename T, int NV, bool GATED>
__global__ void __launch_bounds__(TPB, 4) gated_rmsnorm_kernel(NormParams p, int lpu, int nvec, int vecs) {
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

        // pass 1: every raw load of the lane first (a ragged round's missing
        // vectors read the lane's first one again and count as zero), then g
        // and the sum of its squares
        float g[NV][N];
        float ss = 0.0f;
        if (live) {
            uint4 ry[NV], rz[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int v = lane_in_unit + j * lpu;
                const int64_t off = base + static_cast<int64_t>(v < vecs ? v : lane_in_unit) * N;
                ry[j] = ld16(y + off);
                if constexpr (GATED) rz[j] = ld16(z + off);
            }
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                gate_vec<T, GATED>(ry[j], rz[j], g[j]);
                const bool in = lane_in_unit + j * lpu < vecs;
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    g[j][i] = in ? g[j][i] : 0.0f;
                    ss = fmaf(g[j][i], g[j][i], ss);
                }
            }
            for (int j = NV; j < nvec; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (v >= vecs) break;
                const int64_t off = base + static_cast<int64_t>(v) * N;
                float t[N];
                gate_vec<T, GATED>(ld16(y + off), GATED ? ld16(z + off) : uint4{}, t);
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
            for (int j = 0; j < NV; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (v < vecs) {
                    const int64_t c = static_cast<int64_t>(v) * N;
                    float w[N];
                    weights<N>(p.weight + wbase + c, w);
#pragma unroll
                    for (int i = 0; i < N; ++i) w[i] *= g[j][i] * inv;
                    Vec<T>::store(out + base + c, w);
                }
            }
            for (int j = NV; j < nvec; ++j) {
                const int v = lane_in_unit + j * lpu;
                if (v >= vecs) break;
                const int64_t c = static_cast<int64_t>(v) * N;
                float t[N], w[N];
                gate_vec<T, GATED>(ld16(y + base + c), GATED ? ld16(z + base + c) : uint4{}, t);
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
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        n = 148;
    }
    return n;
}

template <typename T, int NV, bool GATED>
cudaError_t launch_nv(const NormParams& p, int lpu, int64_t nvec, int64_t vecs, cudaStream_t s) {
    const auto kern = gated_rmsnorm_kernel<T, NV, GATED>;
    const int64_t units = p.rows * (p.channels / p.group);
    const int64_t upc = TPB / lpu;
    static int occ;  // CTAs per SM of this instantiation (same on every B200); benign race
    if (occ == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, TPB, 0) != cudaSuccess ||
            n < 1) {
            cudaGetLastError();
            n = 1;
        }
        occ = n;
    }
    const int per_sm = occ;
    const int64_t want = (units + upc - 1) / upc;
    const int64_t cap = static_cast<int64_t>(device_sms()) * per_sm;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    kern<<<grid, TPB, 0, s>>>(p, lpu, static_cast<int>(nvec), static_cast<int>(vecs));
    return cudaGetLastError();
}

template <typename T, bool GATED>
cudaError_t launch(const NormParams& p, cudaStream_t s) {
    constexpr int N = Vec<T>::N;
    const int64_t vecs = p.group / N;                // 16-byte vectors per unit
    // lanes per unit: the smallest power of two (at most a CTA) that leaves
    // each lane at most MAXV vectors, so that a lane keeps as many bytes in
    // flight as its registers hold; the last round of a unit may be ragged
    if (vecs > (int64_t{1} << 30)) return cudaErrorInvalidValue;
    int lpu = 1;
    while (lpu < TPB && static_cast<int64_t>(lpu) * MAXV < vecs) lpu *= 2;
    const int64_t nvec = (vecs + lpu - 1) / lpu;
    switch (nvec) {
        case 1: return launch_nv<T, 1, GATED>(p, lpu, nvec, vecs, s);
        case 2: return launch_nv<T, 2, GATED>(p, lpu, nvec, vecs, s);
        case 3: return launch_nv<T, 3, GATED>(p, lpu, nvec, vecs, s);
        default: return launch_nv<T, MAXV, GATED>(p, lpu, nvec, vecs, s);
    }
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const NormParams& p, bool bf16, cudaStream_t s) {
    if (bf16) return p.z ? launch<__nv_bfloat16, true>(p, s) : launch<__nv_bfloat16, false>(p, s);
    return p.z ? launch<float, true>(p, s) : launch<float, false>(p, s);
}

}  // namespace ssd
