// conv1d.cu -- the causal depthwise convolution in front of the scan and its
// decode step (the page "MAMBA-2 Implementation Gaps", Gap 2 "Convolution
// Layer": a Conv1d with one filter per channel, kernel width K, padding K - 1,
// the output cut to the sequence length, then SiLU):
//
//   out[t, c] = bias[c] + sum_{k<K} w[c, k] xin[t - (K-1) + k, c];  y = silu(out)
//
// xin extends x backwards with the carried inputs (init_state, oldest first).
// Bandwidth-bound: x is read once (plus a K-1 token halo per strip) and y
// written once.  A thread owns one 16-byte vector of channels (8 bf16 or 4
// fp32) and a strip of TS consecutive tokens; consecutive threads take
// consecutive channel vectors of the same strip, so a warp's loads and stores
// are contiguous.  The previous K-1 inputs of its channels live in registers
// as a sliding window; the thread holding the last strip writes the final
// window as the carried state.  The decode step keeps the same state
// [batch, channels, K-1] and shifts it by one token.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int TS = 32;  // tokens per thread strip

template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int V = 4;
    static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
        const float4 q = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int V = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&t);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_kernel(ConvParams p) {
    constexpr int V = Vec<T>::V;
    constexpr int KM = K > 1 ? K - 1 : 1;
    const int64_t L = p.seqlen, Cn = p.channels, ncv = Cn / V;
    const int64_t nstrips = (L + TS - 1) / TS;
    const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (g >= ncv * nstrips) return;
    const int64_t cv = g % ncv, strip = g / ncv;
    const int64_t c0 = cv * V, t0 = strip * TS;

    float w[V][K], bias[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
#pragma unroll
        for (int k = 0; k < K; ++k) w[v][k] = p.weight[(c0 + v) * K + k];
        bias[v] = p.bias ? p.bias[c0 + v] : 0.0f;
    }
    // window[j] = xin[t - (K-1) + j] for the next output token t
    float win[KM][V];
    const T* x = static_cast<const T*>(p.x) + b * L * Cn + c0;
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int64_t i = t0 - (K - 1) + j;
        if (i >= 0) {
            Vec<T>::load(x + i * Cn, win[j]);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v)
                win[j][v] = p.init_state ? p.init_state[((b * Cn) + c0 + v) * (K - 1) + (K - 1 + i)] : 0.0f;
        }
    }
    T* y = static_cast<T*>(p.y) + b * L * Cn + c0;
    const int64_t t1 = (t0 + TS < L) ? t0 + TS : L;
    for (int64_t t = t0; t < t1; ++t) {
        float cur[V], out[V];
        Vec<T>::load(x + t * Cn, cur);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float acc = bias[v];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) acc = fmaf(w[v][k], win[k][v], acc);
            acc = fmaf(w[v][K - 1], cur[v], acc);
            out[v] = p.activation ? silu_f32(acc) : acc;
        }
        Vec<T>::store(y + t * Cn, out);
#pragma unroll
        for (int k = 0; k + 1 < K - 1; ++k)
#pragma unroll
            for (int v = 0; v < V; ++v) win[k][v] = win[k + 1][v];
        if (K > 1) {
#pragma unroll
            for (int v = 0; v < V; ++v) win[KM - 1][v] = cur[v];
        }
    }
    if (p.final_state && t1 == L && K > 1) {
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < K - 1; ++j) p.final_state[((b * Cn) + c0 + v) * (K - 1) + j] = win[j][v];
    }
}

template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_update_kernel(ConvParams p) {
    constexpr int KM = K > 1 ? K - 1 : 1;
    const int64_t Cn = p.channels;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= p.batch * Cn) return;
    const int64_t c = i % Cn;
    float* s = p.update_state + i * (K - 1);
    float st[KM];
#pragma unroll
    for (int k = 0; k < K - 1; ++k) st[k] = s[k];
    const float xv = to_f32(static_cast<const T*>(p.x)[i]);
    float acc = p.bias ? p.bias[c] : 0.0f;
#pragma unroll
    for (int k = 0; k < K - 1; ++k) acc = fmaf(p.weight[c * K + k], st[k], acc);
    acc = fmaf(p.weight[c * K + K - 1], xv, acc);
#pragma unroll
    for (int k = 0; k + 1 < K - 1; ++k) s[k] = st[k + 1];
    if (K > 1) s[KM - 1] = xv;
    static_cast<T*>(p.y)[i] = from_f32<T>(p.activation ? silu_f32(acc) : acc);
}

template <typename T, int K>
cudaError_t launch_k(const ConvParams& p, bool update, cudaStream_t s) {
    if (update) {
        const int64_t n = p.batch * p.channels;
        conv1d_update_kernel<T, K><<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
    } else {
        const int64_t items = (p.channels / Vec<T>::V) * ((p.seqlen + TS - 1) / TS);
        dim3 grid(static_cast<unsigned>((items + 255) / 256), static_cast<unsigned>(p.batch));
        conv1d_kernel<T, K><<<grid, 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

template <typename T>
cudaError_t launch_conv1d(const ConvParams& p, bool update, cudaStream_t s) {
    switch (p.width) {
        case 1: return launch_k<T, 1>(p, update, s);
        case 2: return launch_k<T, 2>(p, update, s);
        case 3: return launch_k<T, 3>(p, update, s);
        case 4: return launch_k<T, 4>(p, update, s);
        case 5: return launch_k<T, 5>(p, update, s);
        case 6: return launch_k<T, 6>(p, update, s);
        case 7: return launch_k<T, 7>(p, update, s);
        case 8: return launch_k<T, 8>(p, update, s);
        default: return cudaErrorInvalidValue;
    }
}

template cudaError_t launch_conv1d<float>(const ConvParams&, bool, cudaStream_t);
template cudaError_t launch_conv1d<__nv_bfloat16>(const ConvParams&, bool, cudaStream_t);

}  // namespace ssd
