// state_passing.cu -- step 3 of the chunked SSD forward: the inter-chunk carry
// ("MAMBA-2 Implementation Gaps", Gap 1: the off-diagonal blocks propagate the
// previous chunk's final state; "MAMBA-2 Reference Implementations
// Comparison", section 3.2: the last state is the carry).
//
//   H_{-1} = init (or 0);   H_c = exp(cumA_c[last]) H_{c-1} + S_c
//
// Sequential over chunks, parallel over batch x heads x headdim x dstate: each
// thread carries one 16-byte vector of state elements (4 fp32 or 8 bf16) in
// fp32 registers.  Slot c receives H_{c-1}, the state that enters chunk c,
// either in place over `states` (in the dtype the states are kept in) or, for
// the tensor-core chunk_scan, as a pair of bf16 arrays in states_hl: hi =
// bf16(H) and lo = bf16(H - hi), so that hi + lo carries H to about 2^-17 of
// its size through a bf16 operand.  The final state H_{nc-1} goes to
// final_state in fp32.  The loads of the next chunks' S do not depend on the
// carry, so UNROLL chunks are loaded before their multiply-adds to keep enough
// bytes in flight.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int UNROLL = 4;

template <typename T> struct Pack;
template <> struct Pack<float> {
    static constexpr int E = 4;
    static __device__ __forceinline__ void unpack(uint4 v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[4]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <> struct Pack<__nv_bfloat16> {
    static constexpr int E = 8;
    static __device__ __forceinline__ void unpack(uint4 v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
    static __device__ __forceinline__ uint4 pack(const float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&t);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <typename T>
__global__ void __launch_bounds__(256) state_passing_kernel(FwdParams p) {
    grid_dep_wait();  // the local states and cumA come from the previous steps
    grid_dep_launch();
    constexpr int E = Pack<T>::E;
    const int64_t H = p.nheads, nc = p.nchunks, Q = p.chunk;
    const int64_t vecs_per_head = p.headdim * p.dstate / E;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.batch * H * vecs_per_head) return;
    const int64_t bh = e / vecs_per_head, off = e % vecs_per_head;
    const int64_t b = bh / H, h = bh % H;
    float carry[E];
    if (p.init_state) {
        const float4* ip = reinterpret_cast<const float4*>(p.init_state + e * E);
#pragma unroll
        for (int k = 0; k < E / 4; ++k) {
            const float4 v = ip[k];
            carry[4 * k] = v.x; carry[4 * k + 1] = v.y; carry[4 * k + 2] = v.z; carry[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) carry[k] = 0.0f;
    }
    uint4* base = reinterpret_cast<uint4*>(p.states) + (b * nc * H + h) * vecs_per_head + off;
    const int64_t cstride = H * vecs_per_head;  // vectors between consecutive chunks
    const float* cs = p.cumA + (b * H + h) * nc * Q + (Q - 1);
    for (int64_t c = 0; c < nc; c += UNROLL) {
        uint4 s[UNROLL];
        float a[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            if (c + u < nc) {
                s[u] = base[(c + u) * cstride];
                a[u] = expf(cs[(c + u) * Q]);
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            if (c + u < nc) {
                float sv[E];
                Pack<T>::unpack(s[u], sv);
                base[(c + u) * cstride] = Pack<T>::pack(carry);
#pragma unroll
                for (int k = 0; k < E; ++k) carry[k] = fmaf(a[u], carry[k], sv[k]);
            }
        }
    }
    if (p.final_state) {
        float4* fp = reinterpret_cast<float4*>(p.final_state + e * E);
#pragma unroll
        for (int k = 0; k < E / 4; ++k)
            fp[k] = make_float4(carry[4 * k], carry[4 * k + 1], carry[4 * k + 2], carry[4 * k + 3]);
    }
}

// The hi / lo form: fp32 local states in, each entering state out as two
// bf16 arrays (hi = bf16(H), lo = bf16(H - hi); H - hi is exact in fp32).
// Each thread carries 8 consecutive state elements: two 16-byte loads per
// chunk (four chunks' loads in flight), one 16-byte store of each half.
constexpr int HL_UNROLL = 4;

__device__ __forceinline__ void split_store(__nv_bfloat16* hi, __nv_bfloat16* lo, const float (&v)[8]) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 hb = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(v[2 * k] - hf.x, v[2 * k + 1] - hf.y);
        hw[k] = *reinterpret_cast<const uint32_t*>(&hb);
        lw[k] = *reinterpret_cast<const uint32_t*>(&lb);
    }
    *reinterpret_cast<uint4*>(hi) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(lo) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// 128-thread blocks, five per SM (<= 102 registers): at seqlen 65536 all 640
// blocks are resident at once (with 256-thread blocks at 95 registers only
// two fit an SM and the last 24 of 320 ran as a second wave).
constexpr int HL_THREADS = 128;

__global__ void __launch_bounds__(HL_THREADS, 5) state_passing_hl_kernel(FwdParams p) {
    grid_dep_wait();  // the local states and cumA come from the previous steps
    grid_dep_launch();
    const int64_t H = p.nheads, nc = p.nchunks, Q = p.chunk;
    const int64_t vecs_per_head = p.headdim * p.dstate / 8;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.batch * H * vecs_per_head) return;
    const int64_t bh = e / vecs_per_head, off = e % vecs_per_head;
    const int64_t b = bh / H, h = bh % H;
    float carry[8];
    if (p.init_state) {
        const float4* ip = reinterpret_cast<const float4*>(p.init_state + e * 8);
        const float4 v0 = ip[0], v1 = ip[1];
        carry[0] = v0.x; carry[1] = v0.y; carry[2] = v0.z; carry[3] = v0.w;
        carry[4] = v1.x; carry[5] = v1.y; carry[6] = v1.z; carry[7] = v1.w;
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) carry[k] = 0.0f;
    }
    const int64_t first = ((b * nc * H + h) * vecs_per_head + off) * 8;  // element of chunk 0
    const int64_t cstride = H * vecs_per_head * 8;                        // elements between chunks
    const float* src = static_cast<const float*>(p.states) + first;
    __nv_bfloat16* hi = static_cast<__nv_bfloat16*>(p.states_hl) + first;
    __nv_bfloat16* lo = hi + p.batch * nc * H * p.headdim * p.dstate;
    const float* cs = p.cumA + (b * H + h) * nc * Q + (Q - 1);
    for (int64_t c = 0; c < nc; c += HL_UNROLL) {
        float4 s0[HL_UNROLL], s1[HL_UNROLL];
        float a[HL_UNROLL];
#pragma unroll
        for (int u = 0; u < HL_UNROLL; ++u) {
            if (c + u < nc) {
                const float4* sp = reinterpret_cast<const float4*>(src + (c + u) * cstride);
                s0[u] = sp[0];
                s1[u] = sp[1];
                a[u] = expf(cs[(c + u) * Q]);
            }
        }
#pragma unroll
        for (int u = 0; u < HL_UNROLL; ++u) {
            if (c + u < nc) {
                split_store(hi + (c + u) * cstride, lo + (c + u) * cstride, carry);
                const float sv[8] = {s0[u].x, s0[u].y, s0[u].z, s0[u].w, s1[u].x, s1[u].y, s1[u].z, s1[u].w};
#pragma unroll
                for (int k = 0; k < 8; ++k) carry[k] = fmaf(a[u], carry[k], sv[k]);
            }
        }
    }
    if (p.final_state) {
        float4* fp = reinterpret_cast<float4*>(p.final_state + e * 8);
        fp[0] = make_float4(carry[0], carry[1], carry[2], carry[3]);
        fp[1] = make_float4(carry[4], carry[5], carry[6], carry[7]);
    }
}

}  // namespace

template <typename T>
cudaError_t launch_state_passing(const FwdParams& p, cudaStream_t s) {
    if (p.states_hl) {
        const int64_t n = p.batch * p.nheads * p.headdim * p.dstate / 8;
        return launch_kernel(state_passing_hl_kernel, dim3((unsigned)((n + HL_THREADS - 1) / HL_THREADS)),
                             dim3(HL_THREADS), 0, s, p.pdl != 0, p);
    }
    const int64_t n = p.batch * p.nheads * p.headdim * p.dstate / Pack<T>::E;
    return launch_kernel(state_passing_kernel<T>, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s,
                         p.pdl != 0, p);
}

template cudaError_t launch_state_passing<float>(const FwdParams&, cudaStream_t);
template cudaError_t launch_state_passing<__nv_bfloat16>(const FwdParams&, cudaStream_t);

}  // namespace ssd
