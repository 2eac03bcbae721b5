// state_passing.cu -- step 3 of the chunked SSD forward: the inter-chunk carry
// ("MAMBA-2 Implementation Gaps", Gap 1: the off-diagonal blocks propagate the
// previous chunk's final state; "MAMBA-2 Reference Implementations
// Comparison", section 3.2: the last state is the carry).
//
//   H_{-1} = init (or 0);   H_c = exp(cumA_c[last]) H_{c-1} + S_c
//
// Sequential over chunks, parallel over batch x heads x headdim x dstate: each
// thread carries 4 consecutive state elements (one 16-byte vector) in
// registers.  In place over `states`: slot c receives H_{c-1}, the state that
// enters chunk c; the final state H_{nc-1} goes to final_state.  The loads of
// the next chunks' S do not depend on the carry, so they are issued ahead of
// the multiply-adds (UNROLL chunks at a time) to keep enough bytes in flight.
#include "internal.cuh"

namespace ssd {
namespace {

constexpr int UNROLL = 4;

__global__ void __launch_bounds__(256) state_passing_kernel(FwdParams p) {
    const int64_t H = p.nheads, nc = p.nchunks, Q = p.chunk;
    const int64_t vecs_per_head = p.headdim * p.dstate / 4;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.batch * H * vecs_per_head) return;
    const int64_t bh = e / vecs_per_head, off = e % vecs_per_head;
    const int64_t b = bh / H, h = bh % H;
    float4 carry = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.init_state) carry = reinterpret_cast<const float4*>(p.init_state)[e];
    float4* st = reinterpret_cast<float4*>(p.states);
    const float* cs = p.cumA + (b * H + h) * nc * Q + (Q - 1);
    const int64_t cstride = H * vecs_per_head;  // float4s between consecutive chunks
    float4* base = st + (b * nc * H + h) * vecs_per_head + off;
    int64_t c = 0;
    for (; c + UNROLL <= nc; c += UNROLL) {
        float4 s[UNROLL];
        float a[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            s[u] = base[(c + u) * cstride];
            a[u] = expf(cs[(c + u) * Q]);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            base[(c + u) * cstride] = carry;
            carry.x = fmaf(a[u], carry.x, s[u].x);
            carry.y = fmaf(a[u], carry.y, s[u].y);
            carry.z = fmaf(a[u], carry.z, s[u].z);
            carry.w = fmaf(a[u], carry.w, s[u].w);
        }
    }
    for (; c < nc; ++c) {
        const float4 s = base[c * cstride];
        const float a = expf(cs[c * Q]);
        base[c * cstride] = carry;
        carry.x = fmaf(a, carry.x, s.x);
        carry.y = fmaf(a, carry.y, s.y);
        carry.z = fmaf(a, carry.z, s.z);
        carry.w = fmaf(a, carry.w, s.w);
    }
    if (p.final_state) reinterpret_cast<float4*>(p.final_state)[e] = carry;
}

}  // namespace

cudaError_t launch_state_passing(const FwdParams& p, cudaStream_t s) {
    const int64_t n = p.batch * p.nheads * p.headdim * p.dstate / 4;
    state_passing_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace ssd
