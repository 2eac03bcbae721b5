// internal.cuh -- shared declarations of the SSD scan kernels (not part of the
// public ABI; see include/ssd.h for the operation and the layouts).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// Sizes and pointers of one forward call, as the kernels see them.
struct FwdParams {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk, nchunks;
    int64_t heads_per_group;
    int32_t flags;         // SSD_FLAG_* of the call
    // launch plumbing (not a user flag): the kernels after the first of a call
    // go out with programmatic dependent launch, and the tensor-core
    // chunk_state forms dt and cumA itself (fusing step 1)
    int32_t pdl;
    int32_t fuse_cumsum;
    // chunk states (workspace and step entry points) in fp32 (1) or in the
    // input dtype (0: the backward's recompute, and the opt-in bf16-states mode)
    int32_t states_f32;
    const void* x;
    const void* dt_raw;
    const float* A;
    const void* B;
    const void* C;
    const float* D;        // may be null
    const float* dt_bias;  // may be null
    const float* init_state;  // may be null
    void* y;
    float* final_state;    // may be null
    const void* z;         // output gate [b, L, H, P] (y *= silu(z)); may be null
    // intermediates (workspace)
    float* dt;      // [b, H, nc, Q]
    float* cumA;    // [b, H, nc, Q]
    void* states;   // [b, nc, H, P, N] in fp32 or the input dtype (states_f32): local states, then states entering each chunk
    // [2][b, nc, H, P, N] bf16, or null: the states entering each chunk as hi
    // and lo halves (hi + lo = the fp32 state), for the tensor-core chunk_scan
    void* states_hl;
    int* status;    // device status word (SSD_ERR_TIMEOUT on a timed-out wait); may be null
};

// One backward call: the forward's sizes and inputs (f, whose dt / cumA /
// states / final_state point into the backward's workspace) plus the
// incoming gradients, the outputs and the backward's own intermediates.
struct BwdParams {
    FwdParams f;
    const void* dy;          // [b, L, H, P]
    const float* d_final;    // [b, H, P, N] or null
    void* dx;                // [b, L, H, P]
    void* ddt;               // [b, L, H] (gradient of the raw dt)
    float* dA;               // [H]
    void* dB;                // [b, L, G, N]
    void* dC;                // [b, L, G, N]
    float* dD;               // [H] or null
    float* ddt_bias;         // [H] or null
    float* d_init;           // [b, H, P, N] or null
    // workspace
    float* dstates;          // [b, nc, H, P, N]: local adjoint, then dJ/d(state leaving chunk c)
    float* dB_h;             // [b, L, H, N] per-head dB (when G < H), else null
    float* dC_h;             // [b, L, H, N] per-head dC (when G < H), else null
    float* xdxs;             // [b, H, L]: x_t . dxs_t
    float* dyx;              // [b, H, L]: dy_t . x_t
    float* mterm;            // [b, H, L]: dt_t x_t . (the dH part of dxs_t)
    float* qterm;            // [b, H, L]: e^{cumA_t} dy_t . (H_c C_t)
    float* colw;             // [b, H, L]: sum over later tokens s of the chunk of W[s, t]
    float* roww;             // [b, H, Q/rblk, L]: per source block of rblk tokens, sum over earlier r of W[t, r]
    int32_t rblk;            // tokens per source block of roww (64: CUDA-core kernels, 128: tensor cores)
    float* k4;               // [b, H, nc]: e^{cumA_c[last]} <dH_c, H_c>
    float* partial;          // [b, H, nc, 3]: per-chunk sums of dt*da, dy.x, ddt_raw
};

// The diagonal-A selective scan (forward and decode step).
struct SelParams {
    int64_t batch, seqlen, channels, dstate, chunk, nchunks;
    const void* x;           // [b, L, Dc] (forward) or [b, Dc] (decode)
    const void* dt_raw;      // like x
    const float* A;          // [Dc, N]
    const void* B;           // [b, L, N] (forward) or [b, N] (decode)
    const void* C;           // like B
    const float* D;          // [Dc] or null
    const float* dt_bias;    // [Dc] or null
    const float* init_state; // [b, Dc, N] or null (forward)
    void* y;                 // like x
    float* final_state;      // [b, Dc, N] or null (forward)
    float* S;                // forward: workspace [b, nc, Dc, N]; decode: the carried state [b, Dc, N]
    float* sdt;              // forward: workspace [b, nc, Dc], the sum of dt over each chunk
};

struct DecodeParams {
    int64_t batch, nheads, headdim, dstate, ngroups, heads_per_group;
    float* state;
    const void* x;
    const void* dt_raw;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    void* y;
    const void* z;         // output gate [b, H, P]; may be null
};

// The causal depthwise convolution (forward and decode step).
struct ConvParams {
    int64_t batch, seqlen, channels, width;
    int32_t activation;            // 1 = SiLU
    const void* x;                 // [b, L, C] (forward) or [b, C] (decode)
    const float* weight;           // [C, width]
    const float* bias;             // [C]; may be null
    const float* init_state;       // [b, C, width-1]; may be null (forward)
    void* y;
    float* final_state;            // [b, C, width-1]; may be null (forward)
    float* update_state;           // [b, C, width-1], in place (decode)
};

// Element loads/stores for the two supported input types.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// silu(z) = z / (1 + e^-z), the output gate's activation.
__device__ __forceinline__ float silu_f32(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// softplus(u) = log(1 + e^u) without overflow.
__device__ __forceinline__ float softplus_f32(float u) {
    return fmaxf(u, 0.0f) + log1pf(expf(-fabsf(u)));
}

// Programmatic dependent launch.  A kernel launched with pdl set may start
// while the previous kernel of the stream is still running; it must call
// grid_dep_wait() before it reads or writes anything that kernel (or an
// earlier one of the same call) produces.  grid_dep_launch() lets the next
// kernel start its own prologue early.  Both are no-ops for plain launches.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// dt = softplus(dt_raw + dt_bias) and the inclusive in-chunk cumulative sum of
// dt * A for one (batch, chunk, head), by one warp: each lane loads its
// tokens of every 32-token segment first, then the warp scans the segments in
// order with shuffles and a running carry.  Entries past the end of a short
// last chunk hold dt = 0 and the last cumulative value, so cumA[Q-1] is the
// chunk's total log-decay.  Writes both to dt_out / cum_out (Q entries).
// "MAMBA-2 Reference Implementations Comparison", section 3.2 (softplus
// discretisation of dt and the exp(A dt) decays whose exponents this sums).
template <typename T>
// When wout is given (shared memory, 8 x 32 = 256 entries), the warp also writes
// each token's decay weight e^{cumA[last] - cumA[l]} dt[l] there (0 past the end):
// the chunk_state weights, without reading back what it just stored.
__device__ __forceinline__ void chunk_cumsum_warp(const FwdParams& p, int64_t b, int64_t c, int64_t h,
                                                  float* dt_out, float* cum_out, int lane,
                                                  float* wout = nullptr) {
    constexpr int MAXSEG = 8;  // chunk <= 256 tokens
    const int64_t Q = p.chunk, H = p.nheads, L = p.seqlen;
    const int64_t t0 = c * Q;
    const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
    const int nseg = static_cast<int>((Q + 31) / 32);
    const T* dtr = static_cast<const T*>(p.dt_raw) + (b * L + t0) * H + h;
    const float A = p.A[h];
    const float bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
    float u[MAXSEG];
#pragma unroll
    for (int s = 0; s < MAXSEG; ++s) {
        const int64_t l = s * 32 + lane;
        u[s] = (s < nseg && l < Lc) ? to_f32(dtr[l * H]) : 0.0f;
    }
    float carry = 0.0f;
    float dts[MAXSEG], cums[MAXSEG];
#pragma unroll
    for (int s = 0; s < MAXSEG; ++s) {
        dts[s] = 0.0f;
        cums[s] = 0.0f;
        if (s >= nseg) continue;
        const int64_t l = s * 32 + lane;
        float dt = 0.0f, v = 0.0f;
        if (l < Lc) {
            dt = softplus_f32(u[s] + bias);
            v = dt * A;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        v += carry;
        if (l < Q) {
            dt_out[l] = dt;
            cum_out[l] = v;
        }
        dts[s] = dt;
        cums[s] = v;
        carry = __shfl_sync(0xffffffffu, v, 31);
    }
    if (wout) {
        // carry is now cumA[last] (entries past the end repeat it); every one
        // of the QMAX entries is written, 0 past the chunk's end, since the
        // weights are read in whole 64-token quarters
#pragma unroll
        for (int s = 0; s < MAXSEG; ++s) {
            const int64_t l = s * 32 + lane;
            wout[l] = (s < nseg && l < Lc) ? expf(carry - cums[s]) * dts[s] : 0.0f;
        }
    }
}

// Launchers (one per kernel family).  Each returns cudaGetLastError().
template <typename T> cudaError_t launch_chunk_cumsum(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_chunk_state_ffma(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_state_passing(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_chunk_scan_ffma(const FwdParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_state_update(const DecodeParams& p, cudaStream_t s);
template <typename T> cudaError_t launch_conv1d(const ConvParams& p, bool update, cudaStream_t s);
template <typename T>
cudaError_t launch_selective_scan(const SelParams& p, bool update, cudaStream_t s);
// The backward pass after the forward recompute (bwd.cu).
template <typename T> cudaError_t launch_ssd_bwd(const BwdParams& p, cudaStream_t s);
// The backward's per-chunk kernels on the tensor cores (bf16, headdim 64,
// dstate 64 or 128, chunk 128 or 256); false when the shape is outside that.
bool bwd_tc_supported(const FwdParams& p);
cudaError_t launch_bwd_tc(const BwdParams& p, cudaStream_t s);
// Shared memory (bytes) the backward's per-chunk kernels need for a shape.
size_t bwd_smem_bytes(int64_t headdim, int64_t dstate, int64_t chunk);
// Copies the forward kernel's device status word to *v and clears it (synchronises s).
cudaError_t conv1d_take_status(int* v, cudaStream_t s);

// Tensor-core (tcgen05) variants for bf16 inputs, with their shape ranges.
bool chunk_state_tc_supported(const FwdParams& p);
cudaError_t launch_chunk_state_tc(const FwdParams& p, cudaStream_t s);
bool chunk_scan_tc_supported(const FwdParams& p);
cudaError_t launch_chunk_scan_tc(const FwdParams& p, cudaStream_t s);
// The whole forward in one kernel (fused_fwd.cu): bf16, headdim 64, dstate 64
// or 128, chunk 128 or 256.  The workspace is its own (fused_fwd_workspace_bytes,
// 16-byte aligned) and is zeroed by the launch itself; status goes to its first word.
// The test hook ssd_debug_set_withhold() sets: the index a kernel's producer
// withholds (SSD_DEBUG_CONV_TILE: a convolution tile; SSD_DEBUG_FWD_CARRY: the
// carry leaving a chunk of the fused forward), -1 when off.  Read on the host
// at launch and passed to the kernel as an argument.
int64_t debug_withhold(int what);

bool fused_fwd_supported(const FwdParams& p);
size_t fused_fwd_workspace_bytes(const FwdParams& p);
cudaError_t launch_fused_fwd(const FwdParams& p, void* ws, cudaStream_t s);

}  // namespace ssd
