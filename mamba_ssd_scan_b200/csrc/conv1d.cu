// conv1d.cu -- the causal depthwise convolution in front of the scan and its
// decode step (the page "MAMBA-2 Implementation Gaps", Gap 2 "Convolution
// Layer": a Conv1d with one filter per channel, kernel width K, padding K - 1,
// the output cut to the sequence length, then SiLU):
//
//   out[t, c] = bias[c] + sum_{k<K} w[c, k] xin[t - (K-1) + k, c];  y = silu(out)
//
// xin extends x backwards with the carried inputs (init_state, oldest first).
// Bandwidth-bound: x is read once (plus a K-1 token halo per sequence
// segment) and y written once.  A CTA owns a block of channels (rows of at
// most 2 KB) over a segment of the sequence.  Its producer warp streams the
// segment's token rows into a ring of shared-memory tiles with bulk copies
// (one row per lane, completing on the tile's "full" mbarrier); the consumer
// warps take 4 channels per thread, keep the previous K-1 inputs in registers
// as a sliding window, compute with packed fp32x2 arithmetic, store their
// outputs directly and release the tile on its "empty" mbarrier.  The decode
// step keeps the same state [batch, channels, K-1] and shifts it by one token.
#include <stdlib.h>

#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

constexpr int TT = 8;          // token rows per shared-memory tile
constexpr int NSTAGE = 4;      // tiles in flight per CTA
constexpr int MAXROWB = 2048;  // bytes of one tile row (the CTA's channel block)
constexpr int CPT = 4;         // channels per consumer thread
template <typename T> constexpr int kMaxConsumers = MAXROWB / (CPT * static_cast<int>(sizeof(T)));

// SSD_ERR_TIMEOUT once a forward launch gave up on a wait; read and cleared
// by ssd_conv1d_check_status.
__device__ int g_conv_status;

// Four consecutive channels of one token, widened to fp32 pairs.
template <typename T> struct Quad;
template <> struct Quad<float> {
    static __device__ __forceinline__ void load(const uint8_t* s, float2& lo, float2& hi) {
        const float4 v = *reinterpret_cast<const float4*>(s);
        lo = make_float2(v.x, v.y);
        hi = make_float2(v.z, v.w);
    }
    static __device__ __forceinline__ void store(float* p, float2 lo, float2 hi) {
        *reinterpret_cast<float4*>(p) = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
};
template <> struct Quad<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const uint8_t* s, float2& lo, float2& hi) {
        const uint2 v = *reinterpret_cast<const uint2*>(s);
        lo = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
        hi = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float2 lo, float2 hi) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(lo.x, lo.y);
        const __nv_bfloat162 b = __floats2bfloat162_rn(hi.x, hi.y);
        *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a),
                                                  *reinterpret_cast<const uint32_t*>(&b));
    }
};

__device__ __forceinline__ float ex2_approx(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float rcp_approx(float v) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// silu(z) = z / (1 + e^-z) on a pair, e^-z = 2^(-z log2 e); a very negative z
// gives 1 + e^-z = inf and 1/inf = 0.
__device__ __forceinline__ float2 silu2(float2 z) {
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 t = __fmul2_rn(z, make_float2(kNegLog2e, kNegLog2e));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(t.x), ex2_approx(t.y)),
                                make_float2(1.0f, 1.0f));
    return __fmul2_rn(z, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// xin[i] for channel c: x[i] for i >= 0, the carried input init[K-1+i] (zero
// without one) for i < 0.
template <typename T, int K>
__device__ __forceinline__ float xin_at(const ConvParams& p, const T* xb, int64_t b, int64_t c,
                                        int64_t i) {
    if (i >= 0) return to_f32(xb[i * p.channels + c]);
    return p.init_state ? p.init_state[(b * p.channels + c) * (K - 1) + (K - 1 + i)] : 0.0f;
}

template <typename T, int K, bool ACT>
// `withhold` >= 0 makes the producer stop before that tile (a test of the
// bounded waits: the consumers time out, every role stops, the copies in
// flight land and the status word reads SSD_ERR_TIMEOUT); -1 in normal use.
__global__ void __launch_bounds__(kMaxConsumers<T> + 32)
    conv1d_kernel(ConvParams p, int64_t seg, int withhold) {
    using namespace tc;
    constexpr int KM = K > 1 ? K - 1 : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t full[NSTAGE], empty[NSTAGE];
    __shared__ int abort_flag, issued;

    const int NT = blockDim.x - 32;  // consumer threads; the last warp is the producer
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t L = p.seqlen, Cn = p.channels, ncq = Cn / CPT;
    const int64_t cqb = static_cast<int64_t>(blockIdx.x) * NT;  // first channel quad
    const int nv = static_cast<int>(ncq - cqb < NT ? ncq - cqb : NT);
    const uint32_t rowb = static_cast<uint32_t>(NT) * CPT * sizeof(T);
    const uint32_t rb = static_cast<uint32_t>(nv) * CPT * sizeof(T);
    const int64_t b = blockIdx.z;
    const int64_t ta = static_cast<int64_t>(blockIdx.y) * seg;  // < L by the grid
    const int64_t te = (ta + seg < L) ? ta + seg : L;
    const int ntiles = static_cast<int>((te - ta + TT - 1) / TT);

    if (tid == 0) {
#pragma unroll
        for (int st = 0; st < NSTAGE; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), static_cast<uint32_t>(NT / 32));
        }
        fence_mbar_init();
        abort_flag = 0;
        issued = 0;
    }
    __syncthreads();

    if (warp == NT / 32) {
        // ----- producer: tile j (TT token rows of this channel block) into stage j % NSTAGE
        const char* xt = static_cast<const char*>(p.x) + ((b * L + ta) * Cn + cqb * CPT) * sizeof(T);
        const int64_t xs = Cn * static_cast<int64_t>(sizeof(T));
        const uint32_t sbase = smem_u32(smem);
        int j = 0;
        for (; j < ntiles; ++j) {
            if (j == withhold) break;
            const int st = j % NSTAGE, use = j / NSTAGE;
            bool ok = true;
            if (use > 0 && lane == 0) ok = wait_or_abort(smem_u32(&empty[st]), (use - 1) & 1, &abort_flag);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int64_t left = te - ta - static_cast<int64_t>(j) * TT;
            const int rows = left < TT ? static_cast<int>(left) : TT;
            const uint32_t bar = smem_u32(&full[st]);
            if (lane == 0) mbar_expect_tx(bar, static_cast<uint32_t>(rows) * rb);
            __syncwarp();
            if (lane < rows)
                bulk_load_1d(sbase + static_cast<uint32_t>(st * TT + lane) * rowb,
                             xt + (static_cast<int64_t>(j) * TT + lane) * xs, rb, bar);
        }
        if (lane == 0) issued = j;
    } else {
        // ----- consumers: channels c0..c0+3 of every token of the segment
        const bool active = tid < nv;
        const int64_t c0 = (cqb + tid) * CPT;
        float2 w[K][2], bias[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t c = c0 + 2 * h;
#pragma unroll
            for (int k = 0; k < K; ++k)
                w[k][h] = active ? make_float2(p.weight[c * K + k], p.weight[(c + 1) * K + k])
                                 : make_float2(0.0f, 0.0f);
            bias[h] = (active && p.bias) ? make_float2(p.bias[c], p.bias[c + 1])
                                         : make_float2(0.0f, 0.0f);
        }
        const T* xb = static_cast<const T*>(p.x) + b * L * Cn;
        T* y = static_cast<T*>(p.y) + b * L * Cn + c0;

        // The first K-1 tokens of a sequence reach back into the carried
        // inputs (fp32): a scalar pass over them, then the window holds x only.
        const int64_t ts = (ta == 0 && K > 1) ? ((K - 1 < te) ? K - 1 : te) : ta;
        if (active) {
            for (int64_t t = ta; t < ts; ++t) {
                float o[CPT];
#pragma unroll
                for (int v = 0; v < CPT; ++v) {
                    float acc = (v & 1) ? bias[v >> 1].y : bias[v >> 1].x;
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const float wk = (v & 1) ? w[k][v >> 1].y : w[k][v >> 1].x;
                        acc = fmaf(wk, xin_at<T, K>(p, xb, b, c0 + v, t - (K - 1) + k), acc);
                    }
                    o[v] = ACT ? silu_f32(acc) : acc;
                }
                Quad<T>::store(y + t * Cn, make_float2(o[0], o[1]), make_float2(o[2], o[3]));
            }
        }
        // win[j] = x[t - (K-1) + j] for the next output token t (indices >= 0:
        // a segment after the first starts at least TT >= K-1 tokens in)
        float2 win[KM][2];
        if (active && ts < te) {
#pragma unroll
            for (int jj = 0; jj < K - 1; ++jj) {
                const T* q = xb + (ts - (K - 1) + jj) * Cn + c0;
                win[jj][0] = make_float2(to_f32(q[0]), to_f32(q[1]));
                win[jj][1] = make_float2(to_f32(q[2]), to_f32(q[3]));
            }
        }
        // one output token from the staged row at s (fp32x2 FMAs in tap order)
        auto step = [&](const uint8_t* s, int64_t t) {
            float2 lo, hi;
            Quad<T>::load(s, lo, hi);
            float2 a0 = bias[0], a1 = bias[1];
#pragma unroll
            for (int k = 0; k < K - 1; ++k) {
                a0 = __ffma2_rn(w[k][0], win[k][0], a0);
                a1 = __ffma2_rn(w[k][1], win[k][1], a1);
            }
            a0 = __ffma2_rn(w[K - 1][0], lo, a0);
            a1 = __ffma2_rn(w[K - 1][1], hi, a1);
            if (ACT) {
                a0 = silu2(a0);
                a1 = silu2(a1);
            }
            Quad<T>::store(y + t * Cn, a0, a1);
#pragma unroll
            for (int k = 0; k + 1 < K - 1; ++k) {
                win[k][0] = win[k + 1][0];
                win[k][1] = win[k + 1][1];
            }
            if (K > 1) {
                win[KM - 1][0] = lo;
                win[KM - 1][1] = hi;
            }
        };
        for (int j = 0; j < ntiles; ++j) {
            const int st = j % NSTAGE;
            const bool ok = wait_or_abort(smem_u32(&full[st]), (j / NSTAGE) & 1, &abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (active) {
                const int64_t tb = ta + static_cast<int64_t>(j) * TT;
                const uint8_t* row = smem + static_cast<uint32_t>(st * TT) * rowb + tid * CPT * sizeof(T);
                if (tb >= ts && tb + TT <= te) {
#pragma unroll
                    for (int r = 0; r < TT; ++r) step(row + r * rowb, tb + r);
                } else {
#pragma unroll
                    for (int r = 0; r < TT; ++r)
                        if (tb + r >= ts && tb + r < te) step(row + r * rowb, tb + r);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
        }
        // the carried inputs after the last token: xin[L-(K-1) .. L-1] (they
        // reach into init_state when L < K-1)
        if (active && p.final_state && te == L && K > 1 && !abort_flag) {
#pragma unroll
            for (int v = 0; v < CPT; ++v)
#pragma unroll
                for (int jj = 0; jj < K - 1; ++jj)
                    p.final_state[((b * Cn) + c0 + v) * (K - 1) + jj] =
                        xin_at<T, K>(p, xb, b, c0 + v, L - (K - 1) + jj);
        }
    }
    __syncthreads();
    if (abort_flag && tid == 0) {
        // A wait gave up: let the copies still in flight land (bounded)
        // before the CTA's shared memory goes away, and report it.
        for (int jj = issued - NSTAGE < 0 ? 0 : issued - NSTAGE; jj < issued; ++jj)
            mbar_wait(smem_u32(&full[jj % NSTAGE]), (jj / NSTAGE) & 1);
        atomicExch(&g_conv_status, static_cast<int>(SSD_ERR_TIMEOUT));
    }
}

// Decode: one thread per (batch row, 4 channels); the carried state of the 4
// channels (4 x (K-1) fp32, contiguous) moves as 16-byte vectors.
template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_update_kernel(ConvParams p) {
    constexpr int KM = K > 1 ? K - 1 : 1;
    const int64_t nq = p.channels / CPT;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= p.batch * nq) return;
    const int64_t c0 = (i % nq) * CPT;
    // consecutive decode steps go out with programmatic dependent launch:
    // wait for the previous step's state, then let the next step's CTAs in
    grid_dep_wait();
    grid_dep_launch();
    float st[CPT * KM];
    float4* s4 = reinterpret_cast<float4*>(p.update_state + i * CPT * (K - 1));
#pragma unroll
    for (int q = 0; q < K - 1; ++q) {
        const float4 v = s4[q];
        st[4 * q] = v.x; st[4 * q + 1] = v.y; st[4 * q + 2] = v.z; st[4 * q + 3] = v.w;
    }
    float2 lo, hi;
    Quad<T>::load(reinterpret_cast<const uint8_t*>(static_cast<const T*>(p.x) + i * CPT), lo, hi);
    const float xv[CPT] = {lo.x, lo.y, hi.x, hi.y};
    float wt[CPT * K];
    const float4* w4 = reinterpret_cast<const float4*>(p.weight + c0 * K);
#pragma unroll
    for (int q = 0; q < K; ++q) {
        const float4 v = __ldg(w4 + q);
        wt[4 * q] = v.x; wt[4 * q + 1] = v.y; wt[4 * q + 2] = v.z; wt[4 * q + 3] = v.w;
    }
    const float4 bv = p.bias ? __ldg(reinterpret_cast<const float4*>(p.bias + c0))
                             : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float bias[CPT] = {bv.x, bv.y, bv.z, bv.w};
    float o[CPT];
#pragma unroll
    for (int v = 0; v < CPT; ++v) {
        // channel v's taps are wt[v*K .. v*K+K-1], its state st[v*(K-1) ..]
        float acc = bias[v];
#pragma unroll
        for (int k = 0; k < K - 1; ++k) acc = fmaf(wt[v * K + k], st[v * (K - 1) + k], acc);
        acc = fmaf(wt[v * K + K - 1], xv[v], acc);
        o[v] = p.activation ? silu_f32(acc) : acc;
    }
    // shift each channel's window by one token, the new input last
    float ns[CPT * KM];
#pragma unroll
    for (int v = 0; v < CPT; ++v) {
#pragma unroll
        for (int k = 0; k + 1 < K - 1; ++k) ns[v * (K - 1) + k] = st[v * (K - 1) + k + 1];
        if (K > 1) ns[v * (K - 1) + K - 2] = xv[v];
    }
#pragma unroll
    for (int q = 0; q < K - 1; ++q)
        s4[q] = make_float4(ns[4 * q], ns[4 * q + 1], ns[4 * q + 2], ns[4 * q + 3]);
    Quad<T>::store(static_cast<T*>(p.y) + i * CPT, make_float2(o[0], o[1]), make_float2(o[2], o[3]));
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        n = 148;
    }
    return n;
}

// Forward grid: channel blocks of at most kMaxConsumers quads split evenly (a
// multiple of 32 consumer threads, plus the producer warp), and the sequence
// cut into segments of whole tiles so that the CTAs of all batch rows fill
// one wave of the SMs at the kernel's occupancy.
template <typename T, int K, bool ACT>
cudaError_t launch_fwd(const ConvParams& p, cudaStream_t s) {
    constexpr int MAXNT = kMaxConsumers<T>;
    const int64_t ncq = p.channels / CPT;
    const int64_t nblk = (ncq + MAXNT - 1) / MAXNT;
    const int nt = static_cast<int>(((ncq + nblk - 1) / nblk + 31) / 32 * 32);
    const size_t smem = static_cast<size_t>(NSTAGE) * TT * nt * CPT * sizeof(T);
    static int occ[MAXNT / 32 + 1];  // CTAs per SM by consumer count; benign race
    int& per_sm = occ[nt / 32];
    if (per_sm == 0) {
        // a full ring (64 KB) exceeds the default 48 KB dynamic limit
        cudaError_t e = cudaFuncSetAttribute(conv1d_kernel<T, K, ACT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             NSTAGE * TT * MAXROWB);
        if (e != cudaSuccess) return e;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, conv1d_kernel<T, K, ACT>,
                                                          nt + 32, smem) != cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            per_sm = 1;
        }
    }
    const int64_t slots = static_cast<int64_t>(sm_count()) * per_sm;
    const int64_t max_seg = (p.seqlen + TT - 1) / TT;
    int64_t nseg = slots / (nblk * p.batch);
    nseg = nseg < 1 ? 1 : (nseg > max_seg ? max_seg : nseg);
    const int64_t seg = ((p.seqlen + nseg - 1) / nseg + TT - 1) / TT * TT;
    nseg = (p.seqlen + seg - 1) / seg;
    dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(nseg),
              static_cast<unsigned>(p.batch));
    // the test hook (ssd_debug_set_withhold): the producer withholds that tile
    const int64_t wh = debug_withhold(SSD_DEBUG_CONV_TILE);
    conv1d_kernel<T, K, ACT><<<grid, nt + 32, smem, s>>>(p, seg, static_cast<int>(wh));
    return cudaGetLastError();
}

template <typename T, int K>
cudaError_t launch_k(const ConvParams& p, bool update, cudaStream_t s) {
    if (!update) return p.activation ? launch_fwd<T, K, true>(p, s) : launch_fwd<T, K, false>(p, s);
    const int64_t n = p.batch * (p.channels / CPT);
    return launch_kernel(conv1d_update_kernel<T, K>, dim3(static_cast<unsigned>((n + 255) / 256)),
                         dim3(256), 0, s, true, p);
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

cudaError_t conv1d_take_status(int* v, cudaStream_t s) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(v, g_conv_status, sizeof(int), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_conv_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e;
}

}  // namespace ssd
