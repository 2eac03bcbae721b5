// chunk_state_tc.cu -- step 2 of the chunked SSD forward on the sm_100a tensor
// cores: every chunk's local state
//   S_c[p,n] = sum_{l in c} (exp(cumA[last] - cumA[l]) dt[l] x[l,p]) B[l,n]
// (the "diagonal block: local state" of "MAMBA-2 Implementation Gaps", Gap 1),
// as one GEMM per CTA with tcgen05.mma (bf16 operands, fp32 accumulation in
// TMEM):
//   D[m, n] = sum_l A[m, l] B[l, n],  m = (head, p) over 128/P heads of one
//   group (M = 128), n = 0..dstate-1 (N = dstate), K = the chunk's tokens.
// Both operands are MN-major: A is the weighted x rows as they sit in memory
// (for a token, the 128/P heads' P values are contiguous), B is the group's B
// rows.  Tokens stream through a 2-stage shared-memory ring of 64 tokens; all
// 256 threads load (16-byte vector loads, the decay weight folded into x while
// staging) while the tensor core consumes the other stage; one thread issues
// the MMAs and commits each stage to its mbarrier.  The epilogue moves the
// fp32 accumulator from TMEM to the states buffer (bf16, the input dtype), one
// row of dstate per thread.
#include "internal.cuh"
#include "tcgen05.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int KT = 64;      // tokens per stage
constexpr int NSTAGE = 2;
constexpr int QMAX = 256;

template <int NST, int PD>
struct StateTile {
    static constexpr int HPC = 128 / PD;               // heads per CTA
    static constexpr int A_BYTES = 2 * KT * 128;       // 2 blocks of 64 rows (m) x 64 tokens
    static constexpr int B_BYTES = (NST / 64) * KT * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = NST;              // 64, 128 or 256 (powers of two)
    static constexpr int W_OFF = NSTAGE * STAGE;       // decay weights [HPC][QMAX] fp32
    static constexpr int BAR_OFF = W_OFF + HPC * QMAX * 4;
    static constexpr int SMEM = BAR_OFF + 64 + 1024;   // + alignment slack
};

__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float w) {
    uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&in[i]);
        const float2 f = __bfloat1622float2(h);
        out[i] = pack_bf16x2(f.x * w, f.y * w);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

template <int NST, int PD>
__global__ void __launch_bounds__(256, 1) chunk_state_tc_kernel(FwdParams p) {
    using T = StateTile<NST, PD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float* wtab = reinterpret_cast<float*>(smem + T::W_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NSTAGE);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks, G = p.ngroups;
    const int64_t hblocks = H / T::HPC;
    const int64_t c = blockIdx.x / hblocks, h0 = (blockIdx.x % hblocks) * T::HPC;
    const int64_t b = blockIdx.y, g = h0 / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(smem_u32(&bars[s]), 1);
        fence_mbar_init();
    }
    for (int i = tid; i < T::HPC * QMAX; i += 256) {
        const int hh = i / QMAX, l = i % QMAX;
        float w = 0.0f;
        if (l < Lc) {
            const int64_t base = ((b * H + h0 + hh) * nc + c) * Q;
            w = expf(p.cumA[base + Q - 1] - p.cumA[base + l]) * p.dt[base + l];
        }
        wtab[i] = w;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
    const __nv_bfloat16* Bm = static_cast<const __nv_bfloat16*>(p.B);
    const int nkt = (Lc + KT - 1) / KT;
    constexpr uint32_t idesc = idesc_bf16(128, NST, true, true);
    bool ok = true;
    for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % NSTAGE;
        uint8_t* As = smem + s * T::STAGE;
        uint8_t* Bs = As + T::A_BYTES;
        if (kt >= NSTAGE) {  // wait until the MMAs that read this stage are done
            const bool w = mbar_wait(smem_u32(&bars[s]), ((kt / NSTAGE) - 1) & 1);
            if (__syncthreads_or(!w)) {
                ok = false;
                break;
            }
        }
        // A: 64 token rows x 16 chunks (two 64-wide m blocks)
#pragma unroll 4
        for (int i = tid; i < KT * 16; i += 256) {
            const int r = i >> 4, cc = i & 15, blk = cc >> 3, ch = cc & 7;
            const int l = kt * KT + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (l < Lc) {
                const int m = blk * 64 + ch * 8;
                v = ldg16(x + ((b * L + t0 + l) * H + h0) * PD + m);
                v = scale_bf16x8(v, wtab[(m / PD) * QMAX + l]);
            }
            st_shared_v4(smem_u32(As) + blk * (KT * 128) + sw128(r, ch), v.x, v.y, v.z, v.w);
        }
        // B: 64 token rows x NST/8 chunks
#pragma unroll 4
        for (int i = tid; i < KT * (NST / 8); i += 256) {
            const int r = i / (NST / 8), cc = i % (NST / 8), blk = cc >> 3, ch = cc & 7;
            const int l = kt * KT + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (l < Lc) v = ldg16(Bm + ((b * L + t0 + l) * G + g) * NST + cc * 8);
            st_shared_v4(smem_u32(Bs) + blk * (KT * 128) + sw128(r, ch), v.x, v.y, v.z, v.w);
        }
        fence_smem_async();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
#pragma unroll
            for (int k = 0; k < KT / 16; ++k) {
                const uint64_t ad = desc_sw128(smem_u32(As) + k * 2048, KT * 128, 1024);
                const uint64_t bd = desc_sw128(smem_u32(Bs) + k * 2048, KT * 128, 1024);
                mma_bf16(tmem, ad, bd, idesc, (kt > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(smem_u32(&bars[s]));
        }
    }
    if (ok) {
        const int last = nkt - 1;
        const bool w = mbar_wait(smem_u32(&bars[last % NSTAGE]), (last / NSTAGE) & 1);
        if (__syncthreads_or(!w)) ok = false;
    }
    fence_after_sync();
    if (ok) {
        // warp w reads TMEM lanes 32*(w%4).. (rows m), warpgroup w/4 half the columns
        const int m = 32 * (warp & 3) + lane;
        const int64_t hh = m / PD, pp = m % PD;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.states) +
                             (((b * nc + c) * H + h0 + hh) * PD + pp) * NST;
        constexpr int HALF = NST / 2;
        const int cbeg = (warp >> 2) * HALF;
#pragma unroll
        for (int col = 0; col < HALF; col += 32) {
            float v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + cbeg + col, v);
            uint4* o = reinterpret_cast<uint4*>(out + cbeg + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]),
                                  pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                  pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        }
    } else if (tid == 0 && p.status) {
        atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

template <int NST, int PD>
cudaError_t launch_nd(const FwdParams& p, cudaStream_t s) {
    using T = StateTile<NST, PD>;
    auto kern = chunk_state_tc_kernel<NST, PD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>(p.nchunks * (p.nheads / T::HPC)), static_cast<unsigned>(p.batch));
    kern<<<grid, 256, T::SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool chunk_state_tc_supported(const FwdParams& p) {
    const int64_t P = p.headdim, N = p.dstate;
    if (!(P == 32 || P == 64 || P == 128)) return false;
    if (!(N == 64 || N == 128 || N == 256)) return false;
    if (p.chunk > QMAX) return false;
    const int64_t hpc = 128 / P;
    return p.heads_per_group % hpc == 0;
}

cudaError_t launch_chunk_state_tc(const FwdParams& p, cudaStream_t s) {
#define SSD_STATE_CASE(NN, PP) \
    if (p.dstate == NN && p.headdim == PP) return launch_nd<NN, PP>(p, s);
    SSD_STATE_CASE(64, 32) SSD_STATE_CASE(64, 64) SSD_STATE_CASE(64, 128)
    SSD_STATE_CASE(128, 32) SSD_STATE_CASE(128, 64) SSD_STATE_CASE(128, 128)
    SSD_STATE_CASE(256, 32) SSD_STATE_CASE(256, 64) SSD_STATE_CASE(256, 128)
#undef SSD_STATE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace ssd
