// chunk_scan_tc.cu -- step 4 of the chunked SSD forward on the sm_100a tensor
// cores.  For one (batch, chunk, head):
//
//   y[l,p] = sum_{j<=l} Mk[l,j] x[j,p]  +  exp(cumA[l]) sum_n C[l,n] H_in[p,n]  +  D x[l,p]
//   Mk[l,j] = (C_l . B_j) exp(cumA[l] - cumA[j]) dt[j]        (j <= l, else 0)
//
// i.e. the masked-attention dual form of SSD inside the chunk ("MAMBA-2
// Reference Implementations Comparison", section 2.2), the carried state's
// off-diagonal contribution ("MAMBA-2 Implementation Gaps", Gap 1) and the D
// skip (Gap 4).
//
// The chunk (Q = 128 or 256 tokens) is cut into 128-row output tiles t.  Per
// tile, tcgen05.mma computes CB = C_t B^T (K = dstate) and the state term
// C_t H_in^T (K = dstate) into TMEM; the CUDA cores read CB back, apply the
// causal decay mask and write Mk as a bf16 K-major operand to shared memory;
// a second MMA accumulates Mk x (K = tokens up to the tile's end).  Decays are
// never formed as exp(cumA_l) / exp(cumA_j): below the 32x32 diagonal blocks
// the factor is split as exp(cumA_l - cumA_r) * exp(cumA_r - cumA_j) with r
// the first row of the thread's 32-row block (both factors <= 1, one table of
// the second per warp), and only the diagonal blocks take one exp per element.
//
// TMEM (512 columns): CB of tile 1 [0,256), CB of tile 0 [256,384), tile 0's
// state/intra accumulators [384,448)/[448,512); tile 1's accumulators reuse
// [256,320)/[320,384) once tile 0's CB has been read.  Shared memory holds C,
// B (later reused for Mk), x and H_in (bf16) as SW128 tiles.
#include "internal.cuh"
#include "tcgen05.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int QMAX = 256;
constexpr int PD = 64;

template <int NST>
struct ScanTile {
    static constexpr int KB_BYTES = QMAX * 128;                    // one 64-wide K block, 256 rows
    static constexpr int C_OFF = 0;
    static constexpr int C_BYTES = (NST / 64) * KB_BYTES;
    static constexpr int B_OFF = C_OFF + C_BYTES;
    static constexpr int MASK_BYTES = 4 * 128 * 128;               // [4 kb][128 rows][128 B]
    static constexpr int B_BYTES = C_BYTES > MASK_BYTES ? C_BYTES : MASK_BYTES;
    static constexpr int X_OFF = B_OFF + B_BYTES;
    static constexpr int X_BYTES = QMAX * 128;                     // MN-major, P = 64
    static constexpr int H_OFF = X_OFF + X_BYTES;
    static constexpr int H_BYTES = (NST / 64) * PD * 128;          // K-major [kb][p][64 n]
    static constexpr int CUM_OFF = H_OFF + H_BYTES;
    static constexpr int DT_OFF = CUM_OFF + QMAX * 4;
    static constexpr int STAB_OFF = DT_OFF + QMAX * 4;             // 8 warps x QMAX fp32
    static constexpr int BAR_OFF = STAB_OFF + 8 * QMAX * 4;
    static constexpr int SMEM = BAR_OFF + 64 + 1024;
};

// TMEM column of tile t's CB, state accumulator and intra-chunk accumulator
__device__ __forceinline__ uint32_t cb_col(int t) { return t == 0 ? 256u : 0u; }
__device__ __forceinline__ uint32_t st_col(int t) { return t == 0 ? 384u : 256u; }
__device__ __forceinline__ uint32_t in_col(int t) { return t == 0 ? 448u : 320u; }

// Mk for the 128 rows of tile t, column groups of 32 split over the two
// warpgroups; written as bf16 into the K-major mask operand.
template <int NST>
__device__ __forceinline__ void build_mask(int t, uint32_t tmem, uint8_t* smem, const float* cum,
                                           const float* dtv, float* stab, int warp, int lane) {
    using T = ScanTile<NST>;
    const int rb = 32 * (warp & 3);             // tile-local row block
    const int lb = 128 * t + rb;                // chunk row of the block's first row
    const int l = lb + lane;                    // this thread's chunk row
    const float cl = cum[l];
    // per-warp table: s[j] = exp(cum[lb] - cum[j]) dt[j], j < lb
    for (int j = lane; j < lb; j += 32) stab[j] = __expf(cum[lb] - cum[j]) * dtv[j];
    __syncwarp();
    const float rl = __expf(cl - cum[lb]);
    const int ngroups = 4 * (t + 1);            // 32-wide column groups in [0, 128(t+1))
    const int half = ngroups / 2;
    const int gbeg = (warp >> 2) * half;
    const uint32_t mbase = smem_u32(smem + T::B_OFF);
    const uint32_t lane_addr = static_cast<uint32_t>(rb) << 16;
    for (int gi = gbeg; gi < gbeg + half; ++gi) {
        const int j0 = 32 * gi;
        float v[32];
        if (j0 + 32 <= lb) {
            tmem_ld32(tmem + lane_addr + cb_col(t) + j0, v);
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= rl * stab[j0 + q];
        } else if (j0 == lb) {
            tmem_ld32(tmem + lane_addr + cb_col(t) + j0, v);
#pragma unroll
            for (int q = 0; q < 32; ++q)
                v[q] = (q <= lane) ? v[q] * __expf(cl - cum[j0 + q]) * dtv[j0 + q] : 0.0f;
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = 0.0f;
        }
        const int kb = j0 >> 6, c0 = (j0 & 63) >> 3;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            st_shared_v4(mbase + kb * (128 * 128) + sw128(rb + lane, c0 + i),
                         pack_bf16x2(v[8 * i + 0], v[8 * i + 1]),
                         pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                         pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                         pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    }
}

// y rows of tile t: warp w%4 -> rows, warpgroup -> 32 of the 64 p columns
template <int NST>
__device__ __forceinline__ void epilogue(int t, uint32_t tmem, const uint8_t* smem,
                                         const float* cum, const FwdParams& p, int64_t b,
                                         int64_t t0, int64_t h, int Lc, int warp, int lane) {
    using T = ScanTile<NST>;
    const int r = 32 * (warp & 3) + lane;
    const int l = 128 * t + r;
    const int pc = 32 * (warp >> 2);
    const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    float vi[32], vs[32];
    tmem_ld32(tmem + lane_addr + in_col(t) + pc, vi);
    tmem_ld32(tmem + lane_addr + st_col(t) + pc, vs);
    if (l >= Lc) return;
    const float sc = __expf(cum[l]);
    const float Dh = p.D ? p.D[h] : 0.0f;
    const uint32_t xbase = smem_u32(smem + T::X_OFF);
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.y) +
                       ((b * p.seqlen + t0 + l) * p.nheads + h) * PD + pc;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 xv = ld_shared_v4(xbase + sw128(l, (pc >> 3) + i));
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[k]));
            const int q = 8 * i + 2 * k;
            o[k] = pack_bf16x2(vi[q] + sc * vs[q] + Dh * xf.x, vi[q + 1] + sc * vs[q + 1] + Dh * xf.y);
        }
        reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

template <int NST>
__global__ void __launch_bounds__(256, 1) chunk_scan_tc_kernel(FwdParams p) {
    using T = ScanTile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float* cum = reinterpret_cast<float*>(smem + T::CUM_OFF);
    float* dtv = reinterpret_cast<float*>(smem + T::DT_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks, G = p.ngroups;
    const int64_t c = blockIdx.x / H, h = blockIdx.x % H, b = blockIdx.y;
    const int64_t g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int ntiles = (Lc + 127) / 128;
    float* stab = reinterpret_cast<float*>(smem + T::STAB_OFF) + warp * QMAX;

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_mbar_init();
    }

    // ---- stage C, B, x, H_in (bf16) and the chunk's dt / cumA ----------------
    const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.C);
    const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
    const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
    const int rows = 128 * ntiles;
    {
        constexpr int CPR = NST / 8;  // 16-byte chunks per row of C / B
#pragma unroll 4
        for (int i = tid; i < rows * CPR; i += 256) {
            const int r = i / CPR, cc = i % CPR;
            uint4 vc = make_uint4(0u, 0u, 0u, 0u), vb = vc;
            if (r < Lc) {
                const int64_t off = ((b * L + t0 + r) * G + g) * NST + cc * 8;
                vc = ldg16(Cg + off);
                vb = ldg16(Bg + off);
            }
            const uint32_t o = (cc >> 3) * T::KB_BYTES + sw128(r, cc & 7);
            st_shared_v4(smem_u32(smem + T::C_OFF) + o, vc.x, vc.y, vc.z, vc.w);
            st_shared_v4(smem_u32(smem + T::B_OFF) + o, vb.x, vb.y, vb.z, vb.w);
        }
#pragma unroll 4
        for (int i = tid; i < rows * 8; i += 256) {
            const int r = i >> 3, ch = i & 7;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < Lc) v = ldg16(xg + ((b * L + t0 + r) * H + h) * PD + ch * 8);
            st_shared_v4(smem_u32(smem + T::X_OFF) + sw128(r, ch), v.x, v.y, v.z, v.w);
        }
        const float* hin = p.states + ((b * nc + c) * H + h) * PD * NST;
#pragma unroll 4
        for (int i = tid; i < PD * CPR; i += 256) {
            const int pr = i / CPR, cc = i % CPR;
            const float4 a = __ldg(reinterpret_cast<const float4*>(hin + pr * NST + cc * 8));
            const float4 d = __ldg(reinterpret_cast<const float4*>(hin + pr * NST + cc * 8 + 4));
            st_shared_v4(smem_u32(smem + T::H_OFF) + (cc >> 3) * (PD * 128) + sw128(pr, cc & 7),
                         pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(d.x, d.y),
                         pack_bf16x2(d.z, d.w));
        }
        const int64_t vbase = ((b * H + h) * nc + c) * Q;
        for (int i = tid; i < QMAX; i += 256) {
            cum[i] = (i < Q) ? p.cumA[vbase + i] : 0.0f;
            dtv[i] = (i < Q) ? p.dt[vbase + i] : 0.0f;
        }
    }
    fence_smem_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sX = smem_u32(smem + T::X_OFF), sH = smem_u32(smem + T::H_OFF);

    // ---- MMA group 1: CB for every tile, state term of tile 0 ----------------
    if (tid == 0) {
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t id = t == 0 ? idesc_bf16(128, 128, false, false)
                                       : idesc_bf16(128, 256, false, false);
            for (int k = 0; k < NST / 16; ++k) {
                const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                mma_bf16(tmem + cb_col(t), desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                         desc_sw128(sB + ko, 16, 1024), id, k > 0 ? 1u : 0u);
            }
        }
        for (int k = 0; k < NST / 16; ++k) {
            const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
            const uint32_t kh = (k >> 2) * (PD * 128) + (k & 3) * 32;
            mma_bf16(tmem + st_col(0), desc_sw128(sC + ko, 16, 1024),
                     desc_sw128(sH + kh, 16, 1024), idesc_bf16(128, PD, false, false),
                     k > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars[0]));
    }
    bool ok = mbar_wait(smem_u32(&bars[0]), 0);
    ok = !__syncthreads_or(!ok);
    fence_after_sync();

    for (int t = 0; ok && t < ntiles; ++t) {
        // ---- CUDA cores: the decay mask of tile t into shared memory ---------
        build_mask<NST>(t, tmem, smem, cum, dtv, stab, warp, lane);
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        // ---- MMA group 2: state term of tile t>0, Mk x for tile t ------------
        if (tid == 0) {
            fence_after_sync();
            if (t > 0) {
                for (int k = 0; k < NST / 16; ++k) {
                    const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                    const uint32_t kh = (k >> 2) * (PD * 128) + (k & 3) * 32;
                    mma_bf16(tmem + st_col(t), desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                             desc_sw128(sH + kh, 16, 1024), idesc_bf16(128, PD, false, false),
                             k > 0 ? 1u : 0u);
                }
            }
            const uint32_t sM = sB;
            for (int k = 0; k < 8 * (t + 1); ++k) {
                mma_bf16(tmem + in_col(t),
                         desc_sw128(sM + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024),
                         desc_sw128(sX + k * 2048, QMAX * 128, 1024),
                         idesc_bf16(128, PD, false, true), k > 0 ? 1u : 0u);
            }
            mma_commit(smem_u32(&bars[1 + t]));
        }
        ok = mbar_wait(smem_u32(&bars[1 + t]), 0);
        ok = !__syncthreads_or(!ok);
        fence_after_sync();
        if (!ok) break;
        epilogue<NST>(t, tmem, smem, cum, p, b, t0, h, Lc, warp, lane);
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
    }
    if (!ok && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

template <int NST>
cudaError_t launch_n(const FwdParams& p, cudaStream_t s) {
    using T = ScanTile<NST>;
    auto kern = chunk_scan_tc_kernel<NST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>(p.nchunks * p.nheads), static_cast<unsigned>(p.batch));
    kern<<<grid, 256, T::SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool chunk_scan_tc_supported(const FwdParams& p) {
    return p.headdim == PD && (p.dstate == 64 || p.dstate == 128) &&
           (p.chunk == 128 || p.chunk == 256);
}

cudaError_t launch_chunk_scan_tc(const FwdParams& p, cudaStream_t s) {
    if (p.dstate == 64) return launch_n<64>(p, s);
    if (p.dstate == 128) return launch_n<128>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace ssd
