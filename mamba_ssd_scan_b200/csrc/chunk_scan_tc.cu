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
// One CTA serves a block of heads that share a group's B and C: TMA brings the
// chunk's C and B rows once, tcgen05.mma computes CB = C B^T once into TMEM
// (K = dstate), and then each head reuses it.  Per head and per 128-row output
// tile t, the CUDA cores read CB back, apply the causal decay mask and write Mk
// as a bf16 K-major operand to shared memory; the tensor core accumulates the
// state term C_t H_in^T and Mk x into TMEM; the epilogue adds D x and stores y.
// Each head's x tile arrives by TMA into one of two buffers while the previous
// head computes; its state entering the chunk (bf16, as state passing left it)
// arrives by TMA too.  Decays are never formed as exp(cumA_l) / exp(cumA_j): below
// the 32x32 diagonal blocks the factor is split as exp(cumA_l - cumA_r) *
// exp(cumA_r - cumA_j) with r the first row of the thread's 32-row block (both
// factors <= 1, one table of the second per warp); only the diagonal blocks
// take one exp per element.
//
// TMEM (512 columns): CB of tile 1 [0,256) and of tile 0 [256,384) stay for
// every head; [384,448) and [448,512) hold the state and intra-chunk
// accumulators of the tile in flight.
#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int QMAX = 256;
constexpr int PD = 64;
constexpr uint32_t ST_COL = 384, IN_COL = 448;

template <int NST>
struct ScanTile {
    static constexpr int KB_BYTES = QMAX * 128;                    // one 64-wide K block, 256 rows
    static constexpr int C_OFF = 0;
    static constexpr int C_BYTES = (NST / 64) * KB_BYTES;
    static constexpr int B_OFF = C_OFF + C_BYTES;
    static constexpr int MASK_BYTES = 4 * 128 * 128;               // [4 kb][128 rows][128 B]
    static constexpr int B_BYTES = C_BYTES > MASK_BYTES ? C_BYTES : MASK_BYTES;
    static constexpr int X_OFF = B_OFF + B_BYTES;
    static constexpr int X_BYTES = QMAX * 128;                     // MN-major [j][64 p]
    static constexpr int H_OFF = X_OFF + 2 * X_BYTES;              // two x buffers
    static constexpr int H_BYTES = (NST / 64) * PD * 128;          // K-major [kb][p][64 n]
    static constexpr int CUM_OFF = H_OFF + H_BYTES;
    static constexpr int DT_OFF = CUM_OFF + QMAX * 4;
    static constexpr int STAB_OFF = DT_OFF + QMAX * 4;             // 8 warps x QMAX fp32
    static constexpr int BAR_OFF = STAB_OFF + 8 * QMAX * 4;
    static constexpr int SMEM = BAR_OFF + 128 + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t cb_col(int t) { return t == 0 ? 256u : 0u; }

// Mk for the 128 rows of tile t, column groups of 32 split over the two
// warpgroups; written as bf16 into the K-major mask operand.
__device__ __forceinline__ void build_mask(int t, uint32_t tmem, uint32_t mbase, const float* cum,
                                           const float* dtv, float* stab, int warp, int lane) {
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
__device__ __forceinline__ void epilogue(int t, uint32_t tmem, uint32_t xbase, const float* cum,
                                         const FwdParams& p, int64_t b, int64_t t0, int64_t h,
                                         int Lc, int warp, int lane) {
    const int r = 32 * (warp & 3) + lane;
    const int l = 128 * t + r;
    const int pc = 32 * (warp >> 2);
    const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    float vi[32], vs[32];
    tmem_ld32x2(tmem + lane_addr + IN_COL + pc, vi, tmem + lane_addr + ST_COL + pc, vs);
    if (l >= Lc) return;
    const float sc = __expf(cum[l]);
    const float Dh = p.D ? p.D[h] : 0.0f;
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
            o[k] = pack_bf16x2(vi[q] + sc * vs[q] + Dh * xf.x,
                               vi[q + 1] + sc * vs[q + 1] + Dh * xf.y);
        }
        reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

template <int NST>
__global__ void __launch_bounds__(256, 1)
    chunk_scan_tc_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_c,
                         const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_h, int hb_size) {
    using T = ScanTile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    float* cum = reinterpret_cast<float*>(smem + T::CUM_OFF);
    float* dtv = reinterpret_cast<float*>(smem + T::DT_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    // barriers: 0 = C/B landed, 1 = CB done, 2/3 = x buffer 0/1 landed, 4 = tile-0 MMAs,
    // 5 = tile-1 MMAs, 6 = H_in landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks, G = p.ngroups;
    const int64_t hpg = p.heads_per_group, nhb = hpg / hb_size;
    const int64_t c = blockIdx.x / (G * nhb), g = (blockIdx.x / nhb) % G;
    const int64_t hfirst = g * hpg + (blockIdx.x % nhb) * hb_size, b = blockIdx.y;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int ntiles = (Lc + 127) / 128;
    float* stab = reinterpret_cast<float*>(smem + T::STAB_OFF) + warp * QMAX;
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sX = smem_u32(smem + T::X_OFF), sH = smem_u32(smem + T::H_OFF);
    const uint32_t sM = sB;  // the mask operand reuses B's space once CB is done
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(bar(i), 1);
        fence_mbar_init();
        tma_prefetch_map(&tm_c);
        tma_prefetch_map(&tm_b);
        tma_prefetch_map(&tm_x);
        tma_prefetch_map(&tm_h);
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t box = static_cast<uint32_t>(Q) * 128;
        mbar_expect_tx(bar(0), 2 * (NST / 64) * box);
        for (int kb = 0; kb < NST / 64; ++kb) {
            tma_load_4d(sC + kb * T::KB_BYTES, &tm_c, bar(0), kb * 64, (int)g, (int)t0, (int)b);
            tma_load_4d(sB + kb * T::KB_BYTES, &tm_b, bar(0), kb * 64, (int)g, (int)t0, (int)b);
        }
        for (int i = 0; i < 2 && i < hb_size; ++i) {
            mbar_expect_tx(bar(2 + i), box);
            tma_load_4d(sX + i * T::X_BYTES, &tm_x, bar(2 + i), 0, (int)(hfirst + i), (int)t0, (int)b);
        }
        mbar_expect_tx(bar(6), T::H_BYTES);
        for (int kb = 0; kb < NST / 64; ++kb)
            tma_load_4d(sH + kb * (PD * 128), &tm_h, bar(6), kb * 64, 0, (int)hfirst,
                        (int)(b * nc + c));
    }
    // first head's decays
    {
        const int64_t vbase = ((b * H + hfirst) * nc + c) * Q;
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

    bool mine = true;
    if (tid == 0) {
        mine = mbar_wait(bar(0), 0);
        if (mine) {
            fence_after_sync();
            for (int t = 0; t < ntiles; ++t) {
                const uint32_t id = t == 0 ? idesc_bf16(128, 128, false, false)
                                           : idesc_bf16(128, 256, false, false);
                for (int k = 0; k < NST / 16; ++k) {
                    const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                    mma_bf16(tmem + cb_col(t), desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                             desc_sw128(sB + ko, 16, 1024), id, k > 0 ? 1u : 0u);
                }
            }
            mma_commit(bar(1));
        }
    }
    bool ok = !__syncthreads_or(!mine);
    if (ok) ok = !__syncthreads_or(!mbar_wait(bar(1), 0));
    fence_after_sync();

    for (int i = 0; ok && i < hb_size; ++i) {
        const int64_t h = hfirst + i;
        const int xb = i & 1;
        const uint32_t xbase = sX + xb * T::X_BYTES;
        // every thread observes the x tile's arrival (the epilogue reads it too)
        ok = !__syncthreads_or(!mbar_wait(bar(2 + xb), (i >> 1) & 1));
        if (!ok) break;
        // the next head's decays, into registers now, into shared memory at the end
        float cum_next = 0.0f, dt_next = 0.0f;
        if (i + 1 < hb_size && tid < Q) {
            const int64_t vbase = ((b * H + h + 1) * nc + c) * Q;
            cum_next = p.cumA[vbase + tid];
            dt_next = p.dt[vbase + tid];
        }
        for (int t = 0; t < ntiles; ++t) {
            // CUDA cores: the decay mask of tile t
            build_mask(t, tmem, sM, cum, dtv, stab, warp, lane);
            fence_smem_async();
            fence_before_sync();
            __syncthreads();
            // tensor core: state term and Mk x of tile t (the state has to have landed)
            bool mine = true;
            if (tid == 0) {
                fence_after_sync();
                if (t == 0) mine = mbar_wait(bar(6), i & 1);
                if (mine) {
                    for (int k = 0; k < NST / 16; ++k) {
                        const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                        const uint32_t kh = (k >> 2) * (PD * 128) + (k & 3) * 32;
                        mma_bf16(tmem + ST_COL, desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                                 desc_sw128(sH + kh, 16, 1024), idesc_bf16(128, PD, false, false),
                                 k > 0 ? 1u : 0u);
                    }
                    for (int k = 0; k < 8 * (t + 1); ++k) {
                        mma_bf16(tmem + IN_COL,
                                 desc_sw128(sM + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024),
                                 desc_sw128(xbase + k * 2048, QMAX * 128, 1024),
                                 idesc_bf16(128, PD, false, true), k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(4 + t));
                }
            }
            ok = !__syncthreads_or(!mine);
            if (ok) ok = !__syncthreads_or(!mbar_wait(bar(4 + t), i & 1));
            fence_after_sync();
            if (!ok) break;
            epilogue(t, tmem, xbase, cum, p, b, t0, h, Lc, warp, lane);
            fence_before_sync();
            __syncthreads();
        }
        if (!ok) break;
        // the next head's decays; its x and state are already on the way
        if (i + 1 < hb_size) {
            cum[tid] = cum_next;
            dtv[tid] = dt_next;
        }
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            // every MMA of this head is done: its H_in buffer takes the next head's
            // state, its x buffer head i + 2's x
            if (i + 1 < hb_size) {
                mbar_expect_tx(bar(6), T::H_BYTES);
                for (int kb = 0; kb < NST / 64; ++kb)
                    tma_load_4d(sH + kb * (PD * 128), &tm_h, bar(6), kb * 64, 0, (int)(h + 1),
                                (int)(b * nc + c));
            }
            if (i + 2 < hb_size) {
                mbar_expect_tx(bar(2 + xb), static_cast<uint32_t>(Q) * 128);
                tma_load_4d(xbase, &tm_x, bar(2 + xb), 0, (int)(h + 2), (int)t0, (int)b);
            }
        }
    }
    if (!ok && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// heads per CTA: the largest divisor of the heads per group that still leaves
// at least two CTAs per SM of work (or every head of the group, when asked)
int heads_per_cta(const FwdParams& p) {
    if (p.flags & SSD_FLAG_WHOLE_GROUPS) return static_cast<int>(p.heads_per_group);
    const int64_t units = p.batch * p.nchunks * p.ngroups;
    int best = 1;
    for (int d = 1; d <= p.heads_per_group; ++d)
        if (p.heads_per_group % d == 0 && units * (p.heads_per_group / d) >= 2 * 148) best = d;
    return best;
}

template <int NST>
cudaError_t launch_n(const FwdParams& p, cudaStream_t s) {
    using T = ScanTile<NST>;
    CUtensorMap tc_, tb_, tx_, th_;
    const uint32_t rows = static_cast<uint32_t>(p.chunk);
    if (!make_tmap_bf16_4d(&tc_, p.C, NST, p.ngroups, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&tb_, p.B, NST, p.ngroups, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&tx_, p.x, PD, p.nheads, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&th_, p.states, NST, PD, p.nheads, p.batch * p.nchunks, PD, 1))
        return cudaErrorInvalidValue;
    auto kern = chunk_scan_tc_kernel<NST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    const int hb = heads_per_cta(p);
    dim3 grid(static_cast<unsigned>(p.nchunks * p.ngroups * (p.heads_per_group / hb)),
              static_cast<unsigned>(p.batch));
    kern<<<grid, 256, T::SMEM, s>>>(p, tc_, tb_, tx_, th_, hb);
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
