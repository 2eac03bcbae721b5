// chunk_state_tc.cu -- step 2 of the chunked SSD forward on the sm_100a tensor
// cores: every chunk's local state
//   S_c[p,n] = sum_{l in c} (exp(cumA[last] - cumA[l]) dt[l] x[l,p]) B[l,n]
// (the "diagonal block: local state" of "MAMBA-2 Implementation Gaps", Gap 1),
// as one GEMM per CTA with tcgen05.mma (bf16 operands, fp32 accumulation in
// TMEM):
//   D[m, n] = sum_l A[m, l] B[l, n],  m = (head, p) over 128/P heads of one
//   group (M = 128), n = 0..dstate-1 (N = dstate), K = the chunk's tokens.
// Both operands are MN-major and arrive by TMA exactly as they sit in memory:
// A is x viewed as 64-element units (for a token, the 128/P heads' P values
// are two contiguous units), B the group's B rows.  The chunk streams through
// a two-slot ring of 64-token quarters.  Warps 0-7 fold the decay weight into
// a quarter of x in place (bf16 -> fp32 -> bf16) as soon as it has landed;
// one lane of warp 8 issues the quarter's MMAs once it is scaled and refills
// the slot by TMA as soon as those MMAs are done, so loads stay in flight
// while the previous quarter is scaled and multiplied (mbarriers per slot:
// loaded, scaled, free).  With 64 KB of shared memory (dstate 128) three CTAs
// share an SM, so one CTA's loads overlap another's MMAs and epilogue.  The
// epilogue moves the fp32 accumulator from TMEM to the states buffer, in fp32
// (the forward's split-step path) or bf16 (the backward's recompute and the
// opt-in bf16-states mode), one row of dstate per thread.  When the forward call fuses step 1, the first
// 128/P warps first form dt and cumA of the CTA's heads with the same warp
// scan as step 1 and store them for steps 3 and 4.
#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int KT = 64;      // tokens per quarter
constexpr int NSLOT = 2;    // ring slots
constexpr int QMAX = 256;
constexpr int NSCALE = 256;             // scaler / epilogue threads (warps 0-7)
constexpr int NTHR = NSCALE + 32;       // + the control warp
enum : int { B_LOADED = 0, B_SCALED = NSLOT, B_FREE = 2 * NSLOT, B_DONE = 3 * NSLOT, B_NBARS };

template <int NST, int PD>
struct StateTile {
    static constexpr int HPC = 128 / PD;                 // heads per CTA
    static constexpr int A_BLK = KT * 128;               // one 64-wide m block of a quarter
    static constexpr int A_BYTES = 2 * A_BLK;
    static constexpr int B_BLK = KT * 128;               // one 64-wide n block of a quarter
    static constexpr int B_BYTES = (NST / 64) * B_BLK;
    static constexpr int SLOT = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = NST;                // 64, 128 or 256
    static constexpr int W_OFF = NSLOT * SLOT;           // decay weights [HPC][QMAX] fp32
    static constexpr int BAR_OFF = W_OFF + HPC * QMAX * 4;
    static constexpr int SMEM = BAR_OFF + B_NBARS * 8 + 16 + 1024;  // + alignment slack
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float w) {
    uint32_t in[4] = {v.x, v.y, v.z, v.w}, out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[i]));
        out[i] = pack_bf16x2(f.x * w, f.y * w);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

template <int NST, int PD>
__global__ void __launch_bounds__(NTHR, NST == 256 ? 2 : 3)  // CTAs per SM that fit
    chunk_state_tc_kernel(const __grid_constant__ FwdParams p,
                          const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_s, int tma_out) {
    using T = StateTile<NST, PD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* wtab = reinterpret_cast<float*>(smem + T::W_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_NBARS);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int64_t hblocks = H / T::HPC;
    const int64_t c = blockIdx.x / hblocks, h0 = (blockIdx.x % hblocks) * T::HPC;
    const int64_t b = blockIdx.y, g = h0 / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int nq = (Lc + KT - 1) / KT;
    const uint32_t s0 = smem_u32(smem);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const int unit0 = static_cast<int>(h0 * PD / 64);     // x in 64-element units
    // quarter q -> slot q % NSLOT: A blocks then B blocks
    auto issue = [&](int q) {
        const int sl = q % NSLOT;
        const uint32_t sa = s0 + sl * T::SLOT;
        mbar_expect_tx(bar(B_LOADED + sl), T::SLOT);
        for (int blk = 0; blk < 2; ++blk)
            tma_load_4d(sa + blk * T::A_BLK, &tm_x, bar(B_LOADED + sl), 0, unit0 + blk,
                        static_cast<int>(t0 + q * KT), static_cast<int>(b));
        for (int nb = 0; nb < NST / 64; ++nb)
            tma_load_4d(sa + T::A_BYTES + nb * T::B_BLK, &tm_b, bar(B_LOADED + sl), nb * 64,
                        static_cast<int>(g), static_cast<int>(t0 + q * KT), static_cast<int>(b));
    };

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < B_NBARS; ++i)
            mbar_init(bar(i), (i >= B_SCALED && i < B_SCALED + NSLOT) ? NSCALE : 1u);
        *abort = 0;
        fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == NSCALE / 32) {
        // ----- control: TMA ring producer and MMA issuer (one lane) -----
        if (lane == 0) {
            tma_prefetch_map(&tm_x);
            tma_prefetch_map(&tm_b);
            for (int q = 0; q < nq && q < NSLOT; ++q) issue(q);  // x and B are inputs
            constexpr uint32_t idesc = idesc_bf16(128, NST, true, true);
            bool ok = true;
            for (int q = 0; ok && q < nq; ++q) {
                const int sl = q % NSLOT, use = q / NSLOT;
                const uint32_t sa = s0 + sl * T::SLOT, sb = sa + T::A_BYTES;
                ok = wait_or_abort(bar(B_SCALED + sl), use & 1, abort);
                if (!ok) break;
                fence_after_sync();
#pragma unroll
                for (int k = 0; k < KT / 16; ++k)
                    mma_bf16(tmem, desc_sw128(sa + k * 2048, T::A_BLK, 1024),
                             desc_sw128(sb + k * 2048, T::B_BLK, 1024), idesc,
                             (q > 0 || k > 0) ? 1u : 0u);
                mma_commit(bar(B_FREE + sl));
                if (q + NSLOT < nq) {  // refill this slot once its MMAs are done
                    ok = wait_or_abort(bar(B_FREE + sl), use & 1, abort);
                    if (ok) issue(q + NSLOT);
                }
            }
            if (ok) mma_commit(bar(B_DONE));
            else *abort = 1;
        }
    } else {
        // ----- scalers (warps 0-7): decay weights, x scaling, epilogue -----
        grid_dep_wait();  // dt and cumA are formed here (step 1 fused) or come from step 1
        if (p.fuse_cumsum) {
            // step 1 here: warp hh forms head hh's dt and cumA, stores them
            // for steps 3 and 4, and writes its decay weights into wtab
            if (warp < T::HPC) {
                const int64_t off = ((b * H + h0 + warp) * nc + c) * Q;
                chunk_cumsum_warp<__nv_bfloat16>(p, b, c, h0 + warp, p.dt + off, p.cumA + off, lane,
                                                 wtab + warp * QMAX);
            }
            if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0 && p.status) *p.status = 0;  // a new call
            grid_dep_launch();
        } else {
            grid_dep_launch();
            for (int i = tid; i < T::HPC * QMAX; i += NSCALE) {
                const int hh = i / QMAX, l = i % QMAX;
                float w = 0.0f;
                if (l < Lc) {
                    const int64_t base = ((b * H + h0 + hh) * nc + c) * Q;
                    w = expf(p.cumA[base + Q - 1] - p.cumA[base + l]) * p.dt[base + l];
                }
                wtab[i] = w;
            }
        }
        named_sync(1, NSCALE);
        bool ok = true;
        for (int q = 0; q < nq; ++q) {
            const int sl = q % NSLOT, use = q / NSLOT;
            const uint32_t sa = s0 + sl * T::SLOT;
            ok = wait_or_abort(bar(B_LOADED + sl), use & 1, abort);
            if (!ok) break;
            // fold the decay weights into this quarter of x: 2 blocks x 64 rows x 8 chunks
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = tid + NSCALE * k;
                const int blk = i >> 9, r = (i >> 3) & 63, ch = i & 7;
                const uint32_t addr = sa + blk * T::A_BLK + sw128(r, ch);
                const int hh = (blk * 64 + ch * 8) / PD;
                const uint4 v = ld_shared_v4(addr);
                const uint4 o = scale_bf16x8(v, wtab[hh * QMAX + q * KT + r]);
                st_shared_v4(addr, o.x, o.y, o.z, o.w);
            }
            fence_smem_async();
            mbar_arrive(bar(B_SCALED + sl));
        }
        if (ok) ok = wait_or_abort(bar(B_DONE), 0, abort);
        fence_after_sync();
        // fp32 states with dstate <= 128: the 128 x NST tile is staged in the
        // ring (free once every MMA is done) in 32-column SW128 boxes and
        // leaves by TMA stores, instead of 16-byte stores from every thread
        if (ok) {
            // warp w reads TMEM lanes 32*(w%4).. (rows m), warpgroup w/4 half the columns
            const int m = 32 * (warp & 3) + lane;
            const int64_t hh = m / PD, pp = m % PD;
            const int64_t row = (((b * nc + c) * H + h0 + hh) * PD + pp) * NST;
            constexpr int HALF = NST / 2;
            const int cbeg = (warp >> 2) * HALF;
#pragma unroll
            for (int col = 0; col < HALF; col += 32) {
                float v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + cbeg + col, v);
                if (NST <= 128 && tma_out) {
                    const uint32_t dst = s0 + ((cbeg + col) / 32) * (128 * 128);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        st_shared_v4(dst + sw128(m, k), __float_as_uint(v[4 * k]), __float_as_uint(v[4 * k + 1]),
                                     __float_as_uint(v[4 * k + 2]), __float_as_uint(v[4 * k + 3]));
                } else if (p.states_f32) {  // fp32 states, as the forward keeps them
                    float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.states) + row + cbeg + col);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        o[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                } else {
                    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.states) + row + cbeg + col);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        o[k] = make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]),
                                          pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                                          pack_bf16x2(v[8 * k + 4], v[8 * k + 5]),
                                          pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
                }
            }
        }
        if (NST <= 128 && tma_out) {
            fence_smem_async();     // the staged tile is read by the TMA (async proxy)
            named_sync(2, NSCALE);  // every row is staged
            if (tid == 0 && ok && !*abort) {
                const int row0 = static_cast<int>(((b * nc + c) * H + h0) * PD);
                for (int box = 0; box < NST / 32; ++box)
                    tma_store_2d(&tm_s, s0 + box * (128 * 128), box * 32, row0);
                bulk_commit_group();
                bulk_wait_all();  // written before the CTA ends (and its shared memory with it)
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (*abort && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

template <int NST, int PD>
cudaError_t launch_nd(const FwdParams& p, cudaStream_t s) {
    using T = StateTile<NST, PD>;
    CUtensorMap tx_, tb_, ts_;
    if (!make_tmap_bf16_4d(&tx_, p.x, 64, p.nheads * PD / 64, p.seqlen, p.batch, 1, KT) ||
        !make_tmap_bf16_4d(&tb_, p.B, NST, p.ngroups, p.seqlen, p.batch, 1, KT))
        return cudaErrorInvalidValue;
    // the fp32 states as rows of NST: [batch * nchunks * nheads * headdim][NST]
    // (row coordinates are 32-bit)
    const int64_t srows = p.batch * p.nchunks * p.nheads * PD;
    const int tma_out = (NST <= 128 && p.states_f32 && srows < (1ll << 31)) ? 1 : 0;
    if (tma_out) {
        if (!make_tmap_f32_2d(&ts_, p.states, NST, srows, 128)) return cudaErrorInvalidValue;
    } else {
        ts_ = tx_;  // not read
    }
    auto kern = chunk_state_tc_kernel<NST, PD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>(p.nchunks * (p.nheads / T::HPC)), static_cast<unsigned>(p.batch));
    return launch_kernel(kern, grid, dim3(NTHR), T::SMEM, s, p.pdl != 0, p, tx_, tb_, ts_, tma_out);
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
