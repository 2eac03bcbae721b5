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
// One CTA serves a block of heads that share a group's B and C.  TMA brings
// the chunk's C and B rows once and tcgen05.mma computes CB = C B^T for the two
// 128-row output tiles once; the CB rows are then repacked in TMEM as fp16
// pairs (192 columns instead of 384), each row scaled by a power of two that
// keeps it inside fp16's range, so that both tiles' accumulators fit beside
// them at ~2^-11 relative rounding.  The CTA is warp-specialised and its roles
// hand work to each other through mbarriers:
//
//   warps 0-7  "workers": per head and tile, read CB back, apply the causal
//              decay mask (with D on the diagonal, so the MMA also forms D x)
//              and write Mk as a bf16 K-major operand to shared memory (one
//              buffer per tile, refilled as soon as its MMA is done); then
//              drain the previous head's accumulators for the same tile
//              (y = intra + exp(cumA) * state, bf16).  Two warps share each
//              32-row block, taking alternate column groups and p halves;
//   warp 8     "control": one lane issues every TMA load (C, B once; x and
//              H_in per head) and every MMA (CB once; per head and tile the
//              state term C_t H_in^T and Mk x);
//   warp 9     "loader": stages each head's decays and D in shared memory
//              (two buffers), so the workers never wait on a global load.
//
// The tensor core thus works on head i while the CUDA cores finish head i-1
// and prepare the next tile.  Decays are never formed as exp(cumA_l) /
// exp(cumA_j): below the 32x32 diagonal blocks the factor is split as
// exp(cumA_l - cumA_r) * exp(cumA_r - cumA_j), r the first row of the 32-row
// block (both factors <= 1), and only the diagonal blocks take one exp per
// element.  Every wait is bounded; a timed-out role raises a shared abort flag
// that the others observe, and the CTA still frees its TMEM.
//
// TMEM columns: [0,64) tile 0's CB and [64,192) tile 1's CB as packed fp16
// pairs (tile 1's fp32 CB sits in [128,384) until packed); [192,256)/[256,320)
// tile 0's state/intra accumulators; [320,384)/[384,448) tile 1's.
#include <stdlib.h>

#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int QMAX = 256;
constexpr int PD = 64;
constexpr int NTHREADS = 320;  // 8 worker warps, 1 control warp, 1 loader warp
constexpr int NMASK = 256;
constexpr uint32_t CB0P = 0, CB1P = 64, CB1F = 128;
__device__ __forceinline__ uint32_t st_col(int t) { return t == 0 ? 192u : 320u; }
__device__ __forceinline__ uint32_t in_col(int t) { return t == 0 ? 256u : 384u; }

template <int NST>
struct ScanTile {
    static constexpr int KB_BYTES = QMAX * 128;              // 64-wide K block of C or B
    static constexpr int C_OFF = 0;
    static constexpr int C_BYTES = (NST / 64) * KB_BYTES;
    static constexpr int B_OFF = C_OFF + C_BYTES;            // B, later tile 1's mask
    static constexpr int MK1_BYTES = 4 * 128 * 128;
    static constexpr int B_BYTES = C_BYTES > MK1_BYTES ? C_BYTES : MK1_BYTES;
    static constexpr int MK0_OFF = B_OFF + B_BYTES;          // tile 0's mask
    static constexpr int MK0_BYTES = 2 * 128 * 128;
    static constexpr int X_OFF = MK0_OFF + MK0_BYTES;
    static constexpr int X_BYTES = QMAX * 128;
    static constexpr int H_OFF = X_OFF + X_BYTES;
    static constexpr int H_BYTES = (NST / 64) * PD * 128;
    // per-head decays, two buffers filled by the loader warp:
    // [log2e * cumA (QMAX) | dt (QMAX) | D, padding (4)] fp32
    static constexpr int DEC_FLOATS = 2 * QMAX + 4;
    static constexpr int DEC_OFF = H_OFF + H_BYTES;
    static constexpr int RINV_OFF = DEC_OFF + 2 * DEC_FLOATS * 4;  // per-row CB scale, 2 tiles
    static constexpr int STAB_OFF = RINV_OFF + 2 * 128 * 4;  // 8 mask warps x QMAX
    static constexpr int BAR_OFF = STAB_OFF + 8 * QMAX * 4;
    static constexpr int SMEM = BAR_OFF + 32 * 8 + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Optional timeline of the first CTAs (builds with -DSSD_TRACE only): each role
// stamps the SM cycle counter at its hand-offs; ssd_scan_trace_copy() reads it
// back.
#ifdef SSD_TRACE
__device__ unsigned long long g_scan_trace[8][256];
#define SCAN_TRACE(slot)                                                              \
    do {                                                                              \
        if (blockIdx.x < 8 && blockIdx.y == 0 && (slot) < 256) {                      \
            g_scan_trace[blockIdx.x][(slot)] = clock64();                             \
        }                                                                             \
    } while (0)
// SM-clock stamps of warp 0 inside the mask routine, head 1 only
#define MASK_CLOCK(slot)                                                              \
    do {                                                                              \
        if (blockIdx.x < 8 && blockIdx.y == 0 && threadIdx.x == 0)                    \
            g_scan_trace[blockIdx.x][(slot)] = clock64();                             \
    } while (0)
#else
#define SCAN_TRACE(slot) \
    do {                 \
    } while (0)
#define MASK_CLOCK(slot) \
    do {                 \
    } while (0)
#endif

enum : int {
    B_CB_LOAD = 0, B_CB_DONE, B_CB_PACKED, B_X_FULL, B_H_FULL, B_H_FREE, B_X_FREE,
    B_MK_FULL, B_MK_EMPTY = B_MK_FULL + 2, B_ACC_FULL = B_MK_EMPTY + 2,
    B_ACC_EMPTY = B_ACC_FULL + 2, B_DEC_FULL = B_ACC_EMPTY + 2, B_DEC_FREE = B_DEC_FULL + 2,
    B_COUNT = B_DEC_FREE + 2
};

// Bounded wait that also gives up when another role has aborted: a few
// non-blocking probes first (most hand-offs are already complete), then
// probes that may suspend the thread for a short, bounded time, so a waiting
// warp gives its issue slots to the worker sharing its scheduler without the
// late wake-up of an unbounded suspend.
__device__ __forceinline__ bool wait_bar(uint32_t mbar, uint32_t parity, volatile int* abort) {
    for (int i = 0; i < 8; ++i)
        if (mbar_test_wait(mbar, parity)) return true;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait_hint(mbar, parity, 100)) return true;
        if ((i & 63) == 63 && *abort) return false;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void unpack_f16x32(const uint32_t (&r)[16], float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Mask warp: rows 128 t + 32 qd + lane of tile t (qd = TMEM lane quarter),
// column groups of 32 with index = hf (mod 2): 2 groups in tile 0, 4 in tile
// 1.  The warp's TMEM reads are issued together and waited for once; the
// per-block decay table is filled while they are in flight.  cum2 holds
// log2(e) * cumA, so every decay is one exp2; rinv undoes the row's CB scale.
// The skip weight D is added to the diagonal (j = l), so the MMA also forms
// D x and the epilogue needs no x.
template <int TT>
__device__ __forceinline__ void build_mask(uint32_t tmem, uint32_t mbase, const float* cum2,
                                           const float* dtv, float* stab, float rinv, float Dh,
                                           int qd, int hf, int lane) {
    constexpr int NG = 2 * (TT + 1);            // this warp's groups
    const int lb = 128 * TT + 32 * qd;          // chunk row of the block's first row
    const int l = lb + lane;
    const uint32_t cbase = tmem + (static_cast<uint32_t>(32 * qd) << 16) + (TT == 0 ? CB0P : CB1P);
    uint32_t addr[NG];
    uint32_t raw[NG][16];
#pragma unroll
    for (int k = 0; k < NG; ++k) addr[k] = cbase + 16 * (hf + 2 * k);   // j0 / 2
    MASK_CLOCK(200 + 10 * TT);
    if constexpr (NG == 2) tmem_ld16x2(addr, raw);
    else tmem_ld16x4(addr, raw);
    MASK_CLOCK(201 + 10 * TT);
    const float cl = cum2[l];
    for (int j = lane; j < lb; j += 32) stab[j] = ex2(cum2[lb] - cum2[j]) * dtv[j];
    __syncwarp();
    const float rl = ex2(cl - cum2[lb]) * rinv;
    MASK_CLOCK(202 + 10 * TT);
    const uint32_t row = 32 * qd + lane;
#pragma unroll
    for (int k = 0; k < NG; ++k) {
        const int j0 = 32 * (hf + 2 * k);
        const uint32_t dst = mbase + (j0 >> 6) * (128 * 128);
        const int c0 = (j0 & 63) >> 3;
        float v[32];
        if (j0 > lb) {  // above the diagonal: zeros
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = 0.0f;
        } else {
            unpack_f16x32(raw[k], v);
            if (j0 + 32 <= lb) {
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] *= rl * stab[j0 + q];
            } else {
                // the diagonal block: one exp2 per element, computed for every
                // lane (exponent clamped at 0, so the entries above the diagonal
                // stay finite) and then selected -- no divergent branches
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float e = ex2(fminf(cl - cum2[j0 + q], 0.0f)) * dtv[j0 + q];
                    const float m = v[q] * rinv * e + (q == lane ? Dh : 0.0f);
                    v[q] = (q <= lane) ? m : 0.0f;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            st_shared_v4(dst + sw128(row, c0 + i), pack_bf16x2(v[8 * i + 0], v[8 * i + 1]),
                         pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                         pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                         pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
        MASK_CLOCK(203 + 10 * TT + k);
    }
}

template <int NST>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_scan_tc_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_c,
                         const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_h, int hb_size) {
    using T = ScanTile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, Q = p.chunk, nc = p.nchunks, G = p.ngroups;
    const int64_t hpg = p.heads_per_group, nhb = hpg / hb_size;
    const int64_t c = blockIdx.x / (G * nhb), g = (blockIdx.x / nhb) % G;
    const int64_t hfirst = g * hpg + (blockIdx.x % nhb) * hb_size, b = blockIdx.y;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int ntiles = (Lc + 127) / 128;
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sM0 = smem_u32(smem + T::MK0_OFF), sM1 = sB;
    const uint32_t sX = smem_u32(smem + T::X_OFF), sH = smem_u32(smem + T::H_OFF);

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t count = 1;
            if (i == B_CB_PACKED) count = 128;
            if (i == B_MK_FULL || i == B_MK_FULL + 1 || i == B_ACC_EMPTY || i == B_ACC_EMPTY + 1 ||
                i == B_DEC_FREE || i == B_DEC_FREE + 1)
                count = NMASK;
            if (i == B_DEC_FULL || i == B_DEC_FULL + 1) count = 32;
            mbar_init(bar(i), count);
        }
        *abort = 0;
        fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------ control ------------------------------
        if (lane == 0) {
            const uint32_t box = static_cast<uint32_t>(Q) * 128;
            auto load_x = [&](int64_t h) {
                mbar_expect_tx(bar(B_X_FULL), box);
                tma_load_4d(sX, &tm_x, bar(B_X_FULL), 0, (int)h, (int)t0, (int)b);
            };
            auto load_h = [&](int64_t h) {
                mbar_expect_tx(bar(B_H_FULL), T::H_BYTES);
                for (int kb = 0; kb < NST / 64; ++kb)
                    tma_load_4d(sH + kb * (PD * 128), &tm_h, bar(B_H_FULL), kb * 64, 0, (int)h,
                                (int)(b * nc + c));
            };
            tma_prefetch_map(&tm_c);
            tma_prefetch_map(&tm_b);
            tma_prefetch_map(&tm_x);
            tma_prefetch_map(&tm_h);
            mbar_expect_tx(bar(B_CB_LOAD), 2 * (NST / 64) * box);
            for (int kb = 0; kb < NST / 64; ++kb) {
                tma_load_4d(sC + kb * T::KB_BYTES, &tm_c, bar(B_CB_LOAD), kb * 64, (int)g,
                            (int)t0, (int)b);
                tma_load_4d(sB + kb * T::KB_BYTES, &tm_b, bar(B_CB_LOAD), kb * 64, (int)g,
                            (int)t0, (int)b);
            }
            SCAN_TRACE(0);
            load_x(hfirst);
            load_h(hfirst);
            bool ok = wait_bar(bar(B_CB_LOAD), 0, abort);
            SCAN_TRACE(1);
            if (ok) {
                fence_after_sync();
                for (int t = 0; t < ntiles; ++t) {
                    const uint32_t id = idesc_bf16(128, 128 * (t + 1), false, false);
                    for (int k = 0; k < NST / 16; ++k) {
                        const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                        mma_bf16(tmem + (t == 0 ? 0u : CB1F),
                                 desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                                 desc_sw128(sB + ko, 16, 1024), id, k > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar(B_CB_DONE));
                ok = wait_bar(bar(B_CB_PACKED), 0, abort);  // CB packed: accumulators free
                SCAN_TRACE(2);
                fence_after_sync();
            }
            for (int i = 0; ok && i < hb_size; ++i) {
                const uint32_t ph = i & 1;
                ok = wait_bar(bar(B_H_FULL), ph, abort);
                SCAN_TRACE(8 + 8 * i);
                for (int t = 0; ok && t < ntiles; ++t) {
                    // state term of tile t, once the epilogue has drained its accumulators
                    if (i > 0) ok = wait_bar(bar(B_ACC_EMPTY + t), (i - 1) & 1, abort);
                    if (!ok) break;
                    fence_after_sync();
                    for (int k = 0; k < NST / 16; ++k) {
                        const uint32_t ko = (k >> 2) * T::KB_BYTES + (k & 3) * 32;
                        const uint32_t kh = (k >> 2) * (PD * 128) + (k & 3) * 32;
                        mma_bf16(tmem + st_col(t), desc_sw128(sC + ko + t * 128 * 128, 16, 1024),
                                 desc_sw128(sH + kh, 16, 1024), idesc_bf16(128, PD, false, false),
                                 k > 0 ? 1u : 0u);
                    }
                    if (t == ntiles - 1) mma_commit(bar(B_H_FREE));
                    SCAN_TRACE(9 + 8 * i + 3 * t);
                    // intra-chunk term of tile t, once its mask (and the head's x) is in
                    ok = wait_bar(bar(B_MK_FULL + t), ph, abort);
                    SCAN_TRACE(10 + 8 * i + 3 * t);
                    if (ok && t == 0) ok = wait_bar(bar(B_X_FULL), ph, abort);
                    if (!ok) break;
                    fence_after_sync();
                    const uint32_t sM = t == 0 ? sM0 : sM1;
                    for (int k = 0; k < 8 * (t + 1); ++k)
                        mma_bf16(tmem + in_col(t),
                                 desc_sw128(sM + (k >> 2) * (128 * 128) + (k & 3) * 32, 16, 1024),
                                 desc_sw128(sX + k * 2048, QMAX * 128, 1024),
                                 idesc_bf16(128, PD, false, true), k > 0 ? 1u : 0u);
                    mma_commit(bar(B_ACC_FULL + t));
                    mma_commit(bar(B_MK_EMPTY + t));
                    SCAN_TRACE(11 + 8 * i + 3 * t);
#ifdef SSD_TRACE
                    if (t == 0 && i < 8) {  // latency of this tile's MMAs and commit
                        wait_bar(bar(B_MK_EMPTY), ph, abort);
                        SCAN_TRACE(176 + i);
                    }
#endif
                }
                if (!ok) break;
                mma_commit(bar(B_X_FREE));
                if (i + 1 < hb_size) {  // refill the state and x buffers for the next head
                    ok = wait_bar(bar(B_H_FREE), ph, abort);
                    if (ok) load_h(hfirst + i + 1);
                    if (ok) ok = wait_bar(bar(B_X_FREE), ph, abort);
                    SCAN_TRACE(15 + 8 * i);
                    if (ok) load_x(hfirst + i + 1);
                }
            }
            if (!ok) *abort = 1;
        }
    } else if (warp == 9) {
        // ------------------------------- loader ------------------------------
        // Stages each head's decays (log2e * cumA, dt) and D into the two
        // shared buffers, so the workers never wait on a global load.
        bool ok = true;
        for (int i = 0; ok && i < hb_size; ++i) {
            const int bsel = i & 1;
            if (i >= 2) ok = wait_bar(bar(B_DEC_FREE + bsel), ((i - 2) >> 1) & 1, abort);
            if (!ok) break;
            float* dec = reinterpret_cast<float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
            const int64_t h = hfirst + i;
            const int64_t vbase = ((b * H + h) * nc + c) * Q;
            float cv[QMAX / 32], dv[QMAX / 32];
#pragma unroll
            for (int k = 0; k < QMAX / 32; ++k) {
                const int j = lane + 32 * k;
                cv[k] = j < Q ? p.cumA[vbase + j] : 0.0f;
                dv[k] = j < Q ? p.dt[vbase + j] : 0.0f;
            }
#pragma unroll
            for (int k = 0; k < QMAX / 32; ++k) {
                dec[lane + 32 * k] = cv[k] * 1.4426950408889634f;
                dec[QMAX + lane + 32 * k] = dv[k];
            }
            if (lane == 0) dec[2 * QMAX] = p.D ? p.D[h] : 0.0f;
            mbar_arrive(bar(B_DEC_FULL + bsel));
        }
        if (!ok) *abort = 1;
    } else {
        // ------------------------------ workers ------------------------------
        const int qd = warp & 3, hf = warp >> 2;
        float* rinv_s = reinterpret_cast<float*>(smem + T::RINV_OFF);
        float* stab = reinterpret_cast<float*>(smem + T::STAB_OFF) + warp * QMAX;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        bool ok = wait_bar(bar(B_CB_DONE), 0, abort);
        if (ok && hf == 0) {
            fence_after_sync();
            // repack CB as fp16 pairs with a per-row power-of-two scale:
            // tile 0 [0,128) -> [0,64), tile 1 [128,384) -> [64,192)
            for (int t = 0; t < ntiles; ++t) {
                const uint32_t src = t == 0 ? 0u : CB1F, dst = t == 0 ? CB0P : CB1P;
                float mx = 0.0f;
                for (int k = 0; k < 4 * (t + 1); ++k) {
                    float v[32];
                    tmem_ld32(tmem + lanes + src + 32 * k, v);
#pragma unroll
                    for (int q = 0; q < 32; ++q) mx = fmaxf(mx, fabsf(v[q]));
                }
                // 2^e with the row's largest |CB| * 2^-e below 2^15
                const int e2 = max(0, ((__float_as_int(mx) >> 23) & 255) - 127 - 14 + 1);
                const float sc = __int_as_float((127 - e2) << 23);
                rinv_s[t * 128 + 32 * qd + lane] = __int_as_float((127 + e2) << 23);
                for (int k = 0; k < 4 * (t + 1); ++k) {
                    float v[32];
                    uint32_t r[16];
                    tmem_ld32(tmem + lanes + src + 32 * k, v);
#pragma unroll
                    for (int q = 0; q < 16; ++q) r[q] = pack_f16x2(v[2 * q] * sc, v[2 * q + 1] * sc);
                    tmem_st16(tmem + lanes + dst + 16 * k, r);
                }
                tmem_wait_st();
            }
            fence_before_sync();
            mbar_arrive(bar(B_CB_PACKED));
            if (warp == 0 && lane == 0) SCAN_TRACE(80);
        }
        if (ok && hf == 1) ok = wait_bar(bar(B_CB_PACKED), 0, abort);
        fence_after_sync();
        const float rinv0 = ok ? rinv_s[32 * qd + lane] : 1.0f;
        const float rinv1 = (ok && ntiles == 2) ? rinv_s[128 + 32 * qd + lane] : 1.0f;

        // The epilogue of head i, tile t, for this warp's rows and 32 p columns.
        // D x came through the mask diagonal and log2e * cumA of the row was kept
        // from the mask phase, so nothing here waits on a global load.
        auto epilogue = [&](int i, int t, float cl2) -> bool {
            const int64_t h = hfirst + i;
            const int l = 128 * t + 32 * qd + lane;
            if (!wait_bar(bar(B_ACC_FULL + t), i & 1, abort)) return false;
            if (warp == 0 && lane == 0) SCAN_TRACE(140 + 4 * i + 2 * t);
            fence_after_sync();
            float vi[32], vs[32];
            tmem_ld32x2(tmem + lanes + in_col(t) + 32 * hf, vi, tmem + lanes + st_col(t) + 32 * hf, vs);
            fence_before_sync();
            mbar_arrive(bar(B_ACC_EMPTY + t));
            if (l < Lc) {
                const float sc = ex2(cl2);
                __nv_bfloat16* yr = static_cast<__nv_bfloat16*>(p.y) +
                                    ((b * L + t0 + l) * H + h) * PD + 32 * hf;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int e = 8 * k4 + 2 * k;
                        o[k] = pack_bf16x2(fmaf(sc, vs[e], vi[e]), fmaf(sc, vs[e + 1], vi[e + 1]));
                    }
                    reinterpret_cast<uint4*>(yr)[k4] = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            if (warp == 0 && lane == 0) SCAN_TRACE(141 + 4 * i + 2 * t);
            return true;
        };

        // Iteration i builds head i's masks and drains head i-1's accumulators,
        // tile by tile, so the tensor core works on one head while the CUDA cores
        // finish the previous one.
        float cl_prev[2] = {0.0f, 0.0f};
        for (int i = 0; i <= hb_size; ++i) {
            const bool mask_now = i < hb_size, epi_now = i > 0;
            const int bsel = i & 1;
            const float* dec = reinterpret_cast<const float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
            float cl_cur[2] = {0.0f, 0.0f};
            float Dh = 0.0f;
            if (mask_now && ok) {
                ok = wait_bar(bar(B_DEC_FULL + bsel), (i >> 1) & 1, abort);
                if (warp == 0 && lane == 0) SCAN_TRACE(82 + 5 * i);
                if (ok) {
                    cl_cur[0] = dec[32 * qd + lane];
                    cl_cur[1] = dec[128 + 32 * qd + lane];
                    Dh = dec[2 * QMAX];
                }
            }
            for (int t = 0; t < ntiles; ++t) {
                if (mask_now && ok) {
                    if (i > 0) ok = wait_bar(bar(B_MK_EMPTY + t), (i - 1) & 1, abort);
                    if (warp == 0 && lane == 0) SCAN_TRACE(83 + 5 * i + 2 * t);
                    if (ok) {
                        if (t == 0)
                            build_mask<0>(tmem, sM0, dec, dec + QMAX, stab, rinv0, Dh, qd, hf, lane);
                        else
                            build_mask<1>(tmem, sM1, dec, dec + QMAX, stab, rinv1, Dh, qd, hf, lane);
                        fence_smem_async();
                        mbar_arrive(bar(B_MK_FULL + t));
                    }
                    if (warp == 0 && lane == 0) SCAN_TRACE(84 + 5 * i + 2 * t);
                }
                if (epi_now && ok) ok = epilogue(i - 1, t, cl_prev[t]);
            }
            if (mask_now && ok) mbar_arrive(bar(B_DEC_FREE + bsel));  // this head's decays are used
            cl_prev[0] = cl_cur[0];
            cl_prev[1] = cl_cur[1];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (*abort && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// Heads per CTA: each CTA pays a fixed set-up (C and B loads, CB, its repack)
// and then pipelines its heads, so with w waves of CTAs over the SMs the
// kernel takes about w * (setup + heads * per_head).  The divisor of the heads
// per group that minimises this, up to 12 heads, is used (or every head of the
// group, when asked).  The two costs are the measured ones (about 5 and 4.5
// us); beyond about a dozen heads per CTA the measured time rises again.
int heads_per_cta(const FwdParams& p, int num_sms) {
    if (p.flags & SSD_FLAG_WHOLE_GROUPS) return static_cast<int>(p.heads_per_group);
    // tuning override: SSD_SCAN_HEADS_PER_CTA=d (used when d divides the heads per group)
    static const int forced = [] {
        const char* e = getenv("SSD_SCAN_HEADS_PER_CTA");
        return e ? atoi(e) : 0;
    }();
    if (forced > 0 && p.heads_per_group % forced == 0) return forced;
    const int64_t units = p.batch * p.nchunks * p.ngroups;
    const double setup = 5.0, per_head = 4.5;
    int best = 1;
    double best_t = 0.0;
    for (int d = 1; d <= p.heads_per_group && d <= 12; ++d) {
        if (p.heads_per_group % d) continue;
        const int64_t ctas = units * (p.heads_per_group / d);
        const int64_t waves = (ctas + num_sms - 1) / num_sms;
        const double t = static_cast<double>(waves) * (setup + per_head * d);
        if (d == 1 || t < best_t) {
            best = d;
            best_t = t;
        }
    }
    return best;
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
    const int hb = heads_per_cta(p, sm_count());
    dim3 grid(static_cast<unsigned>(p.nchunks * p.ngroups * (p.heads_per_group / hb)),
              static_cast<unsigned>(p.batch));
    kern<<<grid, NTHREADS, T::SMEM, s>>>(p, tc_, tb_, tx_, th_, hb);
    return cudaGetLastError();
}

}  // namespace

#ifdef SSD_TRACE
extern "C" int ssd_scan_trace_copy(void* dst) {
    return cudaMemcpyFromSymbol(dst, g_scan_trace, sizeof(g_scan_trace)) == cudaSuccess ? 0 : 1;
}
#endif

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
