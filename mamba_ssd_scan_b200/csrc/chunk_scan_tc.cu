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
//   warps 0-15 "workers": per head and tile, read CB back, apply the causal
//              decay mask (with the diagonal and the D skip folded in) and
//              write Mk as an fp16 operand: tile 0's (K = 128) into TMEM, the A
//              operand of its MMA, tile 1's (K = 256) K-major into shared
//              memory, each refilled as soon as its MMA is done; convert the
//              head's x tile in place to fp16; then drain the previous head's
//              accumulators (y = f * intra + exp(cumA) * state, bf16 staged
//              for the storer).  The four warps of a TMEM lane quarter share
//              its 32 rows and take one column group in four (and a quarter
//              of the p columns in the epilogue);
//   warp 16    "control": one lane issues every TMA load (C, B once; x and
//              H_in per head) and every MMA (CB once; per head and tile the
//              state term C_t H_in^T, bf16, and Mk x, fp16).  H_in comes as
//              the bf16 halves hi + lo of the fp32 state (both resident: 2 x
//              NST / 64 blocks of 8 KB), each against the same C;
//   warp 17    "loader": stages each head's decays and D in shared memory
//              (two buffers), so the mask phase never waits on a global load;
//   warp 18    "storer": the workers stage each head's y tile in shared memory
//              and one lane writes it out with a TMA store, so no worker
//              holds a global store when it next signals an mbarrier.
//
// Balance.  A warp only reaches the TMEM lanes of its quarter (warp % 4),
// which is also the scheduler it issues on, and a causal row's work grows
// with its index.  Tile 0's 32-row blocks are therefore stored in reverse
// order (lane quarter q holds chunk rows 32 (3 - q) ...), so quarter q holds
// row blocks 3 - q and 4 + q: nine column groups per quarter and head.
//
// Decay factors.  For the 32-row block starting at row lb, with a reference
// value M inside the block's cumA range, exp(cumA_l - cumA_j) is split as
// exp(cumA_l - M) * exp(M - cumA_j): the first factor goes to the epilogue
// (one multiply per output element), the second is computed once per column
// by one lane, so each mask element costs one multiply.  M is the midpoint of
// the block's cumA range, so neither factor exceeds 2^(span / 2), span the
// block's log2 decay; blocks whose span exceeds kFastSpan (where such factors
// would leave fp32 range) use M = cumA_lb and one exp2 per diagonal
// element instead, which is exact for any decay.  Every wait is bounded; a
// timed-out role raises a shared abort flag that the others observe, and the
// CTA still frees its TMEM.
//
// TMEM columns: [0,64) tile 0's CB and [128,256) tile 1's CB as packed fp16
// pairs (the fp32 CB sits in [0,128) and [256,512) until packed; the two tiles
// are packed at the same time, so their source and destination columns never
// overlap); [64,128) tile 0's mask (fp16 pairs, written once CB is packed);
// [256,320)/[320,384) tile 0's state/intra accumulators, [384,448)/[448,512)
// tile 1's.
#include <stdlib.h>

#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int QMAX = 256;
constexpr int PD = 64;
constexpr int NWORK = 16;                        // worker warps
constexpr int CTRL_WARP = NWORK, LOAD_WARP = NWORK + 1, STORE_WARP = NWORK + 2;
constexpr int NTHREADS = (NWORK + 3) * 32;
constexpr int NMASK = NWORK * 32;
constexpr uint32_t CB0P = 0, MK0T = 64, CB1P = 128, CB1F = 256;
// largest log2 decay span of a 32-row block that takes the factored path:
// factors stay within 2^90, so masked entries (|CB| scaled below 2^15) and
// their 256-term sums stay far inside fp32 and bf16 range
constexpr float kFastSpan = 180.0f;
constexpr float kMaxExp = 96.0f;
__device__ __forceinline__ uint32_t st_col(int t) { return t == 0 ? 256u : 384u; }
__device__ __forceinline__ uint32_t in_col(int t) { return t == 0 ? 320u : 448u; }
// first chunk row of the 32-row block that TMEM lane quarter qd holds in tile t
__device__ __forceinline__ int block_row(int t, int qd) { return t == 0 ? 32 * (3 - qd) : 128 + 32 * qd; }

template <int NST>
struct ScanTile {
    static constexpr int KB_BYTES = QMAX * 128;              // 64-wide K block of C or B
    static constexpr int C_OFF = 0;
    static constexpr int C_BYTES = (NST / 64) * KB_BYTES;
    static constexpr int B_OFF = C_OFF + C_BYTES;            // B, later tile 1's mask
    static constexpr int MK1_BYTES = 4 * 128 * 128;
    static constexpr int B_BYTES = C_BYTES > MK1_BYTES ? C_BYTES : MK1_BYTES;
    static constexpr int X_OFF = B_OFF + B_BYTES;
    static constexpr int X_BYTES = QMAX * 128;
    // the entering state, in 64-wide K blocks of PD rows (8 KB): the hi
    // blocks, then the lo blocks
    static constexpr int H_OFF = X_OFF + X_BYTES;
    static constexpr int H_SLOT = PD * 128;
    static constexpr int H_BYTES = 2 * (NST / 64) * H_SLOT;
    // per-head decays, two buffers filled by the loader warp:
    // [log2e * cumA (QMAX) | dt (QMAX) | D, max dt, padding (4)] fp32
    static constexpr int DEC_FLOATS = 2 * QMAX + 4;
    static constexpr int DEC_OFF = H_OFF + H_BYTES;
    static constexpr int RINV_OFF = DEC_OFF + 2 * DEC_FLOATS * 4;  // per-row CB scale, 2 tiles
    static constexpr int NORM_OFF = RINV_OFF + 2 * 128 * 4;  // |C_r|^2 per row, max |B_j|^2 partials
    static constexpr int CTAB_OFF = NORM_OFF + (256 + 8) * 4;  // per worker warp: 32 column factors
    static constexpr int XMAX_OFF = CTAB_OFF + NWORK * 32 * 4;  // [2][worker warp]: max |x| bits
    static constexpr int BAR_OFF = XMAX_OFF + 2 * NWORK * 4;
    static constexpr int SMEM = BAR_OFF + 32 * 8 + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Optional timeline of the first CTAs (builds with -DSSD_TRACE only): each role
// stamps the SM cycle counter at its hand-offs into shared memory (a global
// store before an mbarrier arrive would delay the arrive until the store is
// acknowledged); the CTA copies the stamps out when it ends and
// ssd_scan_trace_copy() reads them back.
#ifdef SSD_TRACE
__device__ unsigned long long g_scan_trace[8][256];
#define SCAN_TRACE(slot)                                                              \
    do {                                                                              \
        if ((slot) < 256) s_trace[(slot)] = clock64();                                \
    } while (0)
#else
#define SCAN_TRACE(slot) \
    do {                 \
    } while (0)
#endif

enum : int {
    B_CB_LOAD = 0, B_CB_DONE, B_CB_PACKED, B_X_FULL, B_H_FULL, B_H_FREE, B_X_FREE,
    B_MK_FULL, B_MK_EMPTY = B_MK_FULL + 2, B_ACC_FULL = B_MK_EMPTY + 2,
    B_ACC_EMPTY = B_ACC_FULL + 2, B_DEC_FULL = B_ACC_EMPTY + 2, B_DEC_FREE = B_DEC_FULL + 2,
    B_Y_STAGED = B_DEC_FREE + 2, B_Y_READ, B_MK1A_FULL, B_XCONV, B_COUNT
};

// Bounded wait that also gives up when another role has aborted: a few
// non-blocking probes first (most hand-offs are already complete), then
// probes that may suspend the thread for a short, bounded time, so a waiting
// warp gives its issue slots to the workers sharing its scheduler without the
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

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// 32 fp16 values of one row (16 packed pairs) into the K-major SW128 operand
__device__ __forceinline__ void store_group_packed(uint32_t mbase, uint32_t row, int j0,
                                                   const uint32_t (&o)[16]) {
    const uint32_t dst = mbase + (j0 >> 6) * (128 * 128);
    const int c0 = (j0 & 63) >> 3;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        st_shared_v4(dst + sw128(row, c0 + i), o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

// One packed group of mask values to its operand: tile 0's in TMEM (16
// columns of this warp's lanes at mk_t), tile 1's in shared memory.
__device__ __forceinline__ void put_group(bool to_tmem, uint32_t mk_t, uint32_t mbase, uint32_t row, int j0,
                                          const uint32_t (&o)[16]) {
    if (to_tmem)
        tmem_st16(mk_t, o);
    else
        store_group_packed(mbase, row, j0, o);
}

// Mask warp for tile TT: rows block_row(TT, qd) + lane (TMEM lane 32 qd + lane),
// column groups hf + 4 k (k <= TT) of 32 columns.  Groups above the diagonal
// block are zeros; they are written for the first head only (nothing else
// writes there).  cum2 holds log2(e) * cumA, so every decay is one exp2.
//
// The operand is fp16 (2^-11 relative rounding, against bf16's 2^-8), so each
// row carries a power-of-two scale rs_l into fp16's range: row l holds
// m[l,j] = CBp[l,j] k_j rs_l for j < l, CBp the packed CB (CB = rinv_l CBp,
// |CBp| < 2^14) and k_j = 2^{ref - c_j} dt_j (fast) or 2^{c_l - c_j} dt_j
// (steep), and on the diagonal m[l,l] = (CBp[l,l] dt_l + D / rinv_l) e_l rs_l
// with e_l = 2^{ref - c_l} (fast) or 1 (steep), so that the epilogue factor
// f_l = rinv_l / (e_l rs_l) gives the diagonal term (C_l . B_l dt_l + D) x_l
// and the D skip with the rest of the row.  For j <= l, c_j >= c_l, so
// |m[l,j]| <= (2^14 dmax + |D| / rinv_l) e_l rs_l, dmax the chunk's largest
// dt; rs_l brings that bound to 2^15, below fp16's 65504, so nothing
// overflows and the row's largest entries keep every bit.
struct RowPlan {
    float ref, cl, c_first;
    float f;         // the row's epilogue factor
    float rs;        // the row's power-of-two scale into fp16 range
    float dtl;       // dt_l
    float dadd;      // D / rinv_l * rs_l: the skip term in the mask's units
    float de;        // e_l: the diagonal's decay factor
    bool fast;       // factored decays (warp-uniform)
    int rb;          // 32-row block index of the rows
    uint32_t row;    // TMEM lane = Mk row
    uint32_t cbase;  // TMEM address of the rows' packed CB
};

template <int TT>
__device__ __forceinline__ RowPlan plan_rows(uint32_t tmem, const float* cum2, const float* dtv,
                                             float rinv, float Dh, float dmax, int qd, int lane, int Lc) {
    RowPlan r;
    const int lb = block_row(TT, qd);
    r.rb = lb >> 5;
    r.row = 32 * qd + lane;
    r.cbase = tmem + (static_cast<uint32_t>(32 * qd) << 16) + (TT == 0 ? CB0P : CB1P);
    // the block's log2 decay span picks the path
    const int last = max(lb, min(lb + 31, Lc - 1));
    r.c_first = cum2[lb];
    const float c_last = cum2[last];
    r.fast = (r.c_first - c_last) <= kFastSpan;
    r.ref = r.fast ? 0.5f * (r.c_first + c_last) : r.c_first;
    r.cl = cum2[lb + lane];
    const float irinv = __int_as_float(254 * (1 << 23) - __float_as_int(rinv));  // 1 / rinv (a power of 2)
    const float lg = (r.fast ? r.ref - r.cl : 0.0f) +
                     __log2f(fmaxf(16384.0f * dmax + fabsf(Dh) * irinv, 1e-30f));
    const int e = min(120, max(-120, 15 - static_cast<int>(ceilf(fminf(fmaxf(lg, -200.0f), 200.0f)))));
    r.rs = __int_as_float((127 + e) << 23);
    const float irs = __int_as_float((127 - e) << 23);
    r.f = (r.fast ? rinv * ex2(r.cl - r.ref) : rinv) * irs;
    r.dtl = dtv[lb + lane];
    r.dadd = Dh * irinv * r.rs;
    r.de = r.fast ? ex2(r.ref - r.cl) : 1.0f;
    return r;
}

// One 32-column group g of the plan's rows, to TMEM (mk_t: the group's 16
// columns at this warp's lanes) or to the shared operand at mbase.
__device__ __forceinline__ void mask_group(const RowPlan& r, int g, bool to_tmem, uint32_t mk_t, uint32_t mbase,
                                           const float* cum2, const float* dtv, float* ctab, int lane,
                                           bool first) {
    const int j0 = 32 * g;
    if (g > r.rb) {  // above the diagonal block: zeros, kept from the first head
        if (first) {
            const uint32_t z[16] = {};
            put_group(to_tmem, mk_t, mbase, r.row, j0, z);
        }
        return;
    }
    uint32_t raw[16];
    tmem_ld16(r.cbase + 16 * g, raw);
    // this lane's column factor, shared with the warp through its table
    const float cj = ex2(fminf(r.ref - cum2[j0 + lane], kMaxExp)) * dtv[j0 + lane];
    __syncwarp();
    ctab[lane] = cj;
    __syncwarp();
    const float4* ct = reinterpret_cast<const float4*>(ctab);
    const float2 rs2 = make_float2(r.rs, r.rs);
    if (g < r.rb && r.fast) {  // below the diagonal block: packed fp32x2 products
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c = ct[i];
            const float2 a0 = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&raw[2 * i])), rs2);
            const float2 a1 = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&raw[2 * i + 1])), rs2);
            const float2 m0 = __fmul2_rn(a0, make_float2(c.x, c.y));
            const float2 m1 = __fmul2_rn(a1, make_float2(c.z, c.w));
            o[2 * i] = pack_f16x2(m0.x, m0.y);
            o[2 * i + 1] = pack_f16x2(m1.x, m1.y);
        }
        put_group(to_tmem, mk_t, mbase, r.row, j0, o);
        return;
    }
    float v[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 f = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&raw[i])), rs2);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
    if (g < r.rb) {  // below the diagonal block, steep row block
        const float rr = ex2(r.cl - r.c_first);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c = ct[i];
            v[4 * i + 0] *= rr * c.x;
            v[4 * i + 1] *= rr * c.y;
            v[4 * i + 2] *= rr * c.z;
            v[4 * i + 3] *= rr * c.w;
        }
    } else if (r.fast) {  // the diagonal block, factored; j = l carries dt_l and D
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c = ct[i];
            const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int q = 4 * i + e;
                float m = v[q] * cc[e];
                if (q == lane) m = fmaf(v[q], r.dtl, r.dadd) * r.de;
                v[q] = (q <= lane) ? m : 0.0f;
            }
        }
    } else {  // the diagonal block of a steep block: one exp2 per element
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            float m = v[q] * ex2(fminf(r.cl - cum2[j0 + q], 0.0f)) * dtv[j0 + q];
            if (q == lane) m = fmaf(v[q], r.dtl, r.dadd) * r.de;
            v[q] = (q <= lane) ? m : 0.0f;
        }
    }
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = pack_f16x2(v[2 * i], v[2 * i + 1]);
    put_group(to_tmem, mk_t, mbase, r.row, j0, o);
}

// Per-head MMAs, issued by the control thread.  Descriptors are built once;
// each K step only advances their start-address field (address / 16).
// State term of one tile, one 64-wide K block: C_t's K block ka (K-major) x
// the state block in slot hs (K-major); ACC: add to the accumulator.
__device__ __forceinline__ void issue_state_kb(uint32_t d_tmem, uint64_t dA, uint64_t dB, int ka,
                                               int hs, bool acc) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t oa = (ka * (QMAX * 128) + k * 32) >> 4;
        const uint32_t ob = (hs * (PD * 128) + k * 32) >> 4;
        mma_bf16(d_tmem, dA + oa, dB + ob, idesc_bf16(128, PD, false, false), (acc || k > 0) ? 1u : 0u);
    }
}
// The whole state term of one tile: every hi block, then (when the state
// comes as a hi / lo pair) every lo block against the same C blocks.
template <int NST>
__device__ __forceinline__ void issue_state(uint32_t d_tmem, uint64_t dA, uint64_t dB, bool hl) {
#pragma unroll
    for (int kb = 0; kb < NST / 64; ++kb) issue_state_kb(d_tmem, dA, dB, kb, kb, kb > 0);
    if (hl)
#pragma unroll
        for (int kb = 0; kb < NST / 64; ++kb) issue_state_kb(d_tmem, dA, dB, kb, NST / 64 + kb, true);
}
// Intra-chunk term of tile 0: its mask in TMEM (128 lanes x 64 columns of fp16
// pairs) x x (MN-major), K = 128 in steps of 16 (8 columns of A each).
__device__ __forceinline__ void issue_intra_t0(uint32_t d_tmem, uint32_t a_tmem, uint64_t dB) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
        mma_ts(d_tmem, a_tmem + 8 * k, dB + ((k * 2048) >> 4), idesc_f16(128, PD, false, true),
               k > 0 ? 1u : 0u);
}
// Intra-chunk term of tile 1: Mk_1 (K-major) x x (MN-major), both fp16, K
// steps [K0, K1) of 16; FRESH: the first of them overwrites the accumulator.
template <int K0, int K1, bool FRESH>
__device__ __forceinline__ void issue_intra(uint32_t d_tmem, uint64_t dA, uint64_t dB) {
#pragma unroll
    for (int k = K0; k < K1; ++k) {
        const uint32_t ka = ((k >> 2) * (128 * 128) + (k & 3) * 32) >> 4;
        const uint32_t kb = (k * 2048) >> 4;
        mma_bf16(d_tmem, dA + ka, dB + kb, idesc_f16(128, PD, false, true),
                 (FRESH && k == K0) ? 0u : 1u);
    }
}

template <int NST, bool GATED>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_scan_tc_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_c,
                         const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_h,
                         const __grid_constant__ CUtensorMap tm_y,
                         const __grid_constant__ CUtensorMap tm_z, int hb_size, int64_t withhold) {
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
    constexpr bool gated = GATED;  // y *= silu(z): a separate instantiation
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sM1 = sB;
    const uint32_t sX = smem_u32(smem + T::X_OFF), sH = smem_u32(smem + T::H_OFF);
    // hi / lo state operand (else the bf16 states alone)
    const bool hl = p.states_hl != nullptr;
    // y of one head is staged in tile 1's mask buffer, in its K columns
    // 0-127 (rewritten for every head, never a zero group), between the MMA
    // that read that buffer and the next mask, and leaves by TMA
    const uint32_t sY = sM1;

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t count = 1;
            if (i == B_CB_PACKED) count = NMASK;
            if (i == B_MK_FULL || i == B_MK_FULL + 1 || i == B_ACC_EMPTY || i == B_ACC_EMPTY + 1 ||
                i == B_DEC_FREE || i == B_DEC_FREE + 1 || i == B_Y_STAGED || i == B_MK1A_FULL ||
                i == B_XCONV)
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
#ifdef SSD_TRACE
    __shared__ unsigned long long s_trace[256];
    for (int k = tid; k < 256; k += NTHREADS) s_trace[k] = 0;
    __syncthreads();
#endif

    if (warp == CTRL_WARP) {
        // ------------------------------ control ------------------------------
        if (lane == 0) {
            const uint32_t box = static_cast<uint32_t>(Q) * 128;
            auto load_x = [&](int64_t h) {
                mbar_expect_tx(bar(B_X_FULL), box);
                tma_load_4d(sX, &tm_x, bar(B_X_FULL), 0, (int)h, (int)t0, (int)b);
            };
            // rows of the state map: hi blocks at b * nc + c, lo blocks
            // batch * nc further on
            const int hi_row = (int)(b * nc + c), lo_row = (int)(p.batch * nc + b * nc + c);
            auto load_h = [&](int64_t h) {
                mbar_expect_tx(bar(B_H_FULL), (hl ? 2 : 1) * (NST / 64) * T::H_SLOT);
                for (int kb = 0; kb < NST / 64; ++kb) {
                    tma_load_4d(sH + kb * T::H_SLOT, &tm_h, bar(B_H_FULL), kb * 64, 0, (int)h, hi_row);
                    if (hl)
                        tma_load_4d(sH + (NST / 64 + kb) * T::H_SLOT, &tm_h, bar(B_H_FULL), kb * 64, 0,
                                    (int)h, lo_row);
                }
            };
            auto prefetch_head = [&](int64_t h) {
                tma_prefetch_l2_4d(&tm_x, 0, (int)h, (int)t0, (int)b);
                if (gated) tma_prefetch_l2_4d(&tm_z, 0, (int)h, (int)t0, (int)b);
                for (int kb = 0; kb < NST / 64; ++kb) {
                    tma_prefetch_l2_4d(&tm_h, kb * 64, 0, (int)h, hi_row);
                    if (hl) tma_prefetch_l2_4d(&tm_h, kb * 64, 0, (int)h, lo_row);
                }
            };
            tma_prefetch_map(&tm_c);
            tma_prefetch_map(&tm_b);
            tma_prefetch_map(&tm_x);
            tma_prefetch_map(&tm_h);
            // C in 32-row blocks, each stored where its TMEM lane quarter
            // expects it (tile 0's blocks reversed); B in chunk order
            mbar_expect_tx(bar(B_CB_LOAD), (NST / 64) * (ntiles * 128 * 128 + box));
            for (int kb = 0; kb < NST / 64; ++kb) {
                for (int t = 0; t < ntiles; ++t)
                    for (int q = 0; q < 4; ++q)
                        tma_load_4d(sC + kb * T::KB_BYTES + (128 * t + 32 * q) * 128, &tm_c,
                                    bar(B_CB_LOAD), kb * 64, (int)g, (int)(t0 + block_row(t, q)),
                                    (int)b);
                tma_load_4d(sB + kb * T::KB_BYTES, &tm_b, bar(B_CB_LOAD), kb * 64, (int)g,
                            (int)t0, (int)b);
            }
            SCAN_TRACE(0);
            if (gated) tma_prefetch_l2_4d(&tm_z, 0, (int)hfirst, (int)t0, (int)b);
            load_x(hfirst);
            // C, B and x are inputs; the carried states come from step 3
            grid_dep_wait();
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
            const uint64_t dC0 = desc_sw128(sC, 16, 1024), dC1 = desc_sw128(sC + 128 * 128, 16, 1024);
            const uint64_t dH = desc_sw128(sH, 16, 1024), dX = desc_sw128(sX, QMAX * 128, 1024);
            const uint64_t dM1 = desc_sw128(sM1, 16, 1024);
            for (int i = 0; ok && i < hb_size; ++i) {
                const uint32_t ph = i & 1;
                if (i + 1 < hb_size) prefetch_head(hfirst + i + 1);  // next head's x, H_in into L2
                ok = wait_bar(bar(B_H_FULL), ph, abort);
                SCAN_TRACE(8 + 8 * i);
                for (int t = 0; ok && t < ntiles; ++t) {
                    // state term of tile t, once the epilogue has drained its accumulators
                    if (i > 0) ok = wait_bar(bar(B_ACC_EMPTY + t), (i - 1) & 1, abort);
                    if (!ok) break;
                    fence_after_sync();
                    issue_state<NST>(tmem + st_col(t), t == 0 ? dC0 : dC1, dH, hl);
                    if (t == ntiles - 1) mma_commit(bar(B_H_FREE));
                    SCAN_TRACE(9 + 8 * i + 3 * t);
                    // intra-chunk term of tile t, once its mask (and the head's x) is in
                    ok = wait_bar(bar(B_MK_FULL + t), ph, abort);
                    SCAN_TRACE(10 + 8 * i + 3 * t);
                    if (ok && t == 0) ok = wait_bar(bar(B_XCONV), ph, abort);  // x in fp16
                    if (t == 0) SCAN_TRACE(192 + i);
                    if (!ok) break;
                    fence_after_sync();
                    if (t == 0) {
                        issue_intra_t0(tmem + in_col(0), tmem + MK0T, dX);
                    } else {
                        // tile 1's mask arrives in two halves: K columns
                        // 128-255 first, then 0-127
                        issue_intra<8, 16, true>(tmem + in_col(1), dM1, dX);
                        ok = wait_bar(bar(B_MK1A_FULL), ph, abort);
                        if (!ok) break;
                        fence_after_sync();
                        issue_intra<0, 8, false>(tmem + in_col(1), dM1, dX);
                    }
                    mma_commit(bar(B_ACC_FULL + t));
                    mma_commit(bar(B_MK_EMPTY + t));
                    SCAN_TRACE(11 + 8 * i + 3 * t);
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
    } else if (warp == LOAD_WARP) {
        // ------------------------------- loader ------------------------------
        // Stages each head's decays (log2e * cumA, dt) and D into the two
        // shared buffers.  Slots past the chunk's last token get that token's
        // cumA and dt = 0, so every factor formed from them is finite.
        bool ok = true;
        grid_dep_wait();  // dt and cumA come from steps 1-2
        for (int i = 0; ok && i < hb_size; ++i) {
            const int bsel = i & 1;
            if (i >= 2) ok = wait_bar(bar(B_DEC_FREE + bsel), ((i - 2) >> 1) & 1, abort);
            if (!ok) break;
            float* dec = reinterpret_cast<float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
            const int64_t h = hfirst + i;
            const int64_t vbase = ((b * H + h) * nc + c) * Q;
            const float c_end = p.cumA[vbase + Lc - 1];
            float cv[QMAX / 32], dv[QMAX / 32];
#pragma unroll
            for (int k = 0; k < QMAX / 32; ++k) {
                const int j = lane + 32 * k;
                cv[k] = j < Lc ? p.cumA[vbase + j] : c_end;
                dv[k] = j < Lc ? p.dt[vbase + j] : 0.0f;
            }
#pragma unroll
            for (int k = 0; k < QMAX / 32; ++k) {
                dec[lane + 32 * k] = cv[k] * 1.4426950408889634f;
                dec[QMAX + lane + 32 * k] = dv[k];
            }
            // the chunk's largest dt, for the masks' fp16 row scales
            float dm = 0.0f;
#pragma unroll
            for (int k = 0; k < QMAX / 32; ++k) dm = fmaxf(dm, dv[k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dm = fmaxf(dm, __shfl_xor_sync(0xffffffffu, dm, o));
            if (lane == 0) {
                dec[2 * QMAX] = p.D ? p.D[h] : 0.0f;
                dec[2 * QMAX + 1] = dm;
            }
            // the test hook: the first head of chunk `withhold` never gets its
            // decays, so the workers' bounded waits run out
            if (i > 0 || c != withhold) mbar_arrive(bar(B_DEC_FULL + bsel));
        }
        if (!ok) *abort = 1;
    } else if (warp == STORE_WARP) {
        // ------------------------------- storer ------------------------------
        // Each head's staged y tile goes out as one TMA store; the workers
        // may overwrite the staging buffer once the store has read it.
        if (lane == 0) {
            tma_prefetch_map(&tm_y);
            for (int k = 0; k < hb_size; ++k) {
                if (!wait_bar(bar(B_Y_STAGED), k & 1, abort)) break;
                tma_store_4d(&tm_y, sY, 0, (int)(hfirst + k), (int)t0, (int)b);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(bar(B_Y_READ));
            }
            bulk_wait_all();
        }
    } else {
        // ------------------------------ workers ------------------------------
        const int qd = warp & 3, hf = warp >> 2;
        float* rinv_s = reinterpret_cast<float*>(smem + T::RINV_OFF);
        float* ctab = reinterpret_cast<float*>(smem + T::CTAB_OFF) + warp * 32;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        // CB is repacked as fp16 pairs with a power-of-two scale per row,
        // chosen from |C_l . B_j| <= |C_l| max_j |B_j| (norms of the C and B
        // rows in shared memory, taken while the CB MMA runs) so that the
        // packed row stays below 2^15.  All sixteen workers repack in one pass:
        // tile 1's fp32 [256,512) -> [128,256); tile 0's [0,128) -> [0,64) in
        // place, loaded by every warp before any warp stores.
        float* cn_s = reinterpret_cast<float*>(smem + T::NORM_OFF);
        float* bn_s = cn_s + 256;
        bool ok = wait_bar(bar(B_CB_LOAD), 0, abort);
        if (ok) {
            const int r = 32 * (warp & 7) + lane;           // warps 0-7: C rows, 8-15: B rows
            const bool is_c = warp < 8;
            const bool valid = is_c ? r < 128 * ntiles : r < Q;
            const uint32_t base = (is_c ? sC : sB) + r * 128;
            float ss = 0.0f;
            if (valid) {
#pragma unroll
                for (int kb = 0; kb < NST / 64; ++kb)
#pragma unroll
                    for (int c16 = 0; c16 < 8; ++c16) {  // the row's 128 bytes, rotated by lane
                        const uint4 v = ld_shared_v4(base + kb * T::KB_BYTES + ((c16 + lane) & 7) * 16);
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                        }
                    }
            }
            if (is_c) {
                cn_s[r] = ss;
            } else {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss = fmaxf(ss, __shfl_xor_sync(0xffffffffu, ss, o));
                if (lane == 0) bn_s[warp - 8] = ss;
            }
        }
        named_sync(1, NMASK);
        float sc_t[2] = {1.0f, 1.0f};
        if (ok) {
            float bmax = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) bmax = fmaxf(bmax, bn_s[k]);
            for (int t = 0; t < ntiles; ++t) {
                const int rr = 128 * t + 32 * qd + lane;    // TMEM lane = C row in shared memory
                const float bound = sqrtf(cn_s[rr] * bmax);
                // 2^e with bound * 2^-e below 2^14 (fp16 holds up to 65504)
                const int e2 = max(0, ((__float_as_int(bound) >> 23) & 255) - 127 - 13 + 1);
                sc_t[t] = __int_as_float((127 - e2) << 23);
                if (hf == 0) rinv_s[rr] = __int_as_float((127 + e2) << 23);
            }
        }
        if (ok) ok = wait_bar(bar(B_CB_DONE), 0, abort);
        uint32_t r0[16];
        if (ok) {
            fence_after_sync();
            if (ntiles == 2) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int kk = hf + 4 * k;
                    float v[32];
                    uint32_t r1[16];
                    tmem_ld32(tmem + lanes + CB1F + 32 * kk, v);
#pragma unroll
                    for (int q = 0; q < 16; ++q) r1[q] = pack_f16x2(v[2 * q] * sc_t[1], v[2 * q + 1] * sc_t[1]);
                    tmem_st16(tmem + lanes + CB1P + 16 * kk, r1);
                }
            }
            float v[32];
            tmem_ld32(tmem + lanes + 32 * hf, v);
#pragma unroll
            for (int q = 0; q < 16; ++q) r0[q] = pack_f16x2(v[2 * q] * sc_t[0], v[2 * q + 1] * sc_t[0]);
        }
        fence_before_sync();
        named_sync(2, NMASK);  // every warp has read its part of tile 0's fp32 CB
        fence_after_sync();
        if (ok) {
            tmem_st16(tmem + lanes + CB0P + 16 * hf, r0);
            tmem_wait_st();
        }
        fence_before_sync();
        mbar_arrive(bar(B_CB_PACKED));
        if (warp == 0 && lane == 0) SCAN_TRACE(80);
        if (ok) ok = wait_bar(bar(B_CB_PACKED), 0, abort);
        fence_after_sync();
        const float rinv0 = ok ? rinv_s[32 * qd + lane] : 1.0f;
        const float rinv1 = (ok && ntiles == 2) ? rinv_s[128 + 32 * qd + lane] : 1.0f;

        // The epilogue of head i, tile t, for this warp's rows and 16 p
        // columns: y = f * intra + 2^cl * state (the intra term carries the
        // diagonal and the D skip), so the worker loop never waits on a global
        // load.
        auto epilogue = [&](int i, int t, float cl2, float fr) -> bool {
            const int l = block_row(t, qd) + lane;
            if (!wait_bar(bar(B_ACC_FULL + t), i & 1, abort)) return false;
            if (warp == 0 && lane == 0) SCAN_TRACE(140 + 4 * i + 2 * t);
            fence_after_sync();
            const uint32_t a[2] = {tmem + lanes + in_col(t) + 16 * hf, tmem + lanes + st_col(t) + 16 * hf};
            uint32_t r[2][16];
            tmem_ld16x2(a, r);
            fence_before_sync();
            mbar_arrive(bar(B_ACC_EMPTY + t));
            if (l < Lc) {
                // optional output gate: y *= silu(z), z read after the
                // accumulators are released (no load is in flight at an arrive)
                uint32_t zw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if constexpr (gated) {
                    const uint4* zr = reinterpret_cast<const uint4*>(
                        static_cast<const __nv_bfloat16*>(p.z) + ((b * L + t0 + l) * H + hfirst + i) * PD +
                        16 * hf);
                    const uint4 z0 = ldg16(zr), z1 = ldg16(zr + 1);
                    zw[0] = z0.x; zw[1] = z0.y; zw[2] = z0.z; zw[3] = z0.w;
                    zw[4] = z1.x; zw[5] = z1.y; zw[6] = z1.z; zw[7] = z1.w;
                }
                const float s = ex2(cl2);
                const float2 f2 = make_float2(fr, fr), s2 = make_float2(s, s);
#pragma unroll
                for (int k4 = 0; k4 < 2; ++k4) {
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int e = 8 * k4 + 2 * k;
                        const float2 vi = make_float2(__uint_as_float(r[0][e]), __uint_as_float(r[0][e + 1]));
                        const float2 vs = make_float2(__uint_as_float(r[1][e]), __uint_as_float(r[1][e + 1]));
                        float2 yv = __ffma2_rn(s2, vs, __fmul2_rn(f2, vi));
                        if constexpr (gated) {
                            const float2 zf =
                                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[4 * k4 + k]));
                            yv.x *= silu_f32(zf.x);
                            yv.y *= silu_f32(zf.y);
                        }
                        o[k] = pack_bf16x2(yv.x, yv.y);
                    }
                    st_shared_v4(sY + sw128(l, 2 * hf + k4), o[0], o[1], o[2], o[3]);
                }
            }
            if (warp == 0 && lane == 0) SCAN_TRACE(141 + 4 * i + 2 * t);
            return true;
        };

        // This warp's x entries of the resident x tile (its rows, 16 p
        // columns), in place as the fp16 operand of the intra MMAs: x 2^es
        // with one power of two per head that takes the tile's largest |x| to
        // [2^13, 2^14) (bf16 values are exact in fp16 there; only entries
        // below 2^-27 of that largest lose bits).  Returns 2^-es.  x is
        // overwritten by the next head once the last tile's MMA is done, which
        // waits for this warp's mask.
        // Every worker reaches the named barrier once per head (with `live`
        // false it only takes part in it), so a warp whose wait failed cannot
        // leave the others waiting there.  The partial maxima alternate
        // between two buffers by head, so a warp that runs ahead cannot
        // overwrite one that another warp has still to read.
        auto convert_x = [&](bool live, int par) -> float {
            uint32_t* xmax_s = reinterpret_cast<uint32_t*>(smem + T::XMAX_OFF) + par * NWORK;
            uint32_t w[2][8] = {};
            uint32_t m2 = 0u;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (live && t < ntiles) {
                    const int l = block_row(t, qd) + lane;
                    const uint4 v0 = ld_shared_v4(sX + sw128(l, 2 * hf));
                    const uint4 v1 = ld_shared_v4(sX + sw128(l, 2 * hf + 1));
                    w[t][0] = v0.x; w[t][1] = v0.y; w[t][2] = v0.z; w[t][3] = v0.w;
                    w[t][4] = v1.x; w[t][5] = v1.y; w[t][6] = v1.z; w[t][7] = v1.w;
                    // max |x| as bf16 bit patterns (sign cleared; non-negative
                    // floats order as their bits), both halves at once
#pragma unroll
                    for (int k = 0; k < 8; ++k) m2 = __vmaxu2(m2, w[t][k] & 0x7FFF7FFFu);
                }
            }
            uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (lane == 0) xmax_s[warp] = am;
            named_sync(3, NMASK);
#pragma unroll
            for (int k = 0; k < NWORK; ++k) am = max(am, xmax_s[k]);
            // bf16 bits -> exponent (the inputs are finite)
            const int ex = am ? static_cast<int>((am >> 7) & 255) - 127 : 0;
            const int es = min(100, max(-100, 13 - ex));
            const float sc = __int_as_float((127 + es) << 23);
            const float2 sc2 = make_float2(sc, sc);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!live || t >= ntiles) continue;
                const int l = block_row(t, qd) + lane;
                uint32_t o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float2 f = __fmul2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t][k])), sc2);
                    o[k] = pack_f16x2(f.x, f.y);
                }
                st_shared_v4(sX + sw128(l, 2 * hf), o[0], o[1], o[2], o[3]);
                st_shared_v4(sX + sw128(l, 2 * hf + 1), o[4], o[5], o[6], o[7]);
            }
            return __int_as_float((127 - es) << 23);
        };

        // Iteration i builds head i's tile-0 mask (in TMEM), drains head i-1's
        // accumulators, converts head i's x tile and builds its tile-1 mask, so
        // the tensor core works on one head while the CUDA cores finish the
        // previous one.
        const uint32_t mk0 = tmem + lanes + MK0T + 16 * hf;  // this warp's tile-0 mask columns
        float cl_prev[2] = {0.0f, 0.0f};
        float f_prev[2] = {1.0f, 1.0f};
        for (int i = 0; i <= hb_size; ++i) {
            const bool mask_now = i < hb_size, epi_now = i > 0;
            const int bsel = i & 1;
            const float* dec = reinterpret_cast<const float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
            float cl_cur[2] = {0.0f, 0.0f};
            float f_cur[2] = {1.0f, 1.0f};
            float Dh = 0.0f, dmax = 0.0f;
            if (mask_now && ok) {
                ok = wait_bar(bar(B_DEC_FULL + bsel), (i >> 1) & 1, abort);
                if (warp == 0 && lane == 0) SCAN_TRACE(82 + 5 * i);
                if (ok) {
                    cl_cur[0] = dec[block_row(0, qd) + lane];
                    cl_cur[1] = dec[block_row(1, qd) + lane];
                    Dh = dec[2 * QMAX];
                    dmax = dec[2 * QMAX + 1];
                }
            }
            if (mask_now && ok) {
                if (i > 0) ok = wait_bar(bar(B_MK_EMPTY), (i - 1) & 1, abort);
                if (warp == 0 && lane == 0) SCAN_TRACE(83 + 5 * i);
                if (ok) {
                    const RowPlan r0 = plan_rows<0>(tmem, dec, dec + QMAX, rinv0, Dh, dmax, qd, lane, Lc);
                    mask_group(r0, hf, true, mk0, 0u, dec, dec + QMAX, ctab, lane, i == 0);
                    f_cur[0] = r0.f;
                    tmem_wait_st();
                    fence_before_sync();
                    mbar_arrive(bar(B_MK_FULL));
                }
                if (warp == 0 && lane == 0) SCAN_TRACE(84 + 5 * i);
            }
            if (epi_now && ok) {
                // the staging buffer is free once tile 1's MMA of head i-1 is
                // done with it and the store of head i-2 has read it
                if (ntiles == 2) ok = wait_bar(bar(B_MK_EMPTY + 1), (i - 1) & 1, abort);
                else if (i >= 2) ok = wait_bar(bar(B_Y_READ), (i - 2) & 1, abort);
                for (int t = 0; t < ntiles; ++t)
                    if (ok) ok = epilogue(i - 1, t, cl_prev[t], f_prev[t]);
                if (ok) {
                    fence_smem_async();
                    mbar_arrive(bar(B_Y_STAGED));
                }
            }
            RowPlan r1;
            if (mask_now && ok && ntiles == 2) {
                // tile 1, K columns 128-255 (clear of the y staging area)
                r1 = plan_rows<1>(tmem, dec, dec + QMAX, rinv1, Dh, dmax, qd, lane, Lc);
                mask_group(r1, hf + 4, false, 0u, sM1, dec, dec + QMAX, ctab, lane, i == 0);
                f_cur[1] = r1.f;
                fence_smem_async();
                mbar_arrive(bar(B_MK_FULL + 1));
                if (warp == 0 && lane == 0 && i < 16) SCAN_TRACE(240 + i);
            }
            if (mask_now) {
                if (ok) ok = wait_bar(bar(B_X_FULL), i & 1, abort);
                if (warp == 0 && lane == 0) SCAN_TRACE(200 + 2 * i);
                const float ix = convert_x(ok, i & 1);
                if (ok) {
                    f_cur[0] *= ix;
                    f_cur[1] *= ix;
                    fence_smem_async();
                    mbar_arrive(bar(B_XCONV));
                }
                if (warp == 0 && lane == 0) SCAN_TRACE(201 + 2 * i);
            }
            if (mask_now && ok && ntiles == 2) {
                // tile 1, K columns 0-127, once the staged y has been stored
                if (i > 0) ok = wait_bar(bar(B_Y_READ), (i - 1) & 1, abort);
                if (warp == 0 && lane == 0) SCAN_TRACE(85 + 5 * i);
                if (ok) {
                    mask_group(r1, hf, false, 0u, sM1, dec, dec + QMAX, ctab, lane, i == 0);
                    fence_smem_async();
                    mbar_arrive(bar(B_MK1A_FULL));
                }
                if (warp == 0 && lane == 0) SCAN_TRACE(86 + 5 * i);
            }
            if (mask_now && ok) mbar_arrive(bar(B_DEC_FREE + bsel));  // this head's decays are used
            cl_prev[0] = cl_cur[0];
            cl_prev[1] = cl_cur[1];
            f_prev[0] = f_cur[0];
            f_prev[1] = f_cur[1];
        }
    }
    fence_before_sync();
    __syncthreads();
#ifdef SSD_TRACE
    if (blockIdx.x < 8 && blockIdx.y == 0)
        for (int k = tid; k < 256; k += NTHREADS) g_scan_trace[blockIdx.x][k] = s_trace[k];
#endif
    if (*abort && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// Heads per CTA: each CTA pays a fixed set-up (C and B loads, CB, its repack)
// and then pipelines its heads, so with w waves of CTAs over the SMs the
// kernel takes about w * (setup + heads * per_head).  The divisor of the heads
// per group that minimises this, up to 32 heads, is used (or every head of the
// group, when asked).  The two costs are the measured ones (in microseconds;
// the set-up includes filling and draining the head pipeline).
int heads_per_cta(const FwdParams& p, int num_sms) {
    if (p.flags & SSD_FLAG_WHOLE_GROUPS) return static_cast<int>(p.heads_per_group);
    // tuning override: SSD_SCAN_HEADS_PER_CTA=d (used when d divides the heads per group)
    static const int forced = [] {
        const char* e = getenv("SSD_SCAN_HEADS_PER_CTA");
        return e ? atoi(e) : 0;
    }();
    if (forced > 0 && p.heads_per_group % forced == 0) return forced;
    const int64_t units = p.batch * p.nchunks * p.ngroups;
    const double setup = 9.0, per_head = 4.0;
    int best = 1;
    double best_t = 0.0;
    for (int d = 1; d <= p.heads_per_group && d <= 32; ++d) {
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
    CUtensorMap tc_, tb_, tx_, th_, ty_, tz_;
    const uint32_t rows = static_cast<uint32_t>(p.chunk);
    if (!make_tmap_bf16_4d(&tc_, p.C, NST, p.ngroups, p.seqlen, p.batch, 1, 32) ||
        !make_tmap_bf16_4d(&tb_, p.B, NST, p.ngroups, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&tx_, p.x, PD, p.nheads, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&th_, p.states_hl ? p.states_hl : p.states, NST, PD, p.nheads,
                           (p.states_hl ? 2 : 1) * p.batch * p.nchunks, PD, 1) ||
        !make_tmap_bf16_4d(&ty_, p.y, PD, p.nheads, p.seqlen, p.batch, 1, rows) ||
        !make_tmap_bf16_4d(&tz_, p.z ? p.z : p.x, PD, p.nheads, p.seqlen, p.batch, 1, rows))
        return cudaErrorInvalidValue;
    auto kern = p.z ? chunk_scan_tc_kernel<NST, true> : chunk_scan_tc_kernel<NST, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    const int hb = heads_per_cta(p, sm_count());
    dim3 grid(static_cast<unsigned>(p.nchunks * p.ngroups * (p.heads_per_group / hb)),
              static_cast<unsigned>(p.batch));
    return launch_kernel(kern, grid, dim3(NTHREADS), T::SMEM, s, p.pdl != 0, p, tc_, tb_, tx_, th_, ty_, tz_, hb,
                         debug_withhold(SSD_DEBUG_SCAN_DECAYS));
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
