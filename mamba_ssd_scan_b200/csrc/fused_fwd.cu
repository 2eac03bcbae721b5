// fused_fwd.cu -- the whole chunked SSD forward in one persistent kernel on the
// sm_100a tensor cores (bf16 inputs, headdim 64, dstate 64 or 128, chunk 128 or
// 256): every input is read from HBM once and y written once; the states never
// leave the chip except to cross from one chunk's CTA to the next.
//
// For one (batch, chunk, head) the chunk's tokens are processed as tiles of 128
// ("MAMBA-2 Reference Implementations Comparison", section 2.2: inside a tile
// the masked-attention dual form; "MAMBA-2 Implementation Gaps", Gap 1: across
// tiles and chunks the carried state):
//
//   S_t[n,p]  = sum_{j in t} e^{cumA[end_t]-cumA[j]} dt_j B_j[n] x_j[p]     (tile state)
//   H_1       = e^{cumA[end_0]} H_0 + S_0                                  (H_0 = state entering the chunk)
//   H_out     = e^{cumA[end_1]-cumA[end_0]} H_1 + S_1                      (state leaving the chunk)
//   y[l,p]    = sum_{j<=l in t} e^{cumA[l]-cumA[j]} (C_l.B_j) dt_j x_j[p]
//             + e^{cumA[l]-cumA[start_t]} C_l . H_t[p,:]  +  D x_l[p]
//
// with cumA the in-chunk inclusive cumulative sum of dt*A (dt = softplus(dt_raw
// + dt_bias)), computed here as well.
//
// Work items are (chunk, batch, group, block of heads), handed out by an atomic
// ticket in chunk order, so an item only ever waits for items that started
// before it.  A CTA takes the item's C and B once, forms CB = C B^T for its two
// 128-row tiles on the tensor core and keeps it in TMEM (fp16 pairs with a
// power-of-two row scale), then runs its heads one after the other:
//
//   workers (warps 0-7)   scale x by the state weights into the XH buffer; build
//                         each tile's causal decay mask from CB and write it to
//                         TMEM as the A operand of the intra-chunk MMA; take the
//                         state entering the chunk (from the previous chunk's CTA,
//                         through L2), form H_1 and H_out, publish H_out, and
//                         stage H_0 / H_1 as bf16 hi + lo operands in XH; drain
//                         the accumulators (epilogue) and store y;
//   control (warp 8)      one lane issues every TMA load and every MMA: CB, the
//                         tile states S_t = B_t^T (w x_t), the intra terms
//                         Mk_t x_t and the state terms C_t (H_t^hi + H_t^lo);
//   loader (warp 9)       dt, cumA and the state weights of each head.
//
// The carry between chunks.  The state leaving a chunk goes to a two-slot ring
// in the workspace as 8-byte words, each holding two state entries rounded to
// a 16-bit significand (fp32 with the low 8 bits rounded off) and a 16-bit tag
// (chunk index + 1): the next chunk's CTA polls its own words until every tag
// matches, so no fence or separate flag sits between the two CTAs (an aligned
// 8-byte access is single-copy atomic).  The rounding is 2^-17 relative per
// chunk, against 2^-9 of the bf16 operand that the state term then takes as
// hi + lo.  The ring is zeroed before each call.
//
// TMEM columns: [0,128) CB of tiles 0/1 as packed fp16 (64 each); [128,256)
// masks of tiles 0/1 (bf16 A operands); [256,384) S_0/S_1, then the state terms
// of tiles 0/1; [384,512) intra terms of tiles 0/1.  CB lands in fp32 in
// [256,512) before it is packed.
//
// Balance: a warp reaches only the TMEM lanes of its quarter (warp % 4), and a
// causal row's work grows with its index, so tile 0's 32-row blocks are kept in
// reverse order (lane quarter q holds tile-0 rows 32 (3 - q)..) and tile 1's in
// order: every quarter then has five 32-column mask groups per head.  Ten warps
// leave at most three on a scheduler, so a thread may hold 168 registers (the
// workers need about 130): nothing spills to local memory, which with almost
// all of L1 taken by shared memory would go to L2.
//
// Decay factors in the mask follow the 32-row block midpoint split: with M the
// midpoint of the block's log2 cumA range, e^{cumA_l - cumA_j} = 2^{c_l - M}
// 2^{M - c_j}; the column factor is formed once per column, the row factor goes
// to the epilogue; blocks with a log2 span above kFastSpan use M = c of the
// block's first row and one exp2 per diagonal element.  The diagonal element
// itself (decay 1) is left out of the bf16 mask and added in fp32 in the
// epilogue as (C_l.B_l dt_l + D) x_l.
//
// Every wait is bounded.  A role whose wait runs out raises the CTA's abort
// flag and the workspace's abort word (so CTAs polling the ring stop too),
// records SSD_ERR_TIMEOUT in the status word and the CTA still frees its TMEM.
#include <stdlib.h>

#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int PD = 64;
constexpr int QMAX = 256;
constexpr int NWORK = 8;   // two per TMEM lane quarter, 32 output columns each
constexpr int CTRL_WARP = NWORK, LOAD_WARP = NWORK + 1;
constexpr int NTHREADS = (NWORK + 2) * 32;
constexpr int NW = NWORK * 32;
constexpr uint32_t T_CB = 0, T_MK = 128, T_S = 256, T_YI = 384, T_LAND = 256;
constexpr float kFastSpan = 180.0f;
constexpr float kMaxExp = 96.0f;
constexpr float kLog2e = 1.4426950408889634f;
// ring polling: rounds of 8-word loads with a short sleep between them
constexpr uint32_t kPollLimit = 1u << 21;

// workspace header (bytes): status word, abort word, ticket counter, and the
// first wait that gave up (0x10000 | warp << 8 | barrier, or 0x20000 | warp for
// the ring), for diagnosis
constexpr size_t kHdrStatus = 0, kHdrAbort = 4, kHdrTicket = 8, kHdrWhere = 16, kHdrBytes = 256;

// Optional timeline (builds with -DSSD_TRACE only): worker thread 0 stamps the
// global timer at its hand-offs of the first heads of each CTA, read back with
// ssd_fused_trace_copy().  Events per head (8 slots): X and decays in, masks
// done, S done (carry starts), entering state in, leaving state out, state
// terms done, y stored.
#ifdef SSD_TRACE
constexpr int kTraceCtas = 160, kTraceSlots = 256;
__device__ long long g_fused_trace[kTraceCtas][kTraceSlots];
#define FTRACE(ev)                                                                        \
    do {                                                                                  \
        if (tid == 0 && blockIdx.x < kTraceCtas && head_no * 8 + (ev) < kTraceSlots) {    \
            long long t_;                                                                 \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                        \
            g_fused_trace[blockIdx.x][head_no * 8 + (ev)] = t_;                           \
        }                                                                                 \
    } while (0)
#else
#define FTRACE(ev) \
    do {           \
    } while (0)
#endif

// first tile-local row of the 32-row block that TMEM lane quarter qd holds in tile t
__device__ __forceinline__ int block_row(int t, int qd) { return t == 0 ? 32 * (3 - qd) : 32 * qd; }

template <int NST>
struct FusedSmem {
    static constexpr int KBLK = QMAX * 128;                 // one 64-wide K block of C or B
    static constexpr int C_OFF = 0;
    static constexpr int C_BYTES = (NST / 64) * KBLK;
    static constexpr int B_OFF = C_OFF + C_BYTES;
    static constexpr int B_BYTES = (NST / 64) * KBLK;
    // dstate 64: a zero block right after B is the second 64-row half of the
    // tile-state MMA's A operand (M = 128 state rows, the upper 64 all zero)
    static constexpr int Z_OFF = B_OFF + B_BYTES;
    static constexpr int Z_BYTES = NST == 64 ? KBLK : 0;
    static constexpr int X_OFF = Z_OFF + Z_BYTES;
    static constexpr int X_BYTES = QMAX * 128;
    static constexpr int XH_OFF = X_OFF + X_BYTES;          // scaled x, then H hi / lo
    static constexpr int XH_BYTES = QMAX * 128;
    static constexpr int H_LO = NST * 128;                  // offset of H lo inside XH
    // per-head decays, two buffers: [cum2 (QMAX) | dt (QMAX) | state weight (QMAX) | D, pad]
    static constexpr int DEC_FLOATS = 3 * QMAX + 8;
    static constexpr int DEC_OFF = XH_OFF + XH_BYTES;
    static constexpr int RINV_OFF = DEC_OFF + 2 * DEC_FLOATS * 4;  // CB row scales, TMEM row order
    static constexpr int CBD_OFF = RINV_OFF + QMAX * 4;           // C_l . B_l, TMEM row order
    static constexpr int CN_OFF = CBD_OFF + QMAX * 4;             // |C_r|^2
    static constexpr int BN_OFF = CN_OFF + QMAX * 4;              // max |B_j|^2 per warp
    static constexpr int CTAB_OFF = BN_OFF + 16 * 4;              // per worker warp: 32 column factors
    static constexpr int XSC_OFF = CTAB_OFF + NWORK * 32 * 4;     // per token: 1 / (fp16 scale of x)
    static constexpr int DMAX_OFF = XSC_OFF + QMAX * 4;           // [head parity][tile] max dt / scale
    static constexpr int BAR_OFF = DMAX_OFF + 4 * 4;
    static constexpr int SMEM = BAR_OFF + 32 * 8 + 64 + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(2 * H_LO <= XH_BYTES, "H hi and lo fit in XH");
};

enum : int {
    B_CB_LOAD = 0, B_CB_DONE, B_CB_PACKED, B_X_FULL, B_X_FREE, B_XT_FULL, B_S_DONE, B_MK_FULL,
    B_H0_FULL, B_H0_DONE, B_H1_FULL, B_YS_FULL, B_ACC_FREE, B_DEC_FULL,
    B_DEC_FREE = B_DEC_FULL + 2, B_COUNT = B_DEC_FREE + 2
};

struct Item {
    int64_t c, b, g, hfirst;
    int Lc, ntiles;
};

__device__ __forceinline__ Item decode_item(const FwdParams& p, int64_t ticket, int hb_size) {
    const int64_t nhb = p.heads_per_group / hb_size;
    Item it;
    it.c = ticket / (p.batch * p.ngroups * nhb);
    int64_t r = ticket % (p.batch * p.ngroups * nhb);
    it.b = r / (p.ngroups * nhb);
    r %= p.ngroups * nhb;
    it.g = r / nhb;
    it.hfirst = it.g * p.heads_per_group + (r % nhb) * hb_size;
    const int64_t t0 = it.c * p.chunk;
    it.Lc = static_cast<int>(p.seqlen - t0 < p.chunk ? p.seqlen - t0 : p.chunk);
    it.ntiles = (it.Lc + 127) / 128;
    return it;
}

// Bounded mbarrier wait that gives up when another role aborted.
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

__device__ __forceinline__ void raise_abort(volatile int* abort, int* g_abort) {
    *abort = 1;
    atomicExch(g_abort, 1);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// the 24 high bits of an fp32, rounded at bit 8 (ties away from zero)
__device__ __forceinline__ uint64_t enc24(float v) {
    return static_cast<uint64_t>((__float_as_uint(v) + 0x80u) >> 8);
}
__device__ __forceinline__ float dec24(uint64_t w) { return __uint_as_float(static_cast<uint32_t>(w) << 8); }

__device__ __forceinline__ void st_u64x2_relaxed(uint64_t* p, uint64_t a, uint64_t b) {
    asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
__device__ __forceinline__ void ld_u64x2_relaxed(const uint64_t* p, uint64_t& a, uint64_t& b) {
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Instruction descriptor: f16 x f16 -> fp32 (A and B formats 0), M x N tile.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return idesc_bf16(M, N, a_mn_major, b_mn_major) & ~((7u << 7) | (7u << 10));
}

// A from TMEM: D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        :
        : "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The rows of one mask block: tile t, lane quarter qd; this lane's row.
struct RowPlan {
    float ref, cl, c_first;
    float f, w;      // epilogue row factor and diagonal weight
    float rs;        // the row's power-of-two scale into fp16 range
    bool fast;       // factored decays (warp-uniform)
    int rb;          // 32-row block index inside the tile
    int lb;          // chunk token of the block's first row
};

// The mask row l holds m[l,j] = CBp[l,j] * c_j * rs_l in fp16, CBp the packed CB
// (|CBp| < 2^14), c_j = 2^{ref - c_j} dt_j / s_j (fast) or 2^{c_l - c_j} dt_j / s_j
// (steep), s_j the fp16 scale of x_j.  For j <= l the cumulative log decay
// c_j >= c_l, so |m[l,j]| <= 2^14 * 2^{ref - c_l} * dmax * rs_l with
// dmax = max_j dt_j / s_j over the tile (2^0 in place of 2^{ref - c_l} when
// steep); rs_l brings that bound to 2^15 (fp16 holds 65504), so no element
// overflows and the row's largest elements keep all 11 bits.
__device__ __forceinline__ RowPlan plan_rows(int t, int qd, int lane, const float* cum2,
                                             const float* dtv, float rinv, float cbd, float Dh,
                                             int Lc, float dmax) {
    RowPlan r;
    const int br = block_row(t, qd);
    r.rb = br >> 5;
    r.lb = 128 * t + br;
    const int last = max(r.lb, min(r.lb + 31, Lc - 1));
    r.c_first = cum2[r.lb];
    const float c_last = cum2[last];
    r.fast = (r.c_first - c_last) <= kFastSpan;
    r.ref = r.fast ? 0.5f * (r.c_first + c_last) : r.c_first;
    r.cl = cum2[r.lb + lane];
    // log2 of the row bound: 2^{ref - c_l} is the row's largest decay factor
    // exactly (below 1 for the rows before the block's midpoint, so not
    // clamped: a looser bound would push their elements into fp16's subnormal
    // range); up to ~14 + 90 + log2 dmax on the fast path.  The scale 2^e and
    // its inverse stay normal floats for |e| <= 120.
    const float lg = 14.0f + (r.fast ? r.ref - r.cl : 0.0f) + __log2f(fmaxf(dmax, 1e-30f));
    const int e = min(120, max(-120, 15 - static_cast<int>(ceilf(fminf(fmaxf(lg, -200.0f), 200.0f)))));
    r.rs = __int_as_float((127 + e) << 23);
    const float irs = __int_as_float((127 - e) << 23);
    r.f = (r.fast ? rinv * ex2(r.cl - r.ref) : rinv) * irs;
    r.w = fmaf(cbd, dtv[r.lb + lane], Dh);
    return r;
}

// One 32-column group g of tile t's mask for this warp's rows: CB (packed
// fp16 in TMEM) times the decays and the row scale, to fp16, into the mask
// columns in TMEM.  xsc holds 1 / (fp16 scale of x) per token.
__device__ __forceinline__ void mask_group(const RowPlan& r, int t, int g, uint32_t cb_addr,
                                           uint32_t mk_addr, const float* cum2, const float* dtv,
                                           const float* xsc, float* ctab, int lane, bool first) {
    if (g > r.rb) {  // above the diagonal block: zeros (constant, written once per item)
        if (first) {
            const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            tmem_st16(mk_addr, z);
        }
        return;
    }
    uint32_t raw[16];
    tmem_ld16(cb_addr, raw);
    const int j0 = 128 * t + 32 * g;  // chunk token of the group's first column
    const float cj = ex2(fminf(r.ref - cum2[j0 + lane], kMaxExp)) * dtv[j0 + lane] * xsc[j0 + lane];
    __syncwarp();
    ctab[lane] = cj;
    __syncwarp();
    const float4* ct = reinterpret_cast<const float4*>(ctab);
    uint32_t o[16];
    const float2 rs2 = make_float2(r.rs, r.rs);
    if (g < r.rb && r.fast) {  // below the diagonal block: packed fp32x2 products
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
        tmem_st16(mk_addr, o);
        return;
    }
    float v[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 f = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&raw[i])), rs2);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
    if (g < r.rb) {  // below the diagonal block of a steep row block
        const float rr = ex2(r.cl - r.c_first);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c = ct[i];
            v[4 * i + 0] *= rr * c.x;
            v[4 * i + 1] *= rr * c.y;
            v[4 * i + 2] *= rr * c.z;
            v[4 * i + 3] *= rr * c.w;
        }
    } else if (r.fast) {  // the diagonal block, factored; j = l is left to the epilogue
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c = ct[i];
            const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int q = 4 * i + e;
                v[q] = (q < lane) ? v[q] * cc[e] : 0.0f;
            }
        }
    } else {  // the diagonal block of a steep row block: one exp2 per element
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const float e = ex2(fminf(r.cl - cum2[j0 + q], 0.0f)) * dtv[j0 + q] * xsc[j0 + q];
            v[q] = (q < lane) ? v[q] * e : 0.0f;
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = pack_f16x2(v[2 * i], v[2 * i + 1]);
    tmem_st16(mk_addr, o);
}

// 16 fp32 values -> 8 bf16 hi pairs and 8 bf16 lo pairs (lo = v - hi)
__device__ __forceinline__ void split_hi_lo(const float (&v)[16], uint32_t (&hi)[8], uint32_t (&lo)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const float2 hf = __bfloat1622float2(h);
        hi[i] = *reinterpret_cast<const uint32_t*>(&h);
        lo[i] = pack_bf16x2(v[2 * i] - hf.x, v[2 * i + 1] - hf.y);
    }
}

// H as the MN-major B operand of the state term: row n (K index), 64 p values
// (N) per 128-byte row; this thread's 32 p values are the 16-byte chunks
// 4 hf .. 4 hf + 3.
__device__ __forceinline__ void stage_h(uint32_t sXH, uint32_t lo_off, int n, int hf,
                                        const float (&v)[32]) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float part[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) part[k] = v[16 * hh + k];
        uint32_t hi[8], lo[8];
        split_hi_lo(part, hi, lo);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint32_t c = 4 * hf + 2 * hh + k;
            st_shared_v4(sXH + sw128(n, c), hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
            st_shared_v4(sXH + lo_off + sw128(n, c), lo[4 * k], lo[4 * k + 1], lo[4 * k + 2], lo[4 * k + 3]);
        }
    }
}

template <int NST, bool GATED>
__global__ void __launch_bounds__(NTHREADS, 1)
    fused_fwd_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_x,
                     int hb_size, int64_t total_items, uint64_t* ring, int64_t withhold) {
    using T = FusedSmem<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile long long* s_ticket = reinterpret_cast<volatile long long*>(tmem_slot + 2);  // 2 slots
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    char* hdr = static_cast<char*>(static_cast<void*>(p.status));
    int* g_abort = reinterpret_cast<int*>(hdr + kHdrAbort);
    int* g_where = reinterpret_cast<int*>(hdr + kHdrWhere);
    // bounded wait on barrier i; the first one in the call that gives up is recorded
    auto wb = [&](int i, uint32_t parity) {
        const bool r = wait_bar(bar(i), parity, abort);
        if (!r) atomicCAS(g_where, 0, 0x10000 | ((threadIdx.x >> 5) << 8) | i);
        return r;
    };
    unsigned long long* g_ticket = reinterpret_cast<unsigned long long*>(hdr + kHdrTicket);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = p.nheads, L = p.seqlen, nc = p.nchunks, Bsz = p.batch;
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sX = smem_u32(smem + T::X_OFF), sXH = smem_u32(smem + T::XH_OFF);
    constexpr uint32_t KB = T::KBLK;
    constexpr int64_t kWordsPerState = PD * NST / 2;

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t count = 1;
            if (i == B_CB_PACKED || i == B_XT_FULL || i == B_MK_FULL || i == B_H0_FULL ||
                i == B_H1_FULL || i == B_ACC_FREE || i == B_DEC_FREE || i == B_DEC_FREE + 1)
                count = NW;
            if (i == B_DEC_FULL || i == B_DEC_FULL + 1) count = 32;
            mbar_init(bar(i), count);
        }
        *abort = 0;
        s_ticket[0] = static_cast<long long>(atomicAdd(g_ticket, 1ull));
        float* dm = reinterpret_cast<float*>(smem + T::DMAX_OFF);
        for (int k = 0; k < 4; ++k) dm[k] = 0.0f;
        fence_mbar_init();
    }
    if (NST == 64) {  // the zero half of the tile-state A operand
        uint32_t* z = reinterpret_cast<uint32_t*>(smem + T::Z_OFF);
        for (int i = tid; i < T::Z_BYTES / 4; i += NTHREADS) z[i] = 0u;
        fence_smem_async();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // per-role phase counters that run across items
    uint32_t item_no = 0, head_no = 0;

    if (warp == CTRL_WARP) {
        // ------------------------------ control ------------------------------
        if (lane == 0) {
            tma_prefetch_map(&tm_c);
            tma_prefetch_map(&tm_b);
            tma_prefetch_map(&tm_x);
            bool ok = true;
            long long ticket = s_ticket[0];
            for (; ok && ticket < total_items; ++item_no) {
                const Item it = decode_item(p, ticket, hb_size);
                const int64_t t0 = it.c * p.chunk;
                // the next item: its ticket now (the order stays intact: a CTA
                // runs its items in ticket order), its inputs into L2.  The
                // other roles read it after their wait on this item's C/B load
                // barrier, whose expect-tx arrive below releases this store.
                const long long next = static_cast<long long>(atomicAdd(g_ticket, 1ull));
                s_ticket[(item_no + 1) & 1] = next;
                // C, B, x and the TMEM accumulators are reused once every MMA of
                // the previous head is done and its accumulators are drained
                if (head_no > 0) {
                    ok = wb(B_YS_FULL, (head_no - 1) & 1);
                    if (ok) ok = wb(B_ACC_FREE, (head_no - 1) & 1);
                    if (!ok) break;
                }
                // C in 32-row blocks (tile 0's reversed), B in 128-row tiles
                mbar_expect_tx(bar(B_CB_LOAD), 2u * (NST / 64) * it.ntiles * 128 * 128);
                for (int kb = 0; kb < NST / 64; ++kb)
                    for (int t = 0; t < it.ntiles; ++t) {
                        for (int q = 0; q < 4; ++q)
                            tma_load_4d(sC + kb * KB + (128 * t + 32 * q) * 128, &tm_c, bar(B_CB_LOAD),
                                        kb * 64, (int)it.g, (int)(t0 + 128 * t + block_row(t, q)),
                                        (int)it.b);
                        tma_load_4d(sB + kb * KB + 128 * t * 128, &tm_b, bar(B_CB_LOAD), kb * 64,
                                    (int)it.g, (int)(t0 + 128 * t), (int)it.b);
                    }
                auto load_x = [&](int64_t h) {
                    mbar_expect_tx(bar(B_X_FULL), it.ntiles * 128 * 128);
                    for (int t = 0; t < it.ntiles; ++t)
                        tma_load_4d(sX + t * 128 * 128, &tm_x, bar(B_X_FULL), 0, (int)h,
                                    (int)(t0 + 128 * t), (int)it.b);
                };
                load_x(it.hfirst);
                if (next < total_items) {
                    const Item nx = decode_item(p, next, hb_size);
                    const int64_t n0 = nx.c * p.chunk;
                    for (int kb = 0; kb < NST / 64; ++kb)
                        for (int t = 0; t < nx.ntiles; ++t) {
                            tma_prefetch_l2_4d(&tm_b, kb * 64, (int)nx.g, (int)(n0 + 128 * t), (int)nx.b);
                            for (int q = 0; q < 4; ++q)
                                tma_prefetch_l2_4d(&tm_c, kb * 64, (int)nx.g,
                                                   (int)(n0 + 128 * t + block_row(t, q)), (int)nx.b);
                        }
                }
                ok = wb(B_CB_LOAD, item_no & 1);
                if (ok) {
                    fence_after_sync();
                    for (int t = 0; t < it.ntiles; ++t) {
                        const uint32_t id = idesc_bf16(128, 128, false, false);
                        for (int k = 0; k < NST / 16; ++k) {
                            const uint32_t ko = (k >> 2) * KB + (k & 3) * 32 + 128 * t * 128;
                            mma_bf16(tmem + T_LAND + 128 * t, desc_sw128(sC + ko, 16, 1024),
                                     desc_sw128(sB + ko, 16, 1024), id, k > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(bar(B_CB_DONE));
                    ok = wb(B_CB_PACKED, item_no & 1);
                    fence_after_sync();
                }
                for (int i = 0; ok && i < hb_size; ++i, ++head_no) {
                    const uint32_t ph = head_no & 1;
                    // tile states S_t = B_t^T (w x_t): A = B (MN-major, M = states),
                    // B operand = scaled x (MN-major, N = p)
                    ok = wb(B_XT_FULL, ph);
                    if (ok && head_no > 0) ok = wb(B_ACC_FREE, ph ^ 1);
                    if (!ok) break;
                    fence_after_sync();
                    for (int t = 0; t < it.ntiles; ++t) {
                        const uint32_t id = idesc_bf16(128, PD, true, true);
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t off = 128 * t * 128 + k * 2048;
                            mma_bf16(tmem + T_S + 64 * t, desc_sw128(sB + off, KB, 1024),
                                     desc_sw128(sXH + off, KB, 1024), id, k > 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(bar(B_S_DONE));
                    // intra-chunk terms Mk_t x_t: A = the mask in TMEM, B = x (MN-major)
                    ok = wb(B_MK_FULL, ph);
                    if (!ok) break;
                    fence_after_sync();
                    for (int t = 0; t < it.ntiles; ++t) {
                        const uint32_t id = idesc_f16(128, PD, false, true);  // fp16 mask x fp16 x
                        for (int k = 0; k < 8; ++k)
                            mma_bf16_ts(tmem + T_YI + 64 * t, tmem + T_MK + 64 * t + 8 * k,
                                        desc_sw128(sX + 128 * t * 128 + k * 2048, KB, 1024), id,
                                        k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_X_FREE));
                    if (i + 1 < hb_size) {  // the next head's x, once this one's MMAs are done with it
                        ok = wb(B_X_FREE, ph);
                        if (!ok) break;
                        load_x(it.hfirst + i + 1);
                    } else if (next < total_items) {
                        const Item nx = decode_item(p, next, hb_size);
                        for (int t = 0; t < nx.ntiles; ++t)
                            tma_prefetch_l2_4d(&tm_x, 0, (int)nx.hfirst, (int)(nx.c * p.chunk + 128 * t),
                                               (int)nx.b);
                    }
                    // state terms C_t (H_t^hi + H_t^lo): A = C (K-major), B = H (MN-major)
                    for (int t = 0; ok && t < it.ntiles; ++t) {
                        ok = wb(t == 0 ? B_H0_FULL : B_H1_FULL, ph);
                        if (!ok) break;
                        fence_after_sync();
                        const uint32_t id = idesc_bf16(128, PD, false, true);
                        for (int part = 0; part < 2; ++part)
                            for (int k = 0; k < NST / 16; ++k) {
                                const uint32_t ko = (k >> 2) * KB + (k & 3) * 32 + 128 * t * 128;
                                mma_bf16(tmem + T_S + 64 * t, desc_sw128(sC + ko, 16, 1024),
                                         desc_sw128(sXH + part * T::H_LO + k * 2048, KB, 1024), id,
                                         (part | k) ? 1u : 0u);
                            }
                        if (t == 0) mma_commit(bar(B_H0_DONE));
                    }
                    if (ok) mma_commit(bar(B_YS_FULL));
                }
                ticket = next;
            }
            if (!ok) raise_abort(abort, g_abort);
        }
    } else if (warp == LOAD_WARP) {
        // ------------------------------- loader ------------------------------
        // dt = softplus(dt_raw + dt_bias), the inclusive in-chunk cumulative
        // sum of dt * A (as log2(e) * cumA), and the tile-state weights
        // 2^{cum2[end_t] - cum2[l]} dt_l of each head, into the two buffers.
        // Slots past the chunk's last token hold dt = 0 and its last cumA.
        bool ok = true;
        long long ticket = s_ticket[0];
        const __nv_bfloat16* dtr = static_cast<const __nv_bfloat16*>(p.dt_raw);
        for (; ok && ticket < total_items; ++item_no) {
            const Item it = decode_item(p, ticket, hb_size);
            const int64_t t0 = it.c * p.chunk;
            ok = wb(B_CB_LOAD, item_no & 1);  // (also publishes the next ticket)
            for (int i = 0; ok && i < hb_size; ++i, ++head_no) {
                const int bsel = head_no & 1;
                if (head_no >= 2) ok = wb(B_DEC_FREE + bsel, ((head_no - 2) >> 1) & 1);
                if (!ok) break;
                const int64_t h = it.hfirst + i;
                const float A = p.A[h], bias = p.dt_bias ? p.dt_bias[h] : 0.0f;
                float u[8];
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int l = 32 * s + lane;
                    u[s] = l < it.Lc ? __bfloat162float(dtr[((it.b * L) + t0 + l) * H + h]) : 0.0f;
                }
                float* dec = reinterpret_cast<float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
                float carry = 0.0f, cv[8], dv[8];
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int l = 32 * s + lane;
                    float dt = 0.0f, v = 0.0f;
                    if (l < it.Lc) {
                        dt = softplus_f32(u[s] + bias);
                        v = dt * A;
                    }
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float n = __shfl_up_sync(0xffffffffu, v, o);
                        if (lane >= o) v += n;
                    }
                    v += carry;
                    carry = __shfl_sync(0xffffffffu, v, 31);
                    cv[s] = v * kLog2e;
                    dv[s] = dt;
                }
                const float end0 = __shfl_sync(0xffffffffu, cv[3], 31);
                const float end1 = __shfl_sync(0xffffffffu, cv[7], 31);
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int l = 32 * s + lane;
                    dec[l] = cv[s];
                    dec[QMAX + l] = dv[s];
                    dec[2 * QMAX + l] = ex2((s < 4 ? end0 : end1) - cv[s]) * dv[s];
                }
                if (lane == 0) dec[3 * QMAX] = p.D ? p.D[h] : 0.0f;
                mbar_arrive(bar(B_DEC_FULL + bsel));
            }
            ticket = s_ticket[(item_no + 1) & 1];
        }
        if (!ok) raise_abort(abort, g_abort);
    } else {
        // ------------------------------ workers ------------------------------
        // warp (qd, hf): TMEM lanes 32 qd.., output columns p in [32 hf, 32 hf + 32),
        // mask column groups hf and hf + 2 of each tile
        const int qd = warp & 3, hf = warp >> 2;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        float* rinv_s = reinterpret_cast<float*>(smem + T::RINV_OFF);
        float* cbd_s = reinterpret_cast<float*>(smem + T::CBD_OFF);
        float* cn_s = reinterpret_cast<float*>(smem + T::CN_OFF);
        float* bn_s = reinterpret_cast<float*>(smem + T::BN_OFF);
        float* ctab = reinterpret_cast<float*>(smem + T::CTAB_OFF) + warp * 32;
        const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
        const __nv_bfloat16* zg = static_cast<const __nv_bfloat16*>(p.z);
        __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
        bool ok = true;
        long long ticket = s_ticket[0];
        for (; ok && ticket < total_items; ++item_no) {
            const Item it = decode_item(p, ticket, hb_size);
            const int64_t t0 = it.c * p.chunk;
            // --- CB repack: fp32 landing -> fp16 pairs with a power-of-two
            // scale per row, chosen from |C_l . B_j| <= |C_l| max_j |B_j|
            ok = wb(B_CB_LOAD, item_no & 1);
            if (ok) {
                const int r = tid;  // C row r and B row r (256 each)
                const bool valid = r < 128 * it.ntiles;
                float sc = 0.0f, sb = 0.0f;
                if (valid) {
#pragma unroll
                    for (int kb = 0; kb < NST / 64; ++kb)
#pragma unroll
                        for (int c16 = 0; c16 < 8; ++c16) {
                            const uint32_t o = r * 128 + kb * KB + ((c16 + lane) & 7) * 16;
                            const uint4 vc = ld_shared_v4(sC + o), vb = ld_shared_v4(sB + o);
                            const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wbv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wc[e]));
                                const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wbv[e]));
                                sc = fmaf(f.x, f.x, fmaf(f.y, f.y, sc));
                                sb = fmaf(g2.x, g2.x, fmaf(g2.y, g2.y, sb));
                            }
                        }
                }
                cn_s[r] = sc;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sb = fmaxf(sb, __shfl_xor_sync(0xffffffffu, sb, o));
                if (lane == 0) bn_s[warp] = sb;  // warps 0-3: tile 0 rows, 4-7: tile 1
            }
            named_sync(1, NW);
            float sc_t[2] = {1.0f, 1.0f};
            if (ok) {
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t >= it.ntiles) continue;
                    const float bmax = fmaxf(fmaxf(bn_s[4 * t], bn_s[4 * t + 1]),
                                             fmaxf(bn_s[4 * t + 2], bn_s[4 * t + 3]));
                    const int rr = 128 * t + 32 * qd + lane;  // C row in smem = TMEM row of tile t
                    const float bound = sqrtf(cn_s[rr] * bmax);
                    const int e2 = max(0, ((__float_as_int(bound) >> 23) & 255) - 127 - 13 + 1);
                    sc_t[t] = __int_as_float((127 - e2) << 23);
                    if (hf == 0) rinv_s[rr] = __int_as_float((127 + e2) << 23);
                }
                ok = wb(B_CB_DONE, item_no & 1);
            }
            if (ok) {
                fence_after_sync();
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t >= it.ntiles) continue;
                    const int rb = block_row(t, qd) >> 5;  // the group holding the diagonal
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int g = 2 * hf + k;
                        float v[32];
                        tmem_ld32(tmem + lanes + T_LAND + 128 * t + 32 * g, v);
                        if (g == rb) {
                            float dg = 0.0f;
#pragma unroll
                            for (int q = 0; q < 32; ++q) dg = (q == lane) ? v[q] : dg;
                            cbd_s[128 * t + 32 * qd + lane] = dg;
                        }
                        uint32_t r16[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) r16[q] = pack_f16x2(v[2 * q] * sc_t[t], v[2 * q + 1] * sc_t[t]);
                        tmem_st16(tmem + lanes + T_CB + 64 * t + 16 * g, r16);
                    }
                }
                tmem_wait_st();
            }
            fence_before_sync();
            mbar_arrive(bar(B_CB_PACKED));
            if (ok) ok = wb(B_CB_PACKED, item_no & 1);
            fence_after_sync();
            float rinv_t[2] = {1.0f, 1.0f}, cbd_t[2] = {0.0f, 0.0f};
            if (ok)
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t >= it.ntiles) continue;
                    rinv_t[t] = rinv_s[128 * t + 32 * qd + lane];
                    cbd_t[t] = cbd_s[128 * t + 32 * qd + lane];
                }

            for (int i = 0; ok && i < hb_size; ++i, ++head_no) {
                const uint32_t ph = head_no & 1;
                const int bsel = head_no & 1;
                const int64_t h = it.hfirst + i;
                const float* dec = reinterpret_cast<const float*>(smem + T::DEC_OFF) + bsel * T::DEC_FLOATS;
                const float* cum2 = dec;
                const float* dtv = dec + QMAX;
                const float* wst = dec + 2 * QMAX;
                ok = wb(B_DEC_FULL + bsel, (head_no >> 1) & 1);
                if (ok) ok = wb(B_X_FULL, ph);
                if (!ok) break;
                FTRACE(0);
                // --- scaled x for the tile states (bf16, into XH) and x itself as
                // fp16 in place for the intra-chunk MMA: rows l, 16-byte chunks;
                // the 8 chunks of a row sit in 8 consecutive lanes, which agree
                // on a power-of-two scale s_l taking the row's largest |x| to
                // [2^13, 2^14) (bf16 values are exact in fp16 there)
                float* xsc = reinterpret_cast<float*>(smem + T::XSC_OFF);
                float* dmax_s = reinterpret_cast<float*>(smem + T::DMAX_OFF) + 2 * (head_no & 1);
                float dloc[2] = {0.0f, 0.0f};
                for (int k = tid; k < it.ntiles * 128 * 8; k += NW) {
                    const int l = k >> 3, ch = k & 7;
                    const uint32_t off = sw128(l, ch);
                    const uint4 v = ld_shared_v4(sX + off);
                    const float w = wst[l];
                    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
                    uint32_t out[4];
                    float f8[8];
                    float amax = 0.0f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[e]));
                        out[e] = pack_bf16x2(f.x * w, f.y * w);
                        f8[2 * e] = f.x;
                        f8[2 * e + 1] = f.y;
                        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
                    }
                    st_shared_v4(sXH + off, out[0], out[1], out[2], out[3]);
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                    const int ex = amax > 0.0f ? ((__float_as_int(amax) >> 23) & 255) - 127 : 0;
                    const int es = min(100, max(-100, 13 - ex));  // s = 2^es
                    const float sc = __int_as_float((127 + es) << 23);
#pragma unroll
                    for (int e = 0; e < 4; ++e) out[e] = pack_f16x2(f8[2 * e] * sc, f8[2 * e + 1] * sc);
                    st_shared_v4(sX + off, out[0], out[1], out[2], out[3]);
                    if (ch == 0) {
                        const float inv = __int_as_float((127 - es) << 23);
                        xsc[l] = inv;
                        const float dv = dtv[l] * inv;
                        if (l < 128) dloc[0] = fmaxf(dloc[0], dv);
                        else dloc[1] = fmaxf(dloc[1], dv);
                    }
                }
                fence_smem_async();
                mbar_arrive(bar(B_XT_FULL));
                // the tile's max dt / s: per-warp max, then one shared-memory max
#pragma unroll
                for (int t = 0; t < 2; ++t) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) dloc[t] = fmaxf(dloc[t], __shfl_xor_sync(0xffffffffu, dloc[t], o));
                    if (lane == 0) atomicMax(reinterpret_cast<int*>(dmax_s + t), __float_as_int(dloc[t]));
                }
                named_sync(2, NW);  // every x row converted, its scale and the bound in
                // --- masks of both tiles into TMEM; the epilogue keeps each tile's
                // row factor, diagonal weight and row
                const float Dh = dec[3 * QMAX];
                float ep_f[2], ep_w[2], ep_cl[2];
                int ep_l[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    ep_f[t] = 1.0f; ep_w[t] = 0.0f; ep_cl[t] = 0.0f; ep_l[t] = QMAX;
                    if (t >= it.ntiles) continue;
                    const RowPlan rp = plan_rows(t, qd, lane, cum2, dtv, rinv_t[t], cbd_t[t], Dh, it.Lc, dmax_s[t]);
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int g = hf + 2 * k;
                        mask_group(rp, t, g, tmem + lanes + T_CB + 64 * t + 16 * g,
                                   tmem + lanes + T_MK + 64 * t + 16 * g, cum2, dtv, xsc, ctab, lane, i == 0);
                    }
                    ep_f[t] = rp.f; ep_w[t] = rp.w; ep_cl[t] = rp.cl; ep_l[t] = rp.lb + lane;
                }
                tmem_wait_st();
                fence_before_sync();
                mbar_arrive(bar(B_MK_FULL));
                // the previous head's bound slots are free (every worker is past that
                // head's masks: this head's x pass ended with a workers' barrier)
                if (tid == 0) {
                    float* other = reinterpret_cast<float*>(smem + T::DMAX_OFF) + 2 * ((head_no & 1) ^ 1);
                    other[0] = 0.0f;
                    other[1] = 0.0f;
                }
                FTRACE(1);
                // --- the carry: state entering the chunk, H_1 and the state leaving it
                ok = wb(B_S_DONE, ph);
                if (!ok) break;
                fence_after_sync();
                FTRACE(2);
                const int n = 32 * qd + lane;  // state row (TMEM lane of S_t)
                const bool has_state = n < NST;
                float hin[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) hin[k] = 0.0f;
                if (has_state) {
                    if (it.c == 0) {
                        if (p.init_state) {
                            const float* ip = p.init_state + ((it.b * H + h) * PD + 32 * hf) * NST + n;
#pragma unroll
                            for (int k = 0; k < 32; ++k) hin[k] = ip[k * NST];
                        }
                    } else {
                        const uint64_t* src = ring + (((it.c - 1) & 1) * Bsz + it.b) * H * kWordsPerState +
                                              h * kWordsPerState + n * (PD / 2) + 16 * hf;
                        const uint64_t tag = static_cast<uint64_t>(it.c & 0xFFFF) << 48;
                        uint32_t rounds = 0;
                        // lane 0 polls one word of the warp's rows until its tag
                        // arrives; then every lane loads its sixteen words (the
                        // producer stored them all at about the same time) and
                        // re-polls only while one of them is still stale
                        if (lane == 0) {
                            for (;;) {
                                uint64_t w0, w1;
                                ld_u64x2_relaxed(src, w0, w1);
                                if ((w0 & 0xFFFF000000000000ull) == tag) break;
                                if (++rounds >= kPollLimit ||
                                    ((rounds & 31) == 0 && (*abort || ld_acquire(g_abort)))) {
                                    ok = false;
                                    break;
                                }
                                __nanosleep(32);
                            }
                        }
                        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                        // word pairs one at a time: load (again while stale), decode
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            uint64_t w0 = 0, w1 = 0;
                            for (; ok;) {
                                ld_u64x2_relaxed(src + 2 * k, w0, w1);
                                if ((w0 & 0xFFFF000000000000ull) == tag && (w1 & 0xFFFF000000000000ull) == tag)
                                    break;
                                if (++rounds >= kPollLimit ||
                                    ((rounds & 31) == 0 && (*abort || ld_acquire(g_abort)))) {
                                    ok = false;
                                    break;
                                }
                                __nanosleep(32);
                            }
                            hin[4 * k] = dec24(w0 & 0xFFFFFFull);
                            hin[4 * k + 1] = dec24((w0 >> 24) & 0xFFFFFFull);
                            hin[4 * k + 2] = dec24(w1 & 0xFFFFFFull);
                            hin[4 * k + 3] = dec24((w1 >> 24) & 0xFFFFFFull);
                        }
                        if (!ok && rounds >= kPollLimit) atomicCAS(g_where, 0, 0x20000 | warp);
                    }
                }
                if (!ok) {
                    raise_abort(abort, g_abort);
                    break;
                }
                FTRACE(3);
                {
                    // H_1 = a0 H_0 + S_0 is parked in S_1's TMEM columns (same
                    // [n][p] layout; free once S_1 is read) until the tile-0 state
                    // term has consumed the H_0 operand.  Order keeps at most
                    // three 32-value arrays live: H_0 + S_0 -> H_1; H_0 staged;
                    // S_1 read, H_1 parked, H_out = a1 H_1 + S_1 published.
                    float hmid[32];
                    {
                        uint32_t sr[2][16];
                        const uint32_t a0s[2] = {tmem + lanes + T_S + 32 * hf, tmem + lanes + T_S + 32 * hf + 16};
                        tmem_ld16x2(a0s, sr);  // S_0
                        const float a0 = ex2(cum2[127]);
#pragma unroll
                        for (int k = 0; k < 32; ++k) hmid[k] = fmaf(a0, hin[k], __uint_as_float(sr[k >> 4][k & 15]));
                    }
                    // H_0 as the tile-0 state operand: the state term starts while
                    // the leaving state is formed and published
                    if (has_state) {
                        stage_h(sXH, T::H_LO, n, hf, hin);
                        fence_smem_async();
                    }
                    fence_before_sync();
                    mbar_arrive(bar(B_H0_FULL));
                    {
                        uint32_t sr[2][16];
                        const uint32_t a1s[2] = {tmem + lanes + T_S + 64 + 32 * hf, tmem + lanes + T_S + 64 + 32 * hf + 16};
                        tmem_ld16x2(a1s, sr);  // S_1 (read before H_1 takes its columns)
                        uint32_t hm[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) hm[k] = __float_as_uint(hmid[k]);
                        tmem_st16(a1s[0], hm);
#pragma unroll
                        for (int k = 0; k < 16; ++k) hm[k] = __float_as_uint(hmid[16 + k]);
                        tmem_st16(a1s[1], hm);
                        const float a1 = ex2(cum2[QMAX - 1] - cum2[127]);
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            hmid[k] = it.ntiles == 2 ? fmaf(a1, hmid[k], __uint_as_float(sr[k >> 4][k & 15])) : hmid[k];
                        tmem_wait_st();
                    }
                    // hmid now holds H_out
                    if (has_state) {
                        if (it.c == nc - 1) {
                            if (p.final_state) {
                                float* fp = p.final_state + ((it.b * H + h) * PD + 32 * hf) * NST + n;
#pragma unroll
                                for (int k = 0; k < 32; ++k) fp[k * NST] = hmid[k];
                            }
                        } else if (it.c != withhold) {  // (the test hook withholds one chunk's)
                            uint64_t* dst = ring + ((it.c & 1) * Bsz + it.b) * H * kWordsPerState +
                                            h * kWordsPerState + n * (PD / 2) + 16 * hf;
                            const uint64_t tag = static_cast<uint64_t>((it.c + 1) & 0xFFFF) << 48;
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const uint64_t w0 = tag | (enc24(hmid[4 * k + 1]) & 0xFFFFFFull) << 24 |
                                                    (enc24(hmid[4 * k]) & 0xFFFFFFull);
                                const uint64_t w1 = tag | (enc24(hmid[4 * k + 3]) & 0xFFFFFFull) << 24 |
                                                    (enc24(hmid[4 * k + 2]) & 0xFFFFFFull);
                                st_u64x2_relaxed(dst + 2 * k, w0, w1);
                            }
                        }
                    }
                }
                FTRACE(4);
                // (one phase of H1_FULL per head, also when the chunk has one tile)
                if (it.ntiles == 2) {
                    ok = wb(B_H0_DONE, ph);
                    if (!ok) break;
                    fence_after_sync();
                    float hmid[32];
                    {
                        uint32_t r2[2][16];
                        const uint32_t a1s[2] = {tmem + lanes + T_S + 64 + 32 * hf, tmem + lanes + T_S + 64 + 32 * hf + 16};
                        tmem_ld16x2(a1s, r2);
#pragma unroll
                        for (int k = 0; k < 32; ++k) hmid[k] = __uint_as_float(r2[k >> 4][k & 15]);
                    }
                    if (has_state) stage_h(sXH, T::H_LO, n, hf, hmid);
                    fence_smem_async();
                    fence_before_sync();
                }
                mbar_arrive(bar(B_H1_FULL));
                // --- epilogue: y = f * intra + 2^{c_l - ref_t} * state + w x_l,
                // one tile at a time (each tile's accumulators are 64 registers)
                uint4 xv[4];
                if (ep_l[0] < it.Lc) {
                    const uint4* xr = reinterpret_cast<const uint4*>(
                        xg + ((it.b * L + t0 + ep_l[0]) * H + h) * PD + 32 * hf);
#pragma unroll
                    for (int k = 0; k < 4; ++k) xv[k] = ldg16(xr + k);
                }
                const float c127 = cum2[127];
                ok = wb(B_YS_FULL, ph);
                if (!ok) break;
                fence_after_sync();
                FTRACE(5);
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t >= it.ntiles) continue;
                    const bool live = ep_l[t] < it.Lc;
                    const int64_t off = ((it.b * L + t0 + ep_l[t]) * H + h) * PD + 32 * hf;
                    const float s = ex2(ep_cl[t] - (t == 0 ? 0.0f : c127));
                    const float2 f2 = make_float2(ep_f[t], ep_f[t]), s2 = make_float2(s, s);
                    const float2 w2 = make_float2(ep_w[t], ep_w[t]);
                    uint4* yr = reinterpret_cast<uint4*>(yg + off);
                    if (t == 1 && live) {
                        const uint4* xr = reinterpret_cast<const uint4*>(xg + off);
#pragma unroll
                        for (int k = 0; k < 4; ++k) xv[k] = ldg16(xr + k);
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t acc[2][16];  // [intra, state][16 columns]
                        const uint32_t a2[2] = {tmem + lanes + T_YI + 64 * t + 32 * hf + 16 * hh,
                                                tmem + lanes + T_S + 64 * t + 32 * hf + 16 * hh};
                        tmem_ld16x2(a2, acc);
                        if (hh == 1 && t == it.ntiles - 1) {  // every accumulator of the head is read
                            fence_before_sync();
                            mbar_arrive(bar(B_ACC_FREE));
                            mbar_arrive(bar(B_DEC_FREE + bsel));
                        }
                        if (!live) continue;
                        uint4 zv[2];
                        if (GATED) {
                            const uint4* zr = reinterpret_cast<const uint4*>(zg + off) + 2 * hh;
                            zv[0] = ldg16(zr);
                            zv[1] = ldg16(zr + 1);
                        }
                        const uint32_t xw[8] = {xv[2 * hh].x, xv[2 * hh].y, xv[2 * hh].z, xv[2 * hh].w,
                                                xv[2 * hh + 1].x, xv[2 * hh + 1].y, xv[2 * hh + 1].z,
                                                xv[2 * hh + 1].w};
                        uint32_t o[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[k]));
                            const float2 vi = make_float2(__uint_as_float(acc[0][2 * k]), __uint_as_float(acc[0][2 * k + 1]));
                            const float2 vs = make_float2(__uint_as_float(acc[1][2 * k]), __uint_as_float(acc[1][2 * k + 1]));
                            float2 yv = __ffma2_rn(w2, xf, __ffma2_rn(s2, vs, __fmul2_rn(f2, vi)));
                            if (GATED) {
                                const uint32_t zw[8] = {zv[0].x, zv[0].y, zv[0].z, zv[0].w,
                                                        zv[1].x, zv[1].y, zv[1].z, zv[1].w};
                                const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[k]));
                                yv.x *= silu_f32(zf.x);
                                yv.y *= silu_f32(zf.y);
                            }
                            o[k] = pack_bf16x2(yv.x, yv.y);
                        }
                        yr[2 * hh] = make_uint4(o[0], o[1], o[2], o[3]);
                        yr[2 * hh + 1] = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
                FTRACE(6);
            }
            ticket = s_ticket[(item_no + 1) & 1];  // published before this item's C/B load
        }
        if (!ok) raise_abort(abort, g_abort);
    }
    fence_before_sync();
    __syncthreads();
    if (*abort && tid == 0) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// Heads per work item: each item pays a fixed set-up (C and B, CB and its
// repack) and then runs its heads one after the other; with w waves of items
// over the CTAs the kernel takes about w * (setup + heads * per_head).  The
// divisor of the heads per group that minimises this is used (up to 16).
int fused_heads_per_item(const FwdParams& p, int ctas) {
    static const int forced = [] {
        const char* e = getenv("SSD_FUSED_HEADS_PER_ITEM");
        return e ? atoi(e) : 0;
    }();
    if (forced > 0 && p.heads_per_group % forced == 0) return forced;
    const int64_t units = p.batch * p.nchunks * p.ngroups;
    const double setup = 3.0, per_head = 2.5 * (p.chunk > 128 ? 1.0 : 0.5);
    int best = 1;
    double best_t = 0.0;
    for (int d = 1; d <= p.heads_per_group && d <= 16; ++d) {
        if (p.heads_per_group % d) continue;
        const int64_t items = units * (p.heads_per_group / d);
        const double waves = static_cast<double>(items) / ctas;
        const double t = (waves < 1.0 ? 1.0 : waves) * (setup + per_head * d);
        if (d == 1 || t < best_t) {
            best = d;
            best_t = t;
        }
    }
    return best;
}

template <int NST, bool GATED>
cudaError_t launch_nd(const FwdParams& p, void* ws, cudaStream_t s) {
    using T = FusedSmem<NST>;
    auto kern = fused_fwd_kernel<NST, GATED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, T::SMEM) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        sms = 148;
        per_sm = 1;
    }
    const int ctas_max = sms * per_sm;
    const int hb = fused_heads_per_item(p, ctas_max);
    const int64_t items = p.batch * p.nchunks * p.ngroups * (p.heads_per_group / hb);
    const int grid = static_cast<int>(items < ctas_max ? items : ctas_max);
    CUtensorMap tc_, tb_, tx_;
    if (!make_tmap_bf16_4d(&tc_, p.C, NST, p.ngroups, p.seqlen, p.batch, 1, 32) ||
        !make_tmap_bf16_4d(&tb_, p.B, NST, p.ngroups, p.seqlen, p.batch, 1, 128) ||
        !make_tmap_bf16_4d(&tx_, p.x, PD, p.nheads, p.seqlen, p.batch, 1, 128))
        return cudaErrorInvalidValue;
    // the header (status, abort word, ticket) and the ring start from zero
    e = cudaMemsetAsync(ws, 0, fused_fwd_workspace_bytes(p), s);
    if (e != cudaSuccess) return e;
    FwdParams q = p;
    q.status = static_cast<int*>(ws);
    uint64_t* ring = reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + kHdrBytes);
    return launch_kernel(kern, dim3(grid), dim3(NTHREADS), T::SMEM, s, false, q, tc_, tb_, tx_, hb, items,
                         ring, debug_withhold(SSD_DEBUG_FWD_CARRY));
}

}  // namespace

#ifdef SSD_TRACE
extern "C" int ssd_fused_trace_copy(void* dst) {
    return cudaMemcpyFromSymbol(dst, g_fused_trace, sizeof(g_fused_trace)) == cudaSuccess ? 0 : 1;
}
#endif

bool fused_fwd_supported(const FwdParams& p) {
    return p.headdim == PD && (p.dstate == 64 || p.dstate == 128) &&
           (p.chunk == 128 || p.chunk == 256) && p.nchunks < 65535;
}

size_t fused_fwd_workspace_bytes(const FwdParams& p) {
    return kHdrBytes + 2ull * p.batch * p.nheads * p.headdim * p.dstate * sizeof(float);
}

cudaError_t launch_fused_fwd(const FwdParams& p, void* ws, cudaStream_t s) {
    if (p.dstate == 64) return p.z ? launch_nd<64, true>(p, ws, s) : launch_nd<64, false>(p, ws, s);
    if (p.dstate == 128) return p.z ? launch_nd<128, true>(p, ws, s) : launch_nd<128, false>(p, ws, s);
    return cudaErrorInvalidValue;
}

}  // namespace ssd
