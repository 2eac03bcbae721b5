// fused_fwd.cu -- the whole chunked SSD forward in one persistent kernel on the
// sm_100a tensor cores (bf16 inputs, headdim 64, dstate 64 or 128): every input
// is read from HBM once and y written once; the states never leave the chip
// except to cross from one cluster of CTAs to the next.
//
// The sequence is cut into tiles of 128 tokens ("MAMBA-2 Reference
// Implementations Comparison", section 2.2: inside a tile the masked-attention
// dual form; "MAMBA-2 Implementation Gaps", Gap 1: across tiles the carried
// state).  With c the log2 of the in-tile inclusive cumulative sum of dt*A and
// H_k the state entering tile k:
//
//   S_k[n,p]  = sum_{j in k} 2^{c_end - c_j} dt_j B_j[n] x_j[p]            (tile state)
//   H_{k+1}   = 2^{c_end} H_k + S_k                                        (carry)
//   y[l,p]    = sum_{j<=l in k} 2^{c_l - c_j} (C_l.B_j) dt_j x_j[p] + D x_l[p]
//             + 2^{c_l} C_l . H_k[p,:]
//
// A cluster of KC CTAs (KC = 4 for sequences of three tiles or more) takes KC
// consecutive tiles, one per CTA, for one (batch, group, block of heads):
// a "run".  Inside the run the state is carried as a prefix aggregate through
// distributed shared memory, off the critical path: rank k receives
// P_k = sum_{k'<k} (decay k'+1..k-1) S_k' and the log2 decay of tiles 0..k-1
// from rank k-1 as soon as that rank's tile state is known, and stores
// P_{k+1} = 2^{c_end} P_k + S_k into rank k+1's slot.  The state entering the
// run, H_in, is read by every rank from the previous run's output in L2; each
// forms its own entering state H_k = 2^{log A_<k} H_in + P_k, and the last
// rank publishes H_out = 2^{c_end} H_last + S_last.  So the chain that must
// run in sequence has one link per run, not per tile, and the only data that
// crosses between CTAs of a cluster is one state per tile boundary
// (distributed shared memory moves about 26 GB/s per SM on B200, so the
// entering state is not forwarded that way).
//
// Work items are (run, batch, group, block of heads), in run order; cluster i
// takes items i, i + nclusters, ... (every cluster of the grid is resident, so
// an item only ever waits for items that some cluster is running or has run).
// Inside a CTA the heads of an item go through a pipeline of warp groups on
// mbarriers, two heads in flight:
//
//   mask group (warps 0-3)    x -> bf16 state-weighted x~ (tile-state operand)
//                             and fp16 row-scaled x in place (intra operand);
//                             the causal decay mask from CB into TMEM (the A
//                             operand of the intra MMA), diagonal and D folded in
//   carry group (warps 4-7)   the entering state, staged as bf16 hi + lo operands
//                             of the state term; the last rank publishes the
//                             run's leaving state
//   epilogue (warps 8-11)     y = f_l (intra) + 2^{c_l} (state term), stored; on
//                             the ranks before the last also the prefix step
//                             (tile state -> prefix for the next rank), one head
//                             ahead, so it never waits behind the chain
//   control (warp 12)         TMA loads; CB, tile-state and intra MMAs
//   loader (warp 13)          dt = softplus(dt_raw + dt_bias), cumulative decays
//   state issuer (warp 14)    the state-term MMAs (the only ones that wait on
//                             the chain, so the others never queue behind them)
//
// Shared memory holds two C tiles (C is the only operand whose release waits on
// the chain: the state-term MMAs read it), so the next item's tile-state and
// intra work starts while the last heads of the current one wait.
//
// TMEM columns: [0,64) CB as packed fp16 (row-scaled), [64,128) the mask of the
// current head; CB lands in fp32 in [0,128) once per item.  [128,256) tile
// states (on the ranks between the first and the last, then P_k once the
// prefix is sent), [256,384) intra terms, [384,512) state terms: two heads each.
//
// Mask numerics (per 32-row block of the tile): with M the midpoint of the
// block's log2 decay range, e^{cumA_l - cumA_j} = 2^{c_l - M} 2^{M - c_j}; the
// column factor 2^{M - c_j} dt_j / s_j (s_j the fp16 scale of x_j) is formed
// once per column, the row factor goes to the epilogue; a row scale 2^e brings
// each row's bound to the top of fp16's range.  Blocks with a log2 span above
// kFastSpan use exact decays (one exp2 per diagonal-block element).
//
// The carry between runs goes through a two-slot ring in the workspace as
// 8-byte words, each holding two state entries rounded to a 16-bit significand
// (fp32 with the low 8 bits rounded off) and a 16-bit tag (run index + 1):
// readers poll their words until every tag matches, so no fence or separate
// flag sits between writer and readers (an aligned 8-byte access is
// single-copy atomic).  A slot is rewritten two runs later; its writer first
// waits until every reader of the slot's previous state has counted itself in
// (a release add per reading warp against an acquire load).  The ring and the
// counts are zeroed before each call.
//
// Every wait is bounded.  A role whose wait runs out raises the CTA's abort
// flag and the workspace's abort word (so every other CTA stops too), records
// SSD_ERR_TIMEOUT in the status word, and the CTA still waits for its copies
// in flight, meets its cluster and frees its TMEM.
#include <stdlib.h>

#include "internal.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int PD = 64;    // headdim
constexpr int TL = 128;   // tokens per tile (per CTA)
constexpr int CARRY_W0 = 4, EPI_W0 = 8, CTRL_WARP = 12, LOAD_WARP = 13, HCTRL_WARP = 14;
constexpr int NTHREADS = 15 * 32;
constexpr int GRP = 128;  // threads of one warp group
constexpr uint32_t T_CB = 0, T_MK = 64, T_S = 128, T_YI = 256, T_YS = 384, T_LAND = 0;
constexpr float kFastSpan = 180.0f;
constexpr float kMaxExp = 96.0f;
constexpr float kLog2e = 1.4426950408889634f;
// ring polling: rounds of loads with a short sleep between them (about a second)
constexpr uint32_t kPollLimit = 1u << 21;

// workspace header (bytes): status word, abort word, and the first wait that
// gave up (0x10000 | warp << 8 | barrier, or 0x20000 | warp for the ring)
constexpr size_t kHdrAbort = 4, kHdrWhere = 16, kHdrBytes = 256;  // status word at 0

// Optional timeline (builds with -DSSD_TRACE only): one thread of each role
// stamps the global timer at its hand-offs of the first heads of each CTA,
// read back with ssd_fused_trace_copy().  Events per head: 0 decays in;
// 1 x pass starts, 2 x~ ready, 3 mask starts, 4 mask ready; 5 tile-state MMA
// and 6 intra MMA issued; 7 tile state in, 8 prefix in, 9 prefix sent (or
// aggregate formed), 10 entering state in, 11 state operand ready; 12 state
// MMA issued; 13 epilogue starts, 14 y stored; 15 x load issued.
#ifdef SSD_TRACE
constexpr int kTraceCtas = 160, kTraceHeads = 24, kTraceEv = 16;
__device__ long long g_fused_trace[kTraceCtas][kTraceHeads * kTraceEv];
#define FTRACE(h, ev)                                                                        \
    do {                                                                                     \
        if (blockIdx.x < kTraceCtas && (h) < kTraceHeads) {                                  \
            long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                           \
            g_fused_trace[blockIdx.x][(h) * kTraceEv + (ev)] = t_;                           \
        }                                                                                    \
    } while (0)
#else
#define FTRACE(h, ev) \
    do {              \
    } while (0)
#endif

template <int NST>
struct FSmem {
    static constexpr int KBLK = TL * 128;      // 128 rows x 128 bytes
    static constexpr int NKB = NST / 64;
    static constexpr int C_OFF = 0;                   // two C slots (one per item in flight)
    static constexpr int C_SLOT = NKB * KBLK;
    static constexpr int B_OFF = C_OFF + 2 * C_SLOT;
    // dstate 64: a zero block right after B is the second 64-row half of the
    // tile-state MMA's A operand (M = 128 state rows, the upper 64 all zero)
    static constexpr int Z_OFF = B_OFF + NKB * KBLK;
    static constexpr int Z_BYTES = NST == 64 ? KBLK : 0;
    static constexpr int XR_OFF = Z_OFF + Z_BYTES;   // two x slots (raw, then fp16 in place)
    static constexpr int XT_OFF = XR_OFF + 2 * KBLK;  // state-weighted x (bf16)
    static constexpr int H2_OFF = XT_OFF + KBLK;      // entering state: bf16 hi rows, then lo rows
    static constexpr int H_LO = NST * 128;
    static constexpr int ST_BYTES = NST * PD * 4;     // one fp32 state
    // the prefix slot (from rank k-1): the state, then its log2 decay (16 bytes)
    static constexpr int PB_OFF = H2_OFF + 2 * H_LO;
    static constexpr int PB_BYTES = ST_BYTES + 16;
    // per head, four buffers: [cum2 | dt | state weight | epilogue row factor] x TL, D, c_end
    static constexpr int DEC_FLOATS = 4 * TL + 8;
    static constexpr int DEC_OFF = PB_OFF + PB_BYTES;
    static constexpr int XSC_OFF = DEC_OFF + 4 * DEC_FLOATS * 4;  // [2][TL] 1 / (fp16 scale of x)
    static constexpr int DMW_OFF = XSC_OFF + 2 * TL * 4;          // [2][4] per-warp max dt / s
    static constexpr int BNW_OFF = DMW_OFF + 8 * 4;               // [2][4] per-warp max |B_j|^2
    static constexpr int CTAB_OFF = BNW_OFF + 8 * 4;              // [4][32] column factors
    static constexpr int ALP_OFF = CTAB_OFF + 4 * 32 * 4;         // [2] log2 decay before this tile
    static constexpr int BAR_OFF = ALP_OFF + 16;
    static constexpr int SMEM = BAR_OFF + 48 * 8 + 64 + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(XR_OFF % 1024 == 0 && XT_OFF % 1024 == 0 && H2_OFF % 1024 == 0, "operand alignment");
};

enum : int {
    B_C_FULL = 0, B_B_FULL = B_C_FULL + 2, B_CB_DONE, B_X_FULL, B_X_FREE = B_X_FULL + 2,
    B_XT_FULL = B_X_FREE + 2, B_XT_FREE,
    B_S_FULL, B_S_FREE = B_S_FULL + 2, B_MK_FULL = B_S_FREE + 2, B_MK_FREE, B_YI_FULL,
    B_H2_FULL = B_YI_FULL + 2, B_H2_FREE, B_YS_FULL, B_ACC_FREE = B_YS_FULL + 2,
    B_DEC_FULL = B_ACC_FREE + 2, B_DEC_FREE = B_DEC_FULL + 4, B_EPF_FULL = B_DEC_FREE + 4,
    B_P_FULL = B_EPF_FULL + 4, B_P_FREE, B_PK_READY, B_C_FREE = B_PK_READY + 2, B_B_FREE = B_C_FREE + 2,
    B_COUNT
};
static_assert(B_COUNT <= 48, "barrier slots");

struct Item {
    int64_t run, b, g, hfirst, t0;
    int Lt;  // valid tokens of this CTA's tile (0 past the end of the sequence)
};

// (32-bit arithmetic: the launcher keeps the item count below 2^31; one
// out-of-line copy, called once per item)
__device__ __noinline__ Item decode_item(const FwdParams& p, int64_t ticket, int hc, int kc, uint32_t rank) {
    const uint32_t nhb = static_cast<uint32_t>(p.heads_per_group) / hc;
    const uint32_t ng = static_cast<uint32_t>(p.ngroups);
    const uint32_t per_run = static_cast<uint32_t>(p.batch) * ng * nhb;
    const uint32_t t = static_cast<uint32_t>(ticket);
    Item it;
    it.run = t / per_run;
    uint32_t r = t - static_cast<uint32_t>(it.run) * per_run;
    const uint32_t b = r / (ng * nhb);
    r -= b * (ng * nhb);
    const uint32_t g = r / nhb;
    it.b = b;
    it.g = g;
    it.hfirst = static_cast<int64_t>(g) * p.heads_per_group + static_cast<int64_t>(r - g * nhb) * hc;
    it.t0 = (it.run * kc + rank) * TL;
    const int64_t left = p.seqlen - it.t0;
    it.Lt = static_cast<int>(left <= 0 ? 0 : (left < TL ? left : TL));
    return it;
}

// ---------------------------------------------------------------- cluster ops
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_peer_v4(uint32_t a, float x, float y, float z, float w) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z),
                 "f"(w)
                 : "memory");
}
__device__ __forceinline__ void st_peer_f32(uint32_t a, float x) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(x) : "memory");
}
// arrive on a peer CTA's mbarrier, releasing this thread's prior writes at cluster scope
__device__ __forceinline__ void arrive_peer(uint32_t a) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}
// probe of a local mbarrier whose arrivals come from peers (acquire at cluster scope)
__device__ __forceinline__ bool try_wait_cluster(uint32_t mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(mbar), "r"(parity), "r"(100)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait that gives up when this CTA or any CTA of the call aborted.  The
// first probe is inline; the waiting loop is one out-of-line copy (the kernel's
// roles share an instruction cache, and dozens of inlined loops crowd it).
__device__ __noinline__ bool wait_bar_slow(uint32_t mbar, uint32_t parity, volatile int* abort,
                                           const int* g_abort, bool cluster) {
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (cluster ? try_wait_cluster(mbar, parity) : mbar_try_wait_hint(mbar, parity, 100)) return true;
        if ((i & 63) == 63 && (*abort || ((i & 1023) == 1023 && ld_acquire(g_abort)))) return false;
    }
    *abort = 1;
    return false;
}
template <bool CLUSTER>
__device__ __forceinline__ bool wait_bar(uint32_t mbar, uint32_t parity, volatile int* abort,
                                         const int* g_abort) {
    if (mbar_test_wait(mbar, parity)) return true;
    return wait_bar_slow(mbar, parity, abort, g_abort, CLUSTER);
}

__device__ __forceinline__ void raise_abort(volatile int* abort, int* g_abort) {
    *abort = 1;
    atomicExch(g_abort, 1);
}

// named barrier over one warp group that also ANDs a predicate across it
__device__ __forceinline__ bool group_sync_and(uint32_t id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "r"(id), "r"(GRP)
        : "memory");
    return r != 0;
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

// One row of the mask: this lane's row l of the 32-row block q of the tile.
struct RowPlan {
    float ref, cl, c_first;
    float f;     // epilogue row factor of the intra term
    float rs;    // the row's power-of-two scale into fp16 range
    float dtl;   // dt_l
    float dadd;  // D / rinv_l * rs_l (the skip term, in the mask's units)
    float de;    // 2^{ref - c_l} / s_l (fast) or 1 / s_l (steep): the diagonal's decay factor
    bool fast;   // factored decays (warp-uniform)
};

// The mask row l holds m[l,j] = CBp[l,j] * k_j * rs_l in fp16, CBp the packed
// CB (|CBp| < 2^14, CB = rinv_l CBp), k_j = 2^{ref - c_j} dt_j / s_j (fast) or
// 2^{c_l - c_j} dt_j / s_j (steep), and on the diagonal
// (CBp[l,l] dt_l + D / rinv_l) 2^{ref - c_l} / s_l * rs_l.  For j <= l,
// c_j >= c_l, so |m[l,j]| <= 2^{ref - c_l} (2^14 dmax + |D| / (rinv_l s_l)) rs_l
// with dmax = max_j dt_j / s_j over the tile (2^0 in place of 2^{ref - c_l}
// when steep); rs_l brings that bound to 2^15 (fp16 holds 65504), so no
// element overflows and the row's largest elements keep all 11 bits.
__device__ __forceinline__ RowPlan plan_row(int q, int lane, const float* cum2, const float* dtv, float rinv,
                                            float Dh, int Lt, float dmax, float xs) {
    RowPlan r;
    const int lb = 32 * q;
    const int last = max(lb, min(lb + 31, Lt - 1));
    r.c_first = cum2[lb];
    const float c_last = cum2[last];
    r.fast = (r.c_first - c_last) <= kFastSpan;
    r.ref = r.fast ? 0.5f * (r.c_first + c_last) : r.c_first;
    r.cl = cum2[lb + lane];
    const float irinv = __int_as_float(254 * (1 << 23) - __float_as_int(rinv));  // 1 / rinv (a power of 2)
    const float lg = (r.fast ? r.ref - r.cl : 0.0f) +
                     __log2f(fmaxf(16384.0f * dmax + fabsf(Dh) * irinv * xs, 1e-30f));
    const int e = min(120, max(-120, 15 - static_cast<int>(ceilf(fminf(fmaxf(lg, -200.0f), 200.0f)))));
    r.rs = __int_as_float((127 + e) << 23);
    const float irs = __int_as_float((127 - e) << 23);
    r.f = (r.fast ? rinv * ex2(r.cl - r.ref) : rinv) * irs;
    r.dtl = dtv[lb + lane];
    r.dadd = Dh * irinv * r.rs;
    r.de = (r.fast ? ex2(r.ref - r.cl) : 1.0f) * xs;
    return r;
}

// Column group g (32 columns) of this warp's mask rows (block q): CB (packed
// fp16 in TMEM) times the decays and the row scale, to fp16, into the mask
// columns in TMEM.  xsc holds 1 / (fp16 scale of x) per token.
__device__ __forceinline__ void mask_group(const RowPlan& r, int q, int g, uint32_t cb_addr, uint32_t mk_addr,
                                           const float* cum2, const float* dtv, const float* xsc, float* ctab,
                                           int lane) {
    uint32_t raw[16];
    tmem_ld16(cb_addr, raw);
    const int j0 = 32 * g;
    const float cj = ex2(fminf(r.ref - cum2[j0 + lane], kMaxExp)) * dtv[j0 + lane] * xsc[j0 + lane];
    uint32_t o[16];
    __syncwarp();
    ctab[lane] = cj;
    __syncwarp();
    const float4* ct = reinterpret_cast<const float4*>(ctab);
    const float2 rs2 = make_float2(r.rs, r.rs);
    if (g < q && r.fast) {  // below the diagonal block: packed fp32x2 products
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
    if (g < q) {  // below the diagonal block of a steep row block
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
                const int k = 4 * i + e;
                float m = v[k] * cc[e];
                if (k == lane) m = fmaf(v[k], r.dtl, r.dadd) * r.de;
                v[k] = (k <= lane) ? m : 0.0f;
            }
        }
    } else {  // the diagonal block of a steep row block: one exp2 per element
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            float m = v[k] * ex2(fminf(r.cl - cum2[j0 + k], 0.0f)) * dtv[j0 + k] * xsc[j0 + k];
            if (k == lane) m = fmaf(v[k], r.dtl, r.dadd) * r.de;
            v[k] = (k <= lane) ? m : 0.0f;
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

// 16 entries (p = 16 sl ..) of state row n as the MN-major B operand of the
// state term (row n = K index, 64 p per 128-byte row): hi rows, then lo rows.
__device__ __forceinline__ void stage_slice(uint32_t sH2, uint32_t lo_off, int n, int sl, const float (&v)[16]) {
    uint32_t hi[8], lo[8];
    split_hi_lo(v, hi, lo);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t c = 2 * sl + k;
        st_shared_v4(sH2 + sw128(n, c), hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
        st_shared_v4(sH2 + lo_off + sw128(n, c), lo[4 * k], lo[4 * k + 1], lo[4 * k + 2], lo[4 * k + 3]);
    }
}

template <int NST, bool GATED>
__global__ void __launch_bounds__(512, 1)
    fused_fwd_kernel(const __grid_constant__ FwdParams p, const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_x,
                     int hc, int kc, int64_t total_items, int64_t nruns, uint64_t* ring, int64_t withhold) {
    using T = FSmem<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 48);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    char* hdr = static_cast<char*>(static_cast<void*>(p.status));
    int* g_abort = reinterpret_cast<int*>(hdr + kHdrAbort);
    int* g_where = reinterpret_cast<int*>(hdr + kHdrWhere);
    // bounded waits; the first one in the call that gives up is recorded
    auto wb = [&](int i, uint32_t parity) {
        const bool r = wait_bar<false>(bar(i), parity, abort, g_abort);
        if (!r) atomicCAS(g_where, 0, 0x10000 | ((threadIdx.x >> 5) << 8) | i);
        return r;
    };
    auto wbc = [&](int i, uint32_t parity) {  // arrivals from peer CTAs
        const bool r = wait_bar<true>(bar(i), parity, abort, g_abort);
        if (!r) atomicCAS(g_where, 0, 0x10000 | ((threadIdx.x >> 5) << 8) | i);
        return r;
    };
    // warp-uniform outcome (the tcgen05 loads and stores that follow are warp-collective)
    auto uni = [](bool ok) { return __all_sync(0xffffffffu, ok); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const int64_t cid = cluster_index(), ncl = cluster_count();
    const int64_t H = p.nheads, L = p.seqlen, Bsz = p.batch;
    const uint32_t sC = smem_u32(smem + T::C_OFF), sB = smem_u32(smem + T::B_OFF);
    const uint32_t sXR = smem_u32(smem + T::XR_OFF), sXT = smem_u32(smem + T::XT_OFF);
    const uint32_t sH2 = smem_u32(smem + T::H2_OFF);
    constexpr uint32_t KB = T::KBLK;
    constexpr int64_t kWordsPerState = PD * NST / 2;
    const int64_t n_items = cid < total_items ? (total_items - cid + ncl - 1) / ncl : 0;
    const int last_rank = kc - 1;

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) {
            uint32_t count = 1;
            if (i == B_XT_FULL || i == B_S_FREE || i == B_S_FREE + 1 || i == B_MK_FULL || i == B_H2_FULL ||
                i == B_ACC_FREE || i == B_ACC_FREE + 1 || (i >= B_EPF_FULL && i < B_EPF_FULL + 4) ||
                i == B_P_FULL || i == B_P_FREE || i == B_PK_READY || i == B_PK_READY + 1)
                count = GRP;
            if (i >= B_DEC_FULL && i < B_DEC_FULL + 4) count = 32;
            if (i >= B_DEC_FREE && i < B_DEC_FREE + 4) count = 3 * GRP;
            mbar_init(bar(i), count);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (NST == 64) {  // the zero half of the tile-state A operand
        uint32_t* z = reinterpret_cast<uint32_t*>(smem + T::Z_OFF);
        for (int i = tid; i < T::Z_BYTES / 4; i += NTHREADS) z[i] = 0u;
        fence_smem_async();
    }
    fence_before_sync();
    __syncthreads();
    cluster_sync_all();  // every CTA's barriers exist before any peer arrives on them
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    auto dec_ptr = [&](int s) { return reinterpret_cast<float*>(smem + T::DEC_OFF) + s * T::DEC_FLOATS; };

    if (warp == CTRL_WARP) {
        // ------------------------------ control ------------------------------
        if (lane == 0) {
            tma_prefetch_map(&tm_c);
            tma_prefetch_map(&tm_b);
            tma_prefetch_map(&tm_x);
            bool ok = true, cb_pending = false;
            int64_t x_next = 0, i_done = -1, x_item = -1;
            Item xit = decode_item(p, cid, hc, kc, rank);
            const int64_t heads_total = n_items * hc;
            // x of every head up to `upto` in flight (two slots)
            auto issue_x = [&](int64_t upto) {
                for (; ok && x_next <= upto && x_next < heads_total; ++x_next) {
                    const int s2 = static_cast<int>(x_next & 1);
                    if (x_next >= 2) {
                        ok = wb(B_X_FREE + s2, ((x_next - 2) >> 1) & 1);
                        if (!ok) break;
                    }
                    const uint32_t xi = static_cast<uint32_t>(x_next) / hc;
                    if (xi != static_cast<uint32_t>(x_item)) {
                        x_item = xi;
                        xit = decode_item(p, cid + xi * ncl, hc, kc, rank);
                    }
                    mbar_expect_tx(bar(B_X_FULL + s2), KB);
                    tma_load_4d(sXR + s2 * KB, &tm_x, bar(B_X_FULL + s2), 0,
                                static_cast<int>(xit.hfirst + (static_cast<uint32_t>(x_next) - xi * hc)),
                                static_cast<int>(xit.t0), static_cast<int>(xit.b));
                    FTRACE(x_next, 15);
                }
            };
            for (int64_t i = 0; ok && i < n_items; ++i) {
                const Item it = decode_item(p, cid + i * ncl, hc, kc, rank);
                const int64_t hbase = i * hc;
                const int cs = static_cast<int>(i & 1);
                const uint32_t sCi = sC + cs * T::C_SLOT;
                // B is reused once the previous item's tile-state MMAs are done; C has
                // two slots, the state-term MMAs of the item before that being the
                // only ones that wait on the chain
                if (i > 0) ok = wb(B_B_FREE, (i - 1) & 1);
                if (ok && i > 1) ok = wb(B_C_FREE + cs, ((i - 2) >> 1) & 1);
                if (!ok) break;
                mbar_expect_tx(bar(B_C_FULL + cs), T::NKB * KB);
                mbar_expect_tx(bar(B_B_FULL), T::NKB * KB);
                for (int kb = 0; kb < T::NKB; ++kb) {
                    tma_load_4d(sCi + kb * KB, &tm_c, bar(B_C_FULL + cs), kb * 64, static_cast<int>(it.g),
                                static_cast<int>(it.t0), static_cast<int>(it.b));
                    tma_load_4d(sB + kb * KB, &tm_b, bar(B_B_FULL), kb * 64, static_cast<int>(it.g),
                                static_cast<int>(it.t0), static_cast<int>(it.b));
                }
                cb_pending = true;
                issue_x(hbase + 1);
                if (!ok) break;
                if (i + 1 < n_items) {  // the next item's C and B into L2
                    const Item nx = decode_item(p, cid + (i + 1) * ncl, hc, kc, rank);
                    for (int kb = 0; kb < T::NKB; ++kb) {
                        tma_prefetch_l2_4d(&tm_c, kb * 64, static_cast<int>(nx.g), static_cast<int>(nx.t0),
                                           static_cast<int>(nx.b));
                        tma_prefetch_l2_4d(&tm_b, kb * 64, static_cast<int>(nx.g), static_cast<int>(nx.t0),
                                           static_cast<int>(nx.b));
                    }
                }
                ok = wb(B_C_FULL + cs, (i >> 1) & 1) && wb(B_B_FULL, i & 1);
                if (!ok) break;
                cb_pending = false;
                // the landing columns are free once the previous head's intra MMA is done
                if (hbase > 0) {
                    ok = wb(B_MK_FREE, (hbase - 1) & 1);
                    if (!ok) break;
                }
                fence_after_sync();
                {
                    const uint32_t id = idesc_bf16(128, 128, false, false);
                    for (int k = 0; k < NST / 16; ++k) {
                        const uint32_t ko = (k >> 2) * KB + (k & 3) * 32;
                        mma_bf16(tmem + T_LAND, desc_sw128(sCi + ko, 16, 1024), desc_sw128(sB + ko, 16, 1024), id,
                                 k > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar(B_CB_DONE));
                for (int j = 0; ok && j < hc; ++j) {
                    const int64_t h = hbase + j;
                    const int s = static_cast<int>(h & 1);
                    issue_x(h + 1);
                    if (!ok) break;
                    // tile state S = B^T (w x): A = B (MN-major, M = states), B operand = x~ (MN-major)
                    ok = wb(B_XT_FULL, h & 1);
                    if (ok && h >= 2) ok = wb(B_S_FREE + s, ((h - 2) >> 1) & 1);
                    if (!ok) break;
                    fence_after_sync();
                    {
                        const uint32_t id = idesc_bf16(128, PD, true, true);
                        for (int k = 0; k < 8; ++k)
                            mma_bf16(tmem + T_S + 64 * s, desc_sw128(sB + k * 2048, KB, 1024),
                                     desc_sw128(sXT + k * 2048, KB, 1024), id, k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_S_FULL + s));
                    mma_commit(bar(B_XT_FREE));
                    FTRACE(h, 5);
                    // intra terms: A = the mask in TMEM (fp16), B = x (fp16, MN-major)
                    ok = wb(B_MK_FULL, h & 1);
                    if (ok && h >= 2) ok = wb(B_ACC_FREE + s, ((h - 2) >> 1) & 1);
                    if (!ok) break;
                    fence_after_sync();
                    {
                        const uint32_t id = idesc_f16(128, PD, false, true);
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + T_YI + 64 * s, tmem + T_MK + 8 * k,
                                   desc_sw128(sXR + s * KB + k * 2048, KB, 1024), id, k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_MK_FREE));
                    mma_commit(bar(B_X_FREE + s));
                    mma_commit(bar(B_YI_FULL + s));
                    FTRACE(h, 6);
                }
                if (ok) mma_commit(bar(B_B_FREE));
                i_done = i;
            }
            if (!ok) raise_abort(abort, g_abort);
            // no copy may land after the CTA is gone: wait (bounded) for every load in flight
            if (cb_pending) {
                const int64_t i2 = i_done + 1;
                wait_bar<false>(bar(B_C_FULL + (i2 & 1)), (i2 >> 1) & 1, abort, g_abort);
                wait_bar<false>(bar(B_B_FULL), i2 & 1, abort, g_abort);
            }
            for (int64_t g2 = x_next - 2 < 0 ? 0 : x_next - 2; g2 < x_next; ++g2)
                wait_bar<false>(bar(B_X_FULL + (g2 & 1)), (g2 >> 1) & 1, abort, g_abort);
        }
    } else if (warp == HCTRL_WARP) {
        // --------------------------- state-term issuer ---------------------------
        if (lane == 0) {
            bool ok = true;
            for (int64_t i = 0; ok && i < n_items; ++i) {
                const int cs = static_cast<int>(i & 1);
                const uint32_t sCi = sC + cs * T::C_SLOT;
                ok = wb(B_C_FULL + cs, (i >> 1) & 1);  // C is in
                for (int j = 0; ok && j < hc; ++j) {
                    const int64_t h = i * hc + j;
                    const int s = static_cast<int>(h & 1);
                    ok = wb(B_H2_FULL, h & 1);
                    if (ok && h >= 2) ok = wb(B_ACC_FREE + s, ((h - 2) >> 1) & 1);
                    if (!ok) break;
                    fence_after_sync();
                    // C (H^hi + H^lo): A = C (K-major), B = H (MN-major)
                    const uint32_t id = idesc_bf16(128, PD, false, true);
                    for (int part = 0; part < 2; ++part)
                        for (int k = 0; k < NST / 16; ++k) {
                            const uint32_t ko = (k >> 2) * KB + (k & 3) * 32;
                            mma_bf16(tmem + T_YS + 64 * s, desc_sw128(sCi + ko, 16, 1024),
                                     desc_sw128(sH2 + part * T::H_LO + k * 2048, KB, 1024), id,
                                     (part | k) ? 1u : 0u);
                        }
                    mma_commit(bar(B_H2_FREE));
                    mma_commit(bar(B_YS_FULL + s));
                    FTRACE(h, 12);
                }
                if (ok) mma_commit(bar(B_C_FREE + cs));
            }
            if (!ok) raise_abort(abort, g_abort);
        }
    } else if (warp == LOAD_WARP) {
        // ------------------------------- loader ------------------------------
        // dt = softplus(dt_raw + dt_bias), log2(e) times the inclusive in-tile
        // cumulative sum of dt * A, and the tile-state weights 2^{c_end - c_l} dt_l
        // of each head.  Slots past the tile's last token hold dt = 0 and the
        // last cumulative value.
        bool ok = true;
        const __nv_bfloat16* dtr = static_cast<const __nv_bfloat16*>(p.dt_raw);
        for (int64_t i = 0; ok && i < n_items; ++i) {
            const Item it = decode_item(p, cid + i * ncl, hc, kc, rank);
            for (int j = 0; ok && j < hc; ++j) {
                const int64_t h = i * hc + j;
                const int d4 = static_cast<int>(h & 3);  // decays: four buffers
                if (h >= 4) ok = uni(wb(B_DEC_FREE + d4, ((h - 4) >> 2) & 1));
                if (!ok) break;
                const int64_t hh = it.hfirst + j;
                const float A = p.A[hh], bias = p.dt_bias ? p.dt_bias[hh] : 0.0f;
                float u[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int l = 32 * k + lane;
                    u[k] = l < it.Lt ? __bfloat162float(dtr[((it.b * L) + it.t0 + l) * H + hh]) : 0.0f;
                }
                float* dec = dec_ptr(d4);
                float carry = 0.0f, cv[4], dv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int l = 32 * k + lane;
                    float dt = 0.0f, v = 0.0f;
                    if (l < it.Lt) {
                        dt = softplus_f32(u[k] + bias);
                        v = dt * A;
                    }
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float n = __shfl_up_sync(0xffffffffu, v, o);
                        if (lane >= o) v += n;
                    }
                    v += carry;
                    carry = __shfl_sync(0xffffffffu, v, 31);
                    cv[k] = v * kLog2e;
                    dv[k] = dt;
                }
                const float cend = __shfl_sync(0xffffffffu, cv[3], 31);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int l = 32 * k + lane;
                    dec[l] = cv[k];
                    dec[TL + l] = dv[k];
                    dec[2 * TL + l] = ex2(cend - cv[k]) * dv[k];
                }
                if (lane == 0) {
                    dec[4 * TL] = p.D ? p.D[hh] : 0.0f;
                    dec[4 * TL + 1] = cend;
                }
                mbar_arrive(bar(B_DEC_FULL + d4));
                if (lane == 0) FTRACE(h, 0);
            }
        }
        if (!ok) raise_abort(abort, g_abort);
    } else if (warp < CARRY_W0) {
        // ------------------------------ mask group ------------------------------
        // warp q: TMEM lanes (tile rows) 32 q .. 32 q + 31, mask column groups 0..q
        const int q = warp;
        const int l = 32 * q + lane;
        const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
        float* ctab = reinterpret_cast<float*>(smem + T::CTAB_OFF) + 32 * q;
        float* bnw = reinterpret_cast<float*>(smem + T::BNW_OFF);
        float* dmw = reinterpret_cast<float*>(smem + T::DMW_OFF);
        // Every decision to stop is taken together by the whole group (a
        // named barrier that ANDs the outcome), so no warp is ever left
        // waiting at a barrier the others have abandoned.
        bool ok = true;
        for (int64_t i = 0; i < n_items; ++i) {
            ok = group_sync_and(1, ok);
            if (!ok) break;
            const Item it = decode_item(p, cid + i * ncl, hc, kc, rank);
            // --- CB repack: fp32 landing -> fp16 pairs with a power-of-two
            // scale per row, chosen from |C_l . B_j| <= |C_l| max_j |B_j|
            ok = uni(wb(B_C_FULL + (i & 1), (i >> 1) & 1) && wb(B_B_FULL, i & 1));
            const uint32_t sCi = sC + static_cast<uint32_t>(i & 1) * T::C_SLOT;
            float csq = 0.0f, bsq = 0.0f;
            if (ok) {
#pragma unroll
                for (int kb = 0; kb < T::NKB; ++kb)
#pragma unroll
                    for (int c16 = 0; c16 < 8; ++c16) {
                        const uint32_t o = l * 128 + kb * KB + ((c16 + lane) & 7) * 16;
                        const uint4 vc = ld_shared_v4(sCi + o), vb = ld_shared_v4(sB + o);
                        const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wbv[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wc[e]));
                            const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wbv[e]));
                            csq = fmaf(f.x, f.x, fmaf(f.y, f.y, csq));
                            bsq = fmaf(g2.x, g2.x, fmaf(g2.y, g2.y, bsq));
                        }
                    }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) bsq = fmaxf(bsq, __shfl_xor_sync(0xffffffffu, bsq, o));
                if (lane == 0) bnw[4 * (i & 1) + q] = bsq;
            }
            ok = group_sync_and(1, ok);
            if (!ok) break;
            const float bmax = fmaxf(fmaxf(bnw[4 * (i & 1)], bnw[4 * (i & 1) + 1]),
                                     fmaxf(bnw[4 * (i & 1) + 2], bnw[4 * (i & 1) + 3]));
            const float bound = sqrtf(csq * bmax);
            const int e2 = max(0, ((__float_as_int(bound) >> 23) & 255) - 127 - 13 + 1);
            const float sc_row = __int_as_float((127 - e2) << 23);
            const float rinv = __int_as_float((127 + e2) << 23);
            ok = uni(wb(B_CB_DONE, i & 1));
            if (ok) {
                fence_after_sync();
                // causal groups 0..q of row l (in place: group g reads fp32 columns
                // [32g, 32g+32) and writes packed columns [16g, 16g+16), already read)
                for (int g = 0; g <= q; ++g) {
                    float v[32];
                    tmem_ld32(tmem + lanes + T_LAND + 32 * g, v);
                    uint32_t r16[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) r16[k] = pack_f16x2(v[2 * k] * sc_row, v[2 * k + 1] * sc_row);
                    tmem_st16(tmem + lanes + T_CB + 16 * g, r16);
                }
                // above the diagonal the mask is zero for every head of the item
                const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                for (int g = q + 1; g < 4; ++g) tmem_st16(tmem + lanes + T_MK + 16 * g, z);
                tmem_wait_st();
            }

            for (int j = 0; j < hc; ++j) {
                const int64_t h = i * hc + j;
                const int s = static_cast<int>(h & 1);
                const int d4 = static_cast<int>(h & 3);
                if (ok) {
                    ok = wb(B_DEC_FULL + d4, (h >> 2) & 1);
                    ok = ok && wb(B_X_FULL + s, (h >> 1) & 1);
                    if (ok && h > 0) ok = wb(B_XT_FREE, (h - 1) & 1);
                    ok = uni(ok);
                }
                float* dec = dec_ptr(d4);
                const float* cum2 = dec;
                const float* dtv = dec + TL;
                const float* wst = dec + 2 * TL;
                float* xsc = reinterpret_cast<float*>(smem + T::XSC_OFF) + s * TL;
                const uint32_t xr = sXR + s * KB;
                if (tid == 0) FTRACE(h, 1);
                if (ok) {
                    // --- x: state-weighted bf16 copy into XT, and x itself as fp16
                    // in place for the intra MMA.  Lane = row (this warp's 32 rows):
                    // the row's power-of-two scale s_l takes its largest |x| to
                    // [2^13, 2^14) (bf16 values are exact in fp16 there).  With the
                    // 128-byte swizzle the 32 rows' chunk c fall on distinct bank
                    // groups 8 rows at a time, so each 16-byte access is conflict-free.
                    const int r = l;
                    const float w = wst[r];
                    uint4 v[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) v[c] = ld_shared_v4(xr + sw128(r, c));
                    // max |x| as bf16 bit patterns (sign cleared; the order of
                    // non-negative floats is that of their bits): both halves at
                    // once, eight independent partial maxima
                    uint32_t m8[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        m8[c] = __vmaxu2(__vmaxu2(v[c].x & 0x7FFF7FFFu, v[c].y & 0x7FFF7FFFu),
                                         __vmaxu2(v[c].z & 0x7FFF7FFFu, v[c].w & 0x7FFF7FFFu));
#pragma unroll
                    for (int c = 0; c < 4; ++c) m8[c] = __vmaxu2(m8[c], m8[c + 4]);
                    const uint32_t m2 = __vmaxu2(__vmaxu2(m8[0], m8[1]), __vmaxu2(m8[2], m8[3]));
                    const uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
                    // bf16 bits -> exponent (values are finite bf16 inputs)
                    const int ex = am ? static_cast<int>((am >> 7) & 255) - 127 : 0;
                    const int es = min(100, max(-100, 13 - ex));  // s = 2^es
                    const float scx = __int_as_float((127 + es) << 23);
                    const float2 w2 = make_float2(w, w), sc2 = make_float2(scx, scx);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t e4[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
                        uint32_t ot[4], oh[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e4[e]));
                            const float2 t = __fmul2_rn(f, w2);
                            const float2 hh2 = __fmul2_rn(f, sc2);
                            ot[e] = pack_bf16x2(t.x, t.y);
                            oh[e] = pack_f16x2(hh2.x, hh2.y);
                        }
                        const uint32_t off = sw128(r, c);
                        st_shared_v4(sXT + off, ot[0], ot[1], ot[2], ot[3]);
                        st_shared_v4(xr + off, oh[0], oh[1], oh[2], oh[3]);
                    }
                    const float inv = __int_as_float((127 - es) << 23);
                    xsc[r] = inv;
                    float dloc = dtv[r] * inv;
                    fence_smem_async();
                    mbar_arrive(bar(B_XT_FULL));
                    if (tid == 0) FTRACE(h, 2);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) dloc = fmaxf(dloc, __shfl_xor_sync(0xffffffffu, dloc, o));
                    if (lane == 0) dmw[4 * s + q] = dloc;
                }
                ok = group_sync_and(2, ok);  // every row's scale and the bound are in
                if (!ok) break;
                if (h > 0) ok = uni(wb(B_MK_FREE, (h - 1) & 1));
                if (ok) {
                    if (tid == 0) FTRACE(h, 3);
                    fence_after_sync();
                    const float dmax =
                        fmaxf(fmaxf(dmw[4 * s], dmw[4 * s + 1]), fmaxf(dmw[4 * s + 2], dmw[4 * s + 3]));
                    // --- this head's mask rows into TMEM
                    const RowPlan rp = plan_row(q, lane, cum2, dtv, rinv, dec[4 * TL], it.Lt, dmax, xsc[l]);
                    for (int g = 0; g <= q; ++g)
                        mask_group(rp, q, g, tmem + lanes + T_CB + 16 * g, tmem + lanes + T_MK + 16 * g, cum2,
                                   dtv, xsc, ctab, lane);
                    dec[3 * TL + l] = rp.f;
                    tmem_wait_st();
                    fence_before_sync();
                    mbar_arrive(bar(B_MK_FULL));
                    mbar_arrive(bar(B_EPF_FULL + d4));
                    mbar_arrive(bar(B_DEC_FREE + d4));
                    if (tid == 0) FTRACE(h, 4);
                }
            }
            if (!ok) break;
        }
        if (!ok) raise_abort(abort, g_abort);
    } else if (warp < EPI_W0) {
        // ------------------------------ carry group -----------------------------
        // thread n: state row n, all 64 p.  Per head: the run's entering state
        // H_in from the ring (or the initial state), this tile's entering state
        // H_k = 2^{log A_<k} H_in + P_k staged as the state-term operand; the last
        // rank also publishes H_out = 2^{c_end} H_k + S_k.  P_k is zero on rank 0,
        // in the tile state's TMEM columns on the middle ranks (put there by the
        // prefix step), and on the last rank in the operand rows as bf16 hi + lo
        // (parked there from the prefix slot first, so the slot frees at once).
        const int qd = warp - CARRY_W0;
        const int n = 32 * qd + lane;
        const bool has_state = n < NST;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        const bool last = static_cast<int>(rank) == last_rank;
        int* cnt = reinterpret_cast<int*>(hdr + kHdrBytes);  // [2][batch][nheads] reader counts
        const int64_t heads_total = n_items * hc;
        const volatile float* alp = reinterpret_cast<const volatile float*>(smem + T::ALP_OFF);
        const uint32_t pb = smem_u32(smem + T::PB_OFF);
        bool ok = true;
        Item it = decode_item(p, cid, hc, kc, rank);
        int j = 0;  // head of the item
        for (int64_t h = 0; ok && h < heads_total; ++h, ++j) {
            const int s = static_cast<int>(h & 1), d4 = static_cast<int>(h & 3);
            if (j == hc) {
                j = 0;
                it = decode_item(p, cid + (static_cast<uint32_t>(h) / static_cast<uint32_t>(hc)) * ncl, hc, kc, rank);
            }
            const int64_t hh = it.hfirst + j;
            bool r = wb(B_DEC_FULL + d4, (h >> 2) & 1);
            if (r && h > 0) r = wb(B_H2_FREE, (h - 1) & 1);  // the operand rows are free
            if (r && last) r = wb(B_S_FULL + s, (h >> 1) & 1);
            if (r && !last && rank > 0) r = wb(B_PK_READY + s, (h >> 1) & 1);
            r = uni(r);
            if (r && last && rank > 0) r = uni(wbc(B_P_FULL, h & 1));
            if (!r) {
                ok = false;
                break;
            }
            fence_after_sync();
            float alog_prev = 0.0f, a = 1.0f;
            if (last) {
                a = ex2(dec_ptr(d4)[4 * TL + 1]);
                if (rank > 0) {
                    alog_prev = *reinterpret_cast<const volatile float*>(smem + T::PB_OFF + T::ST_BYTES);
                    if (has_state)
#pragma unroll 1
                        for (int sl = 0; sl < 4; ++sl) {
                            float v[16];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint4 u = ld_shared_v4(pb + ((4 * sl + k) * NST + n) * 16);
                                v[4 * k] = __uint_as_float(u.x);
                                v[4 * k + 1] = __uint_as_float(u.y);
                                v[4 * k + 2] = __uint_as_float(u.z);
                                v[4 * k + 3] = __uint_as_float(u.w);
                            }
                            stage_slice(sH2, T::H_LO, n, sl, v);
                        }
                    arrive_peer(peer_addr(bar(B_P_FREE), rank - 1));  // the slot is read
                }
            } else if (rank > 0) {
                alog_prev = alp[s];
            }
            if (n == 0) FTRACE(h, 9);
            const float a_prev = ex2(alog_prev);
            const bool first_run = it.run == 0;
            const bool last_run = it.run == nruns - 1;
            const int64_t bh = it.b * H + hh;
            const uint64_t* src = ring + (((it.run - 1) & 1) * Bsz * H + bh) * kWordsPerState + 2 * n;
            const uint64_t tag_in = static_cast<uint64_t>(it.run & 0xFFFF) << 48;
            const float* ip = p.init_state ? p.init_state + bh * PD * NST + n : nullptr;
            uint64_t* dstw = ring + ((it.run & 1) * Bsz * H + bh) * kWordsPerState + 2 * n;
            const uint64_t tag_out = static_cast<uint64_t>((it.run + 1) & 0xFFFF) << 48;
            float* fp = p.final_state ? p.final_state + bh * PD * NST + n : nullptr;
            const bool publish = last && !last_run && it.run != withhold;  // (the test hook withholds one run's)
            uint32_t rounds = 0;
            // the last rank overwrites its ring slot only once every rank that
            // read the slot's previous state (two runs back) has counted itself
            if (publish && has_state && kc > 1 && it.run >= 2 && lane == 0) {
                const int target = 4 * (kc - 1) * static_cast<int>(it.run / 2);
                const int* c = cnt + (it.run & 1) * Bsz * H + bh;
                while (ld_acquire(c) < target) {
                    if (++rounds >= kPollLimit || ((rounds & 31) == 0 && (*abort || ld_acquire(g_abort)))) {
                        r = false;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            // lane 0 polls the first word of the warp's rows until its tag arrives
            if (r && has_state && !first_run && lane == 0) {
                for (;;) {
                    uint64_t w0, w1;
                    ld_u64x2_relaxed(src, w0, w1);
                    if ((w0 & 0xFFFF000000000000ull) == tag_in) break;
                    if (++rounds >= kPollLimit || ((rounds & 31) == 0 && (*abort || ld_acquire(g_abort)))) {
                        r = false;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            r = __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
            if (!r) {
                if (rounds >= kPollLimit) atomicCAS(g_where, 0, 0x20000 | warp);
                ok = false;
                break;
            }
            if (n == 0) FTRACE(h, 10);
#pragma unroll 1
            for (int sl = 0; sl < 4; ++sl) {
                // entering state: word pair k holds p = 4k .. 4k + 3
                float hin[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) hin[k] = 0.0f;
                if (has_state && !first_run) {
                    // the slice's four word pairs in flight at once; the ones still
                    // stale (rare: the writer stored them all together) are re-read
                    uint64_t w[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) ld_u64x2_relaxed(src + 2 * NST * (4 * sl + k), w[2 * k], w[2 * k + 1]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        for (; r;) {
                            if ((w[2 * k] & 0xFFFF000000000000ull) == tag_in &&
                                (w[2 * k + 1] & 0xFFFF000000000000ull) == tag_in)
                                break;
                            if (++rounds >= kPollLimit || ((rounds & 31) == 0 && (*abort || ld_acquire(g_abort)))) {
                                r = false;
                                break;
                            }
                            __nanosleep(32);
                            ld_u64x2_relaxed(src + 2 * NST * (4 * sl + k), w[2 * k], w[2 * k + 1]);
                        }
                        hin[4 * k] = dec24(w[2 * k] & 0xFFFFFFull);
                        hin[4 * k + 1] = dec24((w[2 * k] >> 24) & 0xFFFFFFull);
                        hin[4 * k + 2] = dec24(w[2 * k + 1] & 0xFFFFFFull);
                        hin[4 * k + 3] = dec24((w[2 * k + 1] >> 24) & 0xFFFFFFull);
                    }
                } else if (has_state && ip) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) hin[k] = ip[(16 * sl + k) * NST];
                }
                __syncwarp();
                float pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = 0.0f;
                if (!last && rank > 0) {
                    uint32_t pr[16];
                    tmem_ld16(tmem + lanes + T_S + 64 * s + 16 * sl, pr);
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = __uint_as_float(pr[k]);
                } else if (last && rank > 0 && has_state) {  // back from the parked hi + lo
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const uint4 hv = ld_shared_v4(sH2 + sw128(n, 2 * sl + k));
                        const uint4 lv = ld_shared_v4(sH2 + T::H_LO + sw128(n, 2 * sl + k));
                        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 fh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
                            const float2 fl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[e]));
                            pk[8 * k + 2 * e] = fh.x + fl.x;
                            pk[8 * k + 2 * e + 1] = fh.y + fl.y;
                        }
                    }
                }
                float hk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) hk[k] = fmaf(a_prev, hin[k], pk[k]);
                if (last) {  // the leaving state, published as soon as formed
                    uint32_t sr[16];
                    tmem_ld16(tmem + lanes + T_S + 64 * s + 16 * sl, sr);
                    if (has_state && r) {
                        float ho[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) ho[k] = fmaf(a, hk[k], __uint_as_float(sr[k]));
                        if (last_run) {
                            if (fp)
#pragma unroll
                                for (int k = 0; k < 16; ++k) fp[(16 * sl + k) * NST] = ho[k];
                        } else if (publish) {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint64_t w0 = tag_out | (enc24(ho[4 * k + 1]) & 0xFFFFFFull) << 24 |
                                                    (enc24(ho[4 * k]) & 0xFFFFFFull);
                                const uint64_t w1 = tag_out | (enc24(ho[4 * k + 3]) & 0xFFFFFFull) << 24 |
                                                    (enc24(ho[4 * k + 2]) & 0xFFFFFFull);
                                st_u64x2_relaxed(dstw + 2 * NST * (4 * sl + k), w0, w1);
                            }
                        }
                    }
                }
                if (has_state) stage_slice(sH2, T::H_LO, n, sl, hk);
            }
            if (!uni(r)) {
                if (rounds >= kPollLimit) atomicCAS(g_where, 0, 0x20000 | warp);
                ok = false;
                break;
            }
            // every rank but the last counts its read of the ring slot (so the
            // slot's next writer knows it is free)
            if (!last && !first_run) {
                __syncwarp();
                if (lane == 0) red_release_add(cnt + ((it.run - 1) & 1) * Bsz * H + bh, 1);
            }
            if (rank > 0 || last) {  // (rank 0 before the last frees it in the prefix step)
                fence_before_sync();
                mbar_arrive(bar(B_S_FREE + s));
            }
            fence_smem_async();
            mbar_arrive(bar(B_H2_FULL));
            mbar_arrive(bar(B_DEC_FREE + d4));
            if (n == 0) FTRACE(h, 11);
        }
        if (!ok) raise_abort(abort, g_abort);
    } else {
        // ------------------------------- epilogue -------------------------------
        // thread l: tile row l (TMEM lane l), all 64 p.  On the ranks before the
        // last these warps also run the prefix step one head ahead of the
        // epilogue: P_{k+1} = 2^{c_end} P_k + S_k into rank k+1's slot (thread =
        // state row), and P_k into the tile state's TMEM columns, S_k being done.
        const int qd = warp - EPI_W0;
        const int l = 32 * qd + lane;
        const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
        const bool last = static_cast<int>(rank) == last_rank;
        const bool has_state = l < NST;
        const int64_t heads_total = n_items * hc;
        const __nv_bfloat16* zg = static_cast<const __nv_bfloat16*>(p.z);
        __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
        const uint32_t pb = smem_u32(smem + T::PB_OFF);
        volatile float* alp = reinterpret_cast<volatile float*>(smem + T::ALP_OFF);

        auto prefix = [&](int64_t h) -> bool {
            const int s = static_cast<int>(h & 1), d4 = static_cast<int>(h & 3);
            bool r = wb(B_DEC_FULL + d4, (h >> 2) & 1);
            r = uni(r && wb(B_S_FULL + s, (h >> 1) & 1));
            if (r && rank > 0) r = uni(wbc(B_P_FULL, h & 1));
            if (r && h > 0) r = uni(wbc(B_P_FREE, (h - 1) & 1));  // rank k+1 read its slot
            if (!r) return false;
            fence_after_sync();
            const float cend = dec_ptr(d4)[4 * TL + 1];
            const float a = ex2(cend);
            const float alog_prev =
                rank > 0 ? *reinterpret_cast<const volatile float*>(smem + T::PB_OFF + T::ST_BYTES) : 0.0f;
            if (l == 0) FTRACE(h, 8);
            const uint32_t dst = peer_addr(pb, rank + 1);
#pragma unroll 1
            for (int sl = 0; sl < 4; ++sl) {
                uint32_t sr[16];
                tmem_ld16(tmem + lanes + T_S + 64 * s + 16 * sl, sr);
                uint32_t pv[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t off = ((4 * sl + k) * NST + l) * 16;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (rank > 0 && has_state) v = ld_shared_v4(pb + off);
                    pv[4 * k] = v.x;
                    pv[4 * k + 1] = v.y;
                    pv[4 * k + 2] = v.z;
                    pv[4 * k + 3] = v.w;
                    if (has_state)
                        st_peer_v4(dst + off, fmaf(a, __uint_as_float(v.x), __uint_as_float(sr[4 * k])),
                                   fmaf(a, __uint_as_float(v.y), __uint_as_float(sr[4 * k + 1])),
                                   fmaf(a, __uint_as_float(v.z), __uint_as_float(sr[4 * k + 2])),
                                   fmaf(a, __uint_as_float(v.w), __uint_as_float(sr[4 * k + 3])));
                }
                if (rank > 0) tmem_st16(tmem + lanes + T_S + 64 * s + 16 * sl, pv);  // P_k replaces S_k
            }
            if (l == 0) st_peer_f32(dst + T::ST_BYTES, alog_prev + cend);
            arrive_peer(peer_addr(bar(B_P_FULL), rank + 1));
            if (rank > 0) {
                if (l == 0) alp[s] = alog_prev;
                tmem_wait_st();
                fence_before_sync();
                arrive_peer(peer_addr(bar(B_P_FREE), rank - 1));  // the slot is read
                mbar_arrive(bar(B_PK_READY + s));
            } else {
                fence_before_sync();
                mbar_arrive(bar(B_S_FREE + s));  // rank 0 needs no P_k: the tile state is done with
            }
            return true;
        };

        Item eit = decode_item(p, cid, hc, kc, rank);
        int64_t eit_i = 0;
        auto epilogue = [&](int64_t h) -> bool {
            const int s = static_cast<int>(h & 1), d4 = static_cast<int>(h & 3);
            const int64_t ii = static_cast<uint32_t>(h) / static_cast<uint32_t>(hc);
            if (ii != eit_i) {
                eit_i = ii;
                eit = decode_item(p, cid + ii * ncl, hc, kc, rank);
            }
            const Item& it = eit;
            const int64_t hh = it.hfirst + (h - ii * hc);
            const bool live = l < it.Lt;
            bool r = wb(B_DEC_FULL + d4, (h >> 2) & 1);
            r = r && wb(B_EPF_FULL + d4, (h >> 2) & 1);
            r = r && wb(B_YI_FULL + s, (h >> 1) & 1);
            r = uni(r && wb(B_YS_FULL + s, (h >> 1) & 1));
            if (!r) return false;
            fence_after_sync();
            if (l == 0) FTRACE(h, 13);
            const float* dec = dec_ptr(d4);
            const float f = dec[3 * TL + l];
            const float gs = ex2(dec[l]);
            const int64_t off = ((it.b * L + it.t0 + l) * H + hh) * PD;
            const float2 f2 = make_float2(f, f), g2 = make_float2(gs, gs);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t acc[4][16];  // [intra, state] x two 16-column slices
                const uint32_t a4[4] = {tmem + lanes + T_YI + 64 * s + 32 * half,
                                        tmem + lanes + T_YS + 64 * s + 32 * half,
                                        tmem + lanes + T_YI + 64 * s + 32 * half + 16,
                                        tmem + lanes + T_YS + 64 * s + 32 * half + 16};
                tmem_ld16x4(a4, acc);
                if (half == 1) {  // every accumulator of the head is read
                    fence_before_sync();
                    mbar_arrive(bar(B_ACC_FREE + s));
                }
                if (!live) continue;
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    const int p0 = 32 * half + 16 * sl;
                    uint4 zv[2];
                    if (GATED) {
                        const uint4* zr = reinterpret_cast<const uint4*>(zg + off + p0);
                        zv[0] = ldg16(zr);
                        zv[1] = ldg16(zr + 1);
                    }
                    uint32_t o[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float2 vi = make_float2(__uint_as_float(acc[2 * sl][2 * k]),
                                                      __uint_as_float(acc[2 * sl][2 * k + 1]));
                        const float2 vs = make_float2(__uint_as_float(acc[2 * sl + 1][2 * k]),
                                                      __uint_as_float(acc[2 * sl + 1][2 * k + 1]));
                        float2 yv = __ffma2_rn(g2, vs, __fmul2_rn(f2, vi));
                        if (GATED) {
                            const uint32_t zw[8] = {zv[0].x, zv[0].y, zv[0].z, zv[0].w,
                                                    zv[1].x, zv[1].y, zv[1].z, zv[1].w};
                            const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&zw[k]));
                            yv.x *= silu_f32(zf.x);
                            yv.y *= silu_f32(zf.y);
                        }
                        o[k] = pack_bf16x2(yv.x, yv.y);
                    }
                    uint4* yr = reinterpret_cast<uint4*>(yg + off + p0);
                    yr[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    yr[1] = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
            mbar_arrive(bar(B_DEC_FREE + d4));
            if (l == 0) FTRACE(h, 14);
            return true;
        };

        bool ok = true;
        if (last) {
            for (int64_t h = 0; ok && h < heads_total; ++h) ok = epilogue(h);
        } else {
            for (int64_t g = 0; ok && g <= heads_total; ++g) {
                if (g < heads_total) ok = prefix(g);
                if (ok && g >= 1) ok = epilogue(g - 1);
            }
        }
        if (!ok) raise_abort(abort, g_abort);
    }
    fence_before_sync();
    __syncthreads();
    if (*abort && tid == 0) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
    cluster_sync_all();  // no peer touches this CTA's shared memory after it leaves
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// reader counts of the ring slots: [2][batch][nheads] ints, rounded to 256 bytes
size_t counter_bytes(const FwdParams& p) { return (2ull * p.batch * p.nheads * 4 + 255) / 256 * 256; }

int cluster_size_for(const FwdParams& p) {
    const int64_t nt = (p.seqlen + TL - 1) / TL;
    return nt >= 3 ? 4 : (nt == 2 ? 2 : 1);
}

// Heads per work item: an item pays a fixed set-up (C and B in, CB and its
// repack) and then runs its heads through the pipeline; with w waves of items
// over the clusters the kernel takes about w * (setup + heads * per_head).  The
// divisor of the heads per group that minimises this is used (up to 16).
int fused_heads_per_item(const FwdParams& p, int clusters, int kc) {
    static const int forced = [] {
        const char* e = getenv("SSD_FUSED_HEADS_PER_ITEM");
        return e ? atoi(e) : 0;
    }();
    if (forced > 0 && p.heads_per_group % forced == 0) return forced;
    const int64_t nt = (p.seqlen + TL - 1) / TL;
    const int64_t units = p.batch * ((nt + kc - 1) / kc) * p.ngroups;
    const double setup = 4.0, per_head = 1.5;
    int best = 1;
    double best_t = 0.0;
    for (int d = 1; d <= p.heads_per_group && d <= 16; ++d) {
        if (p.heads_per_group % d) continue;
        const int64_t items = units * (p.heads_per_group / d);
        const double waves = static_cast<double>((items + clusters - 1) / clusters);
        const double t = waves * (setup + per_head * d);
        if (d == 1 || t < best_t) {
            best = d;
            best_t = t;
        }
    }
    return best;
}

template <int NST, bool GATED>
cudaError_t launch_nd(const FwdParams& p, void* ws, cudaStream_t s) {
    using T = FSmem<NST>;
    auto kern = fused_fwd_kernel<NST, GATED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    const int kc = cluster_size_for(p);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(kc);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = T::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (max_clusters < 1) return cudaErrorInvalidConfiguration;
    const int hc = fused_heads_per_item(p, max_clusters, kc);
    const int64_t nt = (p.seqlen + TL - 1) / TL;
    const int64_t nruns = (nt + kc - 1) / kc;
    const int64_t items = p.batch * nruns * p.ngroups * (p.heads_per_group / hc);
    const int64_t ncl = items < max_clusters ? items : max_clusters;
    cfg.gridDim = dim3(static_cast<unsigned>(ncl * kc));
    CUtensorMap tc_, tb_, tx_;
    if (!make_tmap_bf16_4d(&tc_, p.C, NST, p.ngroups, p.seqlen, p.batch, 1, TL) ||
        !make_tmap_bf16_4d(&tb_, p.B, NST, p.ngroups, p.seqlen, p.batch, 1, TL) ||
        !make_tmap_bf16_4d(&tx_, p.x, PD, p.nheads, p.seqlen, p.batch, 1, TL))
        return cudaErrorInvalidValue;
    // the header (status, abort word), the reader counts and the ring start from zero
    e = cudaMemsetAsync(ws, 0, fused_fwd_workspace_bytes(p), s);
    if (e != cudaSuccess) return e;
    FwdParams q = p;
    q.status = static_cast<int*>(ws);
    uint64_t* ring = reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + kHdrBytes + counter_bytes(p));
    return cudaLaunchKernelEx(&cfg, kern, q, tc_, tb_, tx_, hc, kc, items, nruns, ring,
                              debug_withhold(SSD_DEBUG_FWD_CARRY));
}

}  // namespace

#ifdef SSD_TRACE
extern "C" int ssd_fused_trace_copy(void* dst) {
    return cudaMemcpyFromSymbol(dst, g_fused_trace, sizeof(g_fused_trace)) == cudaSuccess ? 0 : 1;
}
extern "C" int ssd_fused_trace_clear() {
    static long long zero[kTraceCtas][kTraceHeads * kTraceEv];
    return cudaMemcpyToSymbol(g_fused_trace, zero, sizeof(zero)) == cudaSuccess ? 0 : 1;
}
#endif

bool fused_fwd_supported(const FwdParams& p) {
    return p.headdim == PD && (p.dstate == 64 || p.dstate == 128) &&
           (p.seqlen + TL - 1) / TL < 4 * 65534ll;
}

size_t fused_fwd_workspace_bytes(const FwdParams& p) {
    return kHdrBytes + counter_bytes(p) + 2ull * p.batch * p.nheads * p.headdim * p.dstate * sizeof(float);
}

cudaError_t launch_fused_fwd(const FwdParams& p, void* ws, cudaStream_t s) {
    if (p.dstate == 64) return p.z ? launch_nd<64, true>(p, ws, s) : launch_nd<64, false>(p, ws, s);
    if (p.dstate == 128) return p.z ? launch_nd<128, true>(p, ws, s) : launch_nd<128, false>(p, ws, s);
    return cudaErrorInvalidValue;
}

}  // namespace ssd
