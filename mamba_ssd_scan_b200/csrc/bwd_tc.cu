// bwd_tc.cu -- the per-chunk products of the SSD backward pass on the tensor
// cores (tcgen05, bf16 operands, fp32 accumulation in TMEM), for bf16 inputs
// with headdim 64, dstate 64 or 128 and chunk 128 or 256.  They compute what
// bwd.cu's CUDA-core kernels A and B compute (see there for the formulas),
// on 128-token tiles:
//
//   kernel A, per (b, c, h, source tile s), for every target tile t >= s:
//     T1 = C_t B_s^T, T2 = dy_t x_s^T            (MMA, 128 x 128 in TMEM)
//     masked and decayed by e^{cumA_t - cumA_s} (t >= s), W = T1 T2 dt_s (t > s)
//     row sums of W (per target token) and column sums (per source token)
//     dxs += T1^T dy_t, dB += T2^T C_t          (MMA from the bf16 tiles)
//   then the dH terms B_s dH^T and x_s dH (MMA), and dx, dB and the per-token
//   pieces x . dxs, dy . x and the dH share m;
//   kernel B, per (b, c, h, target tile t), for every source tile s <= t:
//     T2 = dy_t x_s^T, masked, decayed and scaled by dt_s, dC += T2 B_s (MMA)
//   then the H_c term dy_t H_c (MMA), dC, q = C_t . (that term) and, for the
//   first tile, e^{cumA_last} <dH_c, H_c>.
//
// One CTA of 128 threads: thread 0 issues the MMAs and commits them to an
// mbarrier; every warp then reads its 32 TMEM lanes (rows).  Operand tiles are
// staged from global memory with 16-byte loads into the 128-byte-swizzled
// layout (K-major or MN-major per use, one physical tile serving both), and
// the masked T tiles are written back as bf16 in the same layout.  All waits
// are bounded; a timed-out wait stops the CTA and sets the call's status word.
#include "internal.cuh"
#include "bwd_tc.h"
#include "tcgen05.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int R = 128;              // rows of a tile (tokens)
constexpr int BLK = R * 128;        // bytes of one 64-column SW128 block of a 128-row tile
constexpr int TPB = 256;            // threads per CTA: two warps per TMEM lane quarter
constexpr float kLog2eB = 1.4426950408889634f;

// 16 bytes global -> shared without passing through registers; src_bytes 0
// writes zeros (the source is not read)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Bring the 128-byte line holding p into L2 (no register is written, nothing
// waits on it): data a CTA stages only later in its serial chain of phases is
// requested at its start, so the later copies hit L2.
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// rows [r0, r0 + R) x 64-column blocks of a bf16 matrix (row stride `stride`
// elements, `ncol` columns) into SW128 blocks at dst with asynchronous copies
// (all in flight together); rows at or past `lim` are zero.  The caller waits
// (cp_async_wait_all) before the barrier that publishes the tile.
__device__ __forceinline__ void stage_tile(uint32_t dst, const __nv_bfloat16* src, int64_t stride,
                                           int ncol, int r0, int lim, int rows = R) {
    const int chunks = rows * (ncol / 8);  // 16-byte chunks
    for (int i = threadIdx.x; i < chunks; i += TPB) {
        const int r = i / (ncol / 8), c = i % (ncol / 8);
        const bool ok = r0 + r < lim;
        const __nv_bfloat16* g = src + static_cast<int64_t>(ok ? r0 + r : r0) * stride + c * 8;
        cp_async16(dst + (c >> 3) * (rows * 128) + sw128(r, c & 7), g, ok ? 16u : 0u);
    }
}

// After the transposed reduction lane l holds sum over the warp's 32 lanes of
// v[l] (v[j] = this lane's value of column j).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < off; ++j) {
            const float send = upper ? v[j] : v[j + off];
            const float keep = upper ? v[j + off] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

constexpr int PD = 64;  // headdim of the tensor-core path

template <int NST>
struct ATile {
    static constexpr int NBN = NST / 64;               // 64-column blocks of B, C, dH
    static constexpr int B_OFF = 0;                    // B_s
    static constexpr int X_OFF = B_OFF + NBN * BLK;    // x_s
    static constexpr int C_OFF = X_OFF + BLK;          // C_t
    static constexpr int Y_OFF = C_OFF + NBN * BLK;    // dy_t
    static constexpr int T1_OFF = Y_OFF + BLK;         // masked C_t . B_s = hi + lo, bf16 [t][s]
    static constexpr int T1L_OFF = T1_OFF + 2 * BLK;
    static constexpr int T2_OFF = T1L_OFF + 2 * BLK;   // masked dy_t . x_s, bf16 [t][s]
    static constexpr int DH_OFF = T2_OFF;              // after the loop: dH = hi + lo, bf16 [p][n] each
    static constexpr int COL_OFF = T2_OFF + 2 * BLK;   // [4][R] column sums of W
    static constexpr int CS_OFF = COL_OFF + 4 * R * 4;       // [256] cumA, then [256] dt
    static constexpr int ROW_OFF = CS_OFF + 2 * 256 * 4;     // [2][R] the halves' row sums of W
    static constexpr int BAR_OFF = ROW_OFF + 2 * R * 4;
    static constexpr int BYTES = BAR_OFF + 64 + 1024;        // + alignment slack
    static_assert(2 * NBN * 64 * 128 <= 2 * BLK, "dH hi + lo must fit in the T2 tile");
    static_assert(BYTES <= 232448, "kernel A's shared memory exceeds 227 KB");
};

template <int NST>
__global__ void __launch_bounds__(TPB, 1) bwd_tc_a_kernel(BwdParams bp) {
    using T = ATile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int NTT = static_cast<int>(Q / R);
    const int64_t h = blockIdx.x / NTT;
    const int is = blockIdx.x % NTT;
    const int64_t c = blockIdx.y, b = blockIdx.z, g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int s0 = is * R;
    if (s0 >= Lc) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = smem_u32(smem);
    const uint32_t sB = base + T::B_OFF, sX = base + T::X_OFF, sC = base + T::C_OFF;
    const uint32_t sY = base + T::Y_OFF, sT1 = base + T::T1_OFF, sT1L = base + T::T1L_OFF;
    const uint32_t sT2 = base + T::T2_OFF;
    const uint32_t sdH = base + T::DH_OFF, sdL = sdH + T::NBN * 64 * 128;
    float* scol = reinterpret_cast<float*>(smem + T::COL_OFF);
    float* scs = reinterpret_cast<float*>(smem + T::CS_OFF);
    float* sdt = scs + 256;
    float* srow = reinterpret_cast<float*>(smem + T::ROW_OFF);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);
    const int quarter = warp & 3, half = warp >> 2;  // TMEM lanes 32 quarter.., column half

    const int64_t xs = H * PD, bs = G * NST;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(p.x) + ((b * L + t0) * H + h) * PD;
    const __nv_bfloat16* dyb = static_cast<const __nv_bfloat16*>(bp.dy) + ((b * L + t0) * H + h) * PD;
    const __nv_bfloat16* Bb = static_cast<const __nv_bfloat16*>(p.B) + ((b * L + t0) * G + g) * NST;
    const __nv_bfloat16* Cb = static_cast<const __nv_bfloat16*>(p.C) + ((b * L + t0) * G + g) * NST;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;

    if (warp == 0) tmem_alloc(smem_u32(tslot), 512);
    if (tid == 0) {
        mbar_init(smem_u32(bar), 1);
        *abort = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < Q; i += TPB) {
        scs[i] = csc[i];
        sdt[i] = dtc[i];
    }
    // the later target tiles' C and dy rows and the chunk's dH, into L2
    for (int it = is + 1; it < NTT; ++it) {
        const int r = it * R + tid;
        if (tid < R && r < Lc) {
            for (int cb = 0; cb < NST * 2; cb += 128) prefetch_l2(reinterpret_cast<const char*>(Cb + r * bs) + cb);
            prefetch_l2(dyb + r * xs);
        }
    }
    {
        const float* dHp = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST;
        for (int i = tid; i < PD * NST / 32; i += TPB) prefetch_l2(dHp + 32 * i);
    }
    stage_tile(sB, Bb, bs, NST, s0, Lc);
    stage_tile(sX, xb, xs, PD, s0, Lc);
    cp_async_wait_all();
    fence_smem_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
    const uint32_t T1A = tmem, T2A = tmem + 128, DXS = tmem + 256, DBA = tmem + 320;
    const uint32_t mbar = smem_u32(bar);
    uint32_t ph = 0;
    bool failed = false;
    float colacc = 0.0f;  // thread tid < R: column (source token) s0 + tid
    const int64_t tok = (b * H + h) * L + t0;

    for (int it = is; it < NTT; ++it) {
        const int r0 = it * R;
        if (r0 >= Lc) break;
        stage_tile(sC, Cb, bs, NST, r0, Lc);
        stage_tile(sY, dyb, xs, PD, r0, Lc);
        cp_async_wait_all();
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < NST / 16; ++k) {
                const uint32_t o = (k >> 2) * BLK + (k & 3) * 32;
                mma_bf16(T1A, desc_sw128(sC + o, 16, 1024), desc_sw128(sB + o, 16, 1024),
                         idesc_bf16(128, 128, false, false), k > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int k = 0; k < PD / 16; ++k)
                mma_bf16(T2A, desc_sw128(sY + k * 32, 16, 1024), desc_sw128(sX + k * 32, 16, 1024),
                         idesc_bf16(128, 128, false, false), k > 0 ? 1u : 0u);
            mma_commit(mbar);
        }
        const bool ok1 = wait_or_abort(mbar, ph, abort);
        ph ^= 1u;
        if (__syncthreads_or(!ok1)) {
            failed = true;
            break;
        }
        fence_after_sync();
        // row t of the scores, this warp's column half: mask, decay, W sums, bf16 tiles
        const int row = 32 * quarter + lane, tl = r0 + row;
        const float cst = scs[tl];
        float rowp = 0.0f;
#pragma unroll 1
        for (int q = 2 * half; q < 2 * half + 2; ++q) {
            float v1[32], v2[32], wv[32];
            tmem_ld32x2(T1A + lane_off + q * 32, v1, T2A + lane_off + q * 32, v2);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int sl = s0 + q * 32 + j;
                const float w = (tl >= sl && tl < Lc) ? ex2((cst - scs[sl]) * kLog2eB) : 0.0f;
                const float t1 = v1[j] * w;
                const float wst = (tl > sl) ? t1 * v2[j] * sdt[sl] : 0.0f;
                rowp += wst;
                wv[j] = wst;
                v1[j] = t1;
                v2[j] *= w;
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const uint32_t o = (q >> 1) * BLK + sw128(row, (q & 1) * 4 + cc);
                // T1 = hi + lo: the sum over the target tokens in dxs cancels,
                // and bf16 alone (8 bits) leaves too much of each term behind
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a0 = v1[8 * cc + 2 * e], a1 = v1[8 * cc + 2 * e + 1];
                    hi[e] = pack_bf16x2(a0, a1);
                    lo[e] = pack_bf16x2(a0 - __uint_as_float(hi[e] << 16),
                                        a1 - __uint_as_float(hi[e] & 0xffff0000u));
                }
                st_shared_v4(sT1 + o, hi[0], hi[1], hi[2], hi[3]);
                st_shared_v4(sT1L + o, lo[0], lo[1], lo[2], lo[3]);
                st_shared_v4(sT2 + o, pack_bf16x2(v2[8 * cc], v2[8 * cc + 1]),
                             pack_bf16x2(v2[8 * cc + 2], v2[8 * cc + 3]),
                             pack_bf16x2(v2[8 * cc + 4], v2[8 * cc + 5]),
                             pack_bf16x2(v2[8 * cc + 6], v2[8 * cc + 7]));
            }
            scol[quarter * R + q * 32 + lane] = transpose_reduce32(wv, lane);
        }
        srow[half * R + row] = rowp;
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid < R) {
            colacc += (scol[tid] + scol[R + tid]) + (scol[2 * R + tid] + scol[3 * R + tid]);
            if (r0 + tid < Lc) bp.roww[((b * H + h) * NTT + is) * L + t0 + r0 + tid] = srow[tid] + srow[R + tid];
        }
        if (tid == 0) {
            // dxs += T1^T dy_t, dB += T2^T C_t: K = the target tile's 128 tokens
#pragma unroll
            for (int k = 0; k < R / 16; ++k) {
                const uint32_t acc = (it > is || k > 0) ? 1u : 0u;
                mma_bf16(DXS, desc_sw128(sT1 + k * 2048, BLK, 1024), desc_sw128(sY + k * 2048, BLK, 1024),
                         idesc_bf16(128, PD, true, true), acc);
                mma_bf16(DXS, desc_sw128(sT1L + k * 2048, BLK, 1024), desc_sw128(sY + k * 2048, BLK, 1024),
                         idesc_bf16(128, PD, true, true), 1u);
                mma_bf16(DBA, desc_sw128(sT2 + k * 2048, BLK, 1024), desc_sw128(sC + k * 2048, BLK, 1024),
                         idesc_bf16(128, NST, true, true), acc);
            }
            mma_commit(mbar);
        }
        const bool ok2 = wait_or_abort(mbar, ph, abort);
        ph ^= 1u;
        if (__syncthreads_or(!ok2)) {
            failed = true;
            break;
        }
        fence_after_sync();
    }
    if (!failed) {
        // the dH terms: dH (fp32) = hi + lo, both bf16 [p][n] tiles (the carried
        // adjoint is large next to a chunk's own terms; hi alone would round it
        // to 8 bits), then B_s dH^T and x_s dH as two MMAs each
        const float* dHg = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST;
        for (int i = tid; i < PD * NST / 8; i += TPB) {
            const int pr = i / (NST / 8), cc = i % (NST / 8);
            const float4 a0 = reinterpret_cast<const float4*>(dHg + pr * NST + cc * 8)[0];
            const float4 a1 = reinterpret_cast<const float4*>(dHg + pr * NST + cc * 8)[1];
            const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hi[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                const float h0 = __uint_as_float(hi[e] << 16), h1 = __uint_as_float(hi[e] & 0xffff0000u);
                lo[e] = pack_bf16x2(v[2 * e] - h0, v[2 * e + 1] - h1);
            }
            const uint32_t o = (cc >> 3) * (64 * 128) + sw128(pr, cc & 7);
            st_shared_v4(sdH + o, hi[0], hi[1], hi[2], hi[3]);
            st_shared_v4(sdL + o, lo[0], lo[1], lo[2], lo[3]);
        }
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t sd = part == 0 ? sdH : sdL;
#pragma unroll
                for (int k = 0; k < NST / 16; ++k)
                    mma_bf16(T1A, desc_sw128(sB + (k >> 2) * BLK + (k & 3) * 32, 16, 1024),
                             desc_sw128(sd + (k >> 2) * (64 * 128) + (k & 3) * 32, 16, 1024),
                             idesc_bf16(128, PD, false, false), (part > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < PD / 16; ++k)
                    mma_bf16(T2A, desc_sw128(sX + k * 32, 16, 1024),
                             desc_sw128(sd + k * 2048, 64 * 128, 1024),
                             idesc_bf16(128, NST, false, true), (part > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(mbar);
        }
        const bool ok3 = wait_or_abort(mbar, ph, abort);
        failed = __syncthreads_or(!ok3);
        fence_after_sync();
    }
    if (!failed) {
        // outputs of the source row s: dx and its per-token pieces in the low
        // half of the warps, dB in the high half
        const int row = 32 * quarter + lane, sl = s0 + row;
        const bool valid = sl < Lc;
        const float dts = valid ? sdt[sl] : 0.0f;
        const float wsr = valid ? ex2((scs[Q - 1] - scs[sl]) * kLog2eB) : 0.0f;
        if (half == 0) {
            const float Dh = p.D ? p.D[h] : 0.0f;
            float xv[PD], dyv[PD];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint4 v = ld_shared_v4(sX + sw128(row, cc));
                const uint4 u = valid ? ldg16(dyb + static_cast<int64_t>(sl) * xs + cc * 8)
                                      : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t vw[4] = {v.x, v.y, v.z, v.w}, uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xv[cc * 8 + 2 * e] = __uint_as_float(vw[e] << 16);
                    xv[cc * 8 + 2 * e + 1] = __uint_as_float(vw[e] & 0xffff0000u);
                    dyv[cc * 8 + 2 * e] = __uint_as_float(uw[e] << 16);
                    dyv[cc * 8 + 2 * e + 1] = __uint_as_float(uw[e] & 0xffff0000u);
                }
            }
            float pxd = 0.0f, pm = 0.0f, pyx = 0.0f;
            __nv_bfloat16* dxo = static_cast<__nv_bfloat16*>(bp.dx) + ((b * L + t0) * H + h) * PD;
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                float vi[32], vs[32];
                tmem_ld32x2(DXS + lane_off + hp * 32, vi, T1A + lane_off + hp * 32, vs);
                uint32_t o[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const int pp = hp * 32 + j;
                    const float st0 = wsr * vs[j], st1 = wsr * vs[j + 1];
                    const float d0 = vi[j] + st0, d1 = vi[j + 1] + st1;
                    pxd = fmaf(xv[pp], d0, fmaf(xv[pp + 1], d1, pxd));
                    pm = fmaf(xv[pp], st0, fmaf(xv[pp + 1], st1, pm));
                    pyx = fmaf(dyv[pp], xv[pp], fmaf(dyv[pp + 1], xv[pp + 1], pyx));
                    o[j >> 1] = pack_bf16x2(fmaf(dts, d0, Dh * dyv[pp]), fmaf(dts, d1, Dh * dyv[pp + 1]));
                }
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(dxo + static_cast<int64_t>(sl) * xs + hp * 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
                }
            }
            if (valid) {
                bp.xdxs[tok + sl] = pxd;
                bp.dyx[tok + sl] = pyx;
                bp.mterm[tok + sl] = dts * pm;
                bp.colw[tok + sl] = colacc;  // row == tid in this half
            }
        } else {
#pragma unroll
            for (int q = 0; q < NST / 32; ++q) {
                float vi[32], vs[32];
                tmem_ld32x2(DBA + lane_off + q * 32, vi, T2A + lane_off + q * 32, vs);
                if (valid) {
                    if (bp.dB_h) {
                        float* dst = bp.dB_h + ((b * L + t0 + sl) * H + h) * NST + q * 32;
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(dst + j) = make_float4(
                                dts * fmaf(wsr, vs[j], vi[j]), dts * fmaf(wsr, vs[j + 1], vi[j + 1]),
                                dts * fmaf(wsr, vs[j + 2], vi[j + 2]), dts * fmaf(wsr, vs[j + 3], vi[j + 3]));
                    } else {
                        __nv_bfloat16* dst =
                            static_cast<__nv_bfloat16*>(bp.dB) + ((b * L + t0 + sl) * G + g) * NST + q * 32;
#pragma unroll
                        for (int j = 0; j < 32; j += 8)
                            *reinterpret_cast<uint4*>(dst + j) = make_uint4(
                                pack_bf16x2(dts * fmaf(wsr, vs[j], vi[j]), dts * fmaf(wsr, vs[j + 1], vi[j + 1])),
                                pack_bf16x2(dts * fmaf(wsr, vs[j + 2], vi[j + 2]), dts * fmaf(wsr, vs[j + 3], vi[j + 3])),
                                pack_bf16x2(dts * fmaf(wsr, vs[j + 4], vi[j + 4]), dts * fmaf(wsr, vs[j + 5], vi[j + 5])),
                                pack_bf16x2(dts * fmaf(wsr, vs[j + 6], vi[j + 6]), dts * fmaf(wsr, vs[j + 7], vi[j + 7])));
                    }
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
    if (failed && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
}

template <int NST>
struct BTile {
    static constexpr int NBN = NST / 64;
    static constexpr int Y_OFF = 0;                    // dy_t
    static constexpr int X_OFF = Y_OFF + BLK;          // x_s
    static constexpr int B_OFF = X_OFF + BLK;          // B_s
    static constexpr int T_OFF = B_OFF + NBN * BLK;    // masked, decayed, dt-scaled dy_t . x_s, bf16 [t][s]
    // H_c, bf16 [p][n], staged after the source loop into the x tile, which
    // no MMA reads any more by then; the kernel stays under half an SM's
    // shared memory, so two CTAs share an SM (TMEM: 256 columns each)
    static constexpr int H_OFF = X_OFF;
    static constexpr int CS_OFF = T_OFF + 2 * BLK;
    static constexpr int SQ_OFF = CS_OFF + 2 * 256 * 4;  // [2][R] the halves' q partials, then [8] sums
    static constexpr int BAR_OFF = SQ_OFF + (2 * R + 8) * 4;
    static constexpr int BYTES = BAR_OFF + 64 + 1024;
    static_assert(NBN * 64 * 128 <= BLK, "H_c must fit in the x tile");
    static_assert(2 * (BYTES + 1024) <= 233472, "two CTAs of kernel B per SM");
};

template <int NST>
__global__ void __launch_bounds__(TPB, 2) bwd_tc_b_kernel(BwdParams bp) {
    using T = BTile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int NTT = static_cast<int>(Q / R);
    const int64_t h = blockIdx.x / NTT;
    const int it = blockIdx.x % NTT;
    const int64_t c = blockIdx.y, b = blockIdx.z, g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int r0 = it * R;
    if (r0 >= Lc) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = smem_u32(smem);
    const uint32_t sY = base + T::Y_OFF, sX = base + T::X_OFF, sB = base + T::B_OFF;
    const uint32_t sT = base + T::T_OFF, sH = base + T::H_OFF;
    float* scs = reinterpret_cast<float*>(smem + T::CS_OFF);
    float* sdt = scs + 256;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);
    float* sq = reinterpret_cast<float*>(smem + T::SQ_OFF);
    float* wsum = sq + 2 * R;  // [8]
    const int quarter = warp & 3, half = warp >> 2;

    const int64_t xs = H * PD, bs = G * NST;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(p.x) + ((b * L + t0) * H + h) * PD;
    const __nv_bfloat16* dyb = static_cast<const __nv_bfloat16*>(bp.dy) + ((b * L + t0) * H + h) * PD;
    const __nv_bfloat16* Bb = static_cast<const __nv_bfloat16*>(p.B) + ((b * L + t0) * G + g) * NST;
    const __nv_bfloat16* Cb = static_cast<const __nv_bfloat16*>(p.C) + ((b * L + t0) * G + g) * NST;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;
    const float* dtc = p.dt + ((b * H + h) * nc + c) * Q;

    if (warp == 0) tmem_alloc(smem_u32(tslot), 256);
    if (tid == 0) {
        mbar_init(smem_u32(bar), 1);
        *abort = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < Q; i += TPB) {
        scs[i] = csc[i];
        sdt[i] = dtc[i];
    }
    stage_tile(sY, dyb, xs, PD, r0, Lc);
    // the chunk's H_c (staged after the source loop) into L2
    {
        const __nv_bfloat16* Hp = static_cast<const __nv_bfloat16*>(p.states) +
                                  ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST;
        for (int i = tid; i < PD * NST / 64; i += TPB) prefetch_l2(Hp + 64 * i);
    }
    const uint32_t mbar = smem_u32(bar);
    uint32_t ph = 0;
    bool failed = false;
    uint32_t tmem = 0;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
    const int row = 32 * quarter + lane, tl = r0 + row;
    for (int is = 0; is <= it; ++is) {
        const int s0 = is * R;
        stage_tile(sX, xb, xs, PD, s0, Lc);
        stage_tile(sB, Bb, bs, NST, s0, Lc);
        cp_async_wait_all();
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        tmem = *tslot;
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < PD / 16; ++k)
                mma_bf16(tmem, desc_sw128(sY + k * 32, 16, 1024), desc_sw128(sX + k * 32, 16, 1024),
                         idesc_bf16(128, 128, false, false), k > 0 ? 1u : 0u);
            mma_commit(mbar);
        }
        const bool ok1 = wait_or_abort(mbar, ph, abort);
        ph ^= 1u;
        if (__syncthreads_or(!ok1)) {
            failed = true;
            break;
        }
        fence_after_sync();
        const float cst = scs[tl];
#pragma unroll 1
        for (int q = 2 * half; q < 2 * half + 2; ++q) {
            float v[32];
            tmem_ld32(tmem + lane_off + q * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int sl = s0 + q * 32 + j;
                const float w = (tl >= sl && tl < Lc) ? ex2((cst - scs[sl]) * kLog2eB) * sdt[sl] : 0.0f;
                v[j] *= w;
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
                st_shared_v4(sT + (q >> 1) * BLK + sw128(row, (q & 1) * 4 + cc),
                             pack_bf16x2(v[8 * cc], v[8 * cc + 1]), pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]),
                             pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]), pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]));
        }
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            // dC += T B_s: A the [t][s] tile (K-major, K = s), B = B_s (MN-major, N = n)
#pragma unroll
            for (int k = 0; k < R / 16; ++k)
                mma_bf16(tmem + 128, desc_sw128(sT + (k >> 2) * BLK + (k & 3) * 32, 16, 1024),
                         desc_sw128(sB + k * 2048, BLK, 1024), idesc_bf16(128, NST, false, true),
                         (is > 0 || k > 0) ? 1u : 0u);
            mma_commit(mbar);
        }
        const bool ok2 = wait_or_abort(mbar, ph, abort);
        ph ^= 1u;
        if (__syncthreads_or(!ok2)) {
            failed = true;
            break;
        }
        fence_after_sync();
    }
    const __nv_bfloat16* Hg = static_cast<const __nv_bfloat16*>(p.states) +
                              ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST;
    if (!failed) {
        // the H_c term e^{cumA_t} dy_t H_c: A = dy_t (K-major, K = p), B = H_c (MN-major, N = n)
        stage_tile(sH, Hg, NST, NST, 0, PD, PD);
        cp_async_wait_all();
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
#pragma unroll
            for (int k = 0; k < PD / 16; ++k)
                mma_bf16(tmem, desc_sw128(sY + k * 32, 16, 1024), desc_sw128(sH + k * 2048, 64 * 128, 1024),
                         idesc_bf16(128, NST, false, true), k > 0 ? 1u : 0u);
            mma_commit(mbar);
        }
        const bool ok3 = wait_or_abort(mbar, ph, abort);
        failed = __syncthreads_or(!ok3);
        fence_after_sync();
    }
    if (!failed) {
        const bool valid = tl < Lc;
        const float wt = valid ? ex2(scs[tl] * kLog2eB) : 0.0f;
        float pq = 0.0f;
#pragma unroll
        for (int q = half * (NST / 64); q < (half + 1) * (NST / 64); ++q) {
            float vi[32], vs[32];
            tmem_ld32x2(tmem + 128 + lane_off + q * 32, vi, tmem + lane_off + q * 32, vs);
            if (valid) {
                float cv[32];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 u = ldg16(Cb + static_cast<int64_t>(tl) * bs + q * 32 + 8 * k);
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        cv[8 * k + 2 * e] = __uint_as_float(uw[e] << 16);
                        cv[8 * k + 2 * e + 1] = __uint_as_float(uw[e] & 0xffff0000u);
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float st = wt * vs[j];
                    pq = fmaf(cv[j], st, pq);
                    vi[j] += st;
                }
                if (bp.dC_h) {
                    float* dst = bp.dC_h + ((b * L + t0 + tl) * H + h) * NST + q * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(dst + j) = make_float4(vi[j], vi[j + 1], vi[j + 2], vi[j + 3]);
                } else {
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(bp.dC) + ((b * L + t0 + tl) * G + g) * NST + q * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *reinterpret_cast<uint4*>(dst + j) = make_uint4(
                            pack_bf16x2(vi[j], vi[j + 1]), pack_bf16x2(vi[j + 2], vi[j + 3]),
                            pack_bf16x2(vi[j + 4], vi[j + 5]), pack_bf16x2(vi[j + 6], vi[j + 7]));
                }
            }
        }
        sq[half * R + row] = pq;
        __syncthreads();
        if (half == 0 && valid) bp.qterm[(b * H + h) * L + t0 + tl] = sq[row] + sq[R + row];
        if (it == 0) {
            // e^{cumA_last} <dH_c, H_c>, reduced in a fixed order
            const float* dHg = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST;
            float v = 0.0f;
            for (int i = tid; i < PD * NST; i += TPB) v = fmaf(dHg[i], __bfloat162float(Hg[i]), v);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0) wsum[warp] = v;
            __syncthreads();
            if (tid == 0)
                bp.k4[(b * H + h) * nc + c] = ex2(scs[Q - 1] * kLog2eB) *
                                              (((wsum[0] + wsum[1]) + (wsum[2] + wsum[3])) +
                                               ((wsum[4] + wsum[5]) + (wsum[6] + wsum[7])));
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(*tslot, 256);
    }
    if (failed && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
}

// The chunk-local adjoint dS_c = sum_t e^{cumA_t} dy_t C_t^T, as its transpose
// dS^T[n][p] (M = the state index, zero-padded to 128 rows when dstate is 64;
// K = the chunk's tokens; N = headdim) so that the A operand is C scaled per
// token: e^{cumA_t} C_t enters as bf16 hi + lo (the scaling is not rounded to
// 8 bits), dy_t as staged.  One CTA per (b, c, h); fp32 out, [p][n].
template <int NST>
struct DTile {
    static constexpr int Y_OFF = 0;                  // dy_t, bf16 [t][p]
    static constexpr int AH_OFF = Y_OFF + BLK;       // e^{cumA_t} C_t, hi: 2 blocks of 64 states
    static constexpr int AL_OFF = AH_OFF + 2 * BLK;  // lo
    static constexpr int CS_OFF = AL_OFF + 2 * BLK;
    static constexpr int BAR_OFF = CS_OFF + 256 * 4;
    static constexpr int BYTES = BAR_OFF + 64 + 1024;
};

template <int NST>
__global__ void __launch_bounds__(TPB) bwd_tc_ds_kernel(BwdParams bp) {
    using T = DTile<NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const FwdParams& p = bp.f;
    const int64_t H = p.nheads, G = p.ngroups, L = p.seqlen, Q = p.chunk, nc = p.nchunks;
    const int NTT = static_cast<int>(Q / R);
    const int64_t h = blockIdx.x, c = blockIdx.y, b = blockIdx.z, g = h / p.heads_per_group;
    const int64_t t0 = c * Q;
    const int Lc = static_cast<int>((L - t0 < Q) ? (L - t0) : Q);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t base = smem_u32(smem);
    const uint32_t sY = base + T::Y_OFF, sAh = base + T::AH_OFF, sAl = base + T::AL_OFF;
    float* scs = reinterpret_cast<float*>(smem + T::CS_OFF);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tslot + 1);
    const int64_t xs = H * PD, bs = G * NST;
    const __nv_bfloat16* dyb = static_cast<const __nv_bfloat16*>(bp.dy) + ((b * L + t0) * H + h) * PD;
    const __nv_bfloat16* Cb = static_cast<const __nv_bfloat16*>(p.C) + ((b * L + t0) * G + g) * NST;
    const float* csc = p.cumA + ((b * H + h) * nc + c) * Q;

    if (warp == 0) tmem_alloc(smem_u32(tslot), 64);
    if (tid == 0) {
        mbar_init(smem_u32(bar), 1);
        *abort = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < Q; i += TPB) scs[i] = csc[i];
    if (NST == 64) {  // the padding states 64..127 of A stay zero
        for (int i = tid; i < R * 8; i += TPB) {
            st_shared_v4(sAh + BLK + sw128(i >> 3, i & 7), 0u, 0u, 0u, 0u);
            st_shared_v4(sAl + BLK + sw128(i >> 3, i & 7), 0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();
    const uint32_t tmem = *tslot;
    const uint32_t mbar = smem_u32(bar);
    uint32_t ph = 0;
    bool failed = false;
    for (int it = 0; it < NTT; ++it) {
        const int r0 = it * R;
        if (r0 >= Lc) break;
        stage_tile(sY, dyb, xs, PD, r0, Lc);
        // e^{cumA_t} C_t as hi + lo, rows t, 16-byte chunks of 8 states
        for (int i = tid; i < R * (NST / 8); i += TPB) {
            const int r = i / (NST / 8), cc = i % (NST / 8);
            uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
            if (r0 + r < Lc) {
                const float w = ex2(scs[r0 + r] * kLog2eB);
                const uint4 u = ldg16(Cb + static_cast<int64_t>(r0 + r) * bs + cc * 8);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a0 = w * __uint_as_float(uw[e] << 16);
                    const float a1 = w * __uint_as_float(uw[e] & 0xffff0000u);
                    hi[e] = pack_bf16x2(a0, a1);
                    lo[e] = pack_bf16x2(a0 - __uint_as_float(hi[e] << 16),
                                        a1 - __uint_as_float(hi[e] & 0xffff0000u));
                }
            }
            const uint32_t o = (cc >> 3) * BLK + sw128(r, cc & 7);
            st_shared_v4(sAh + o, hi[0], hi[1], hi[2], hi[3]);
            st_shared_v4(sAl + o, lo[0], lo[1], lo[2], lo[3]);
        }
        cp_async_wait_all();
        fence_smem_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 0) {
            // dS^T += (e^{cumA} C)^T dy: A MN-major (M = state, K = t), B MN-major (N = p, K = t)
#pragma unroll
            for (int k = 0; k < R / 16; ++k) {
                mma_bf16(tmem, desc_sw128(sAh + k * 2048, BLK, 1024), desc_sw128(sY + k * 2048, BLK, 1024),
                         idesc_bf16(128, PD, true, true), (it > 0 || k > 0) ? 1u : 0u);
                mma_bf16(tmem, desc_sw128(sAl + k * 2048, BLK, 1024), desc_sw128(sY + k * 2048, BLK, 1024),
                         idesc_bf16(128, PD, true, true), 1u);
            }
            mma_commit(mbar);
        }
        const bool ok = wait_or_abort(mbar, ph, abort);
        ph ^= 1u;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        fence_after_sync();
    }
    if (!failed) {
        // lane n of the accumulator holds dS^T[n][*]; this warp's half of the 64 columns
        const int n = 32 * quarter + lane;
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + half * 32, v);
        if (n < NST) {
            float* out = bp.dstates + ((b * nc + c) * H + h) * static_cast<int64_t>(PD) * NST + n;
#pragma unroll
            for (int j = 0; j < 32; ++j) out[static_cast<int64_t>(half * 32 + j) * NST] = v[j];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tmem, 64);
    }
    if (failed && tid == 0 && p.status) atomicExch(p.status, static_cast<int>(SSD_ERR_TIMEOUT));
}

template <int NST>
cudaError_t launch_ds(const BwdParams& bp, cudaStream_t s) {
    const FwdParams& p = bp.f;
    const int sd = DTile<NST>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(bwd_tc_ds_kernel<NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, sd);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(p.nheads), static_cast<unsigned>(p.nchunks),
                    static_cast<unsigned>(p.batch));
    bwd_tc_ds_kernel<NST><<<grid, TPB, sd, s>>>(bp);
    return cudaGetLastError();
}

template <int NST>
cudaError_t launch_nst(const BwdParams& bp, cudaStream_t s) {
    const FwdParams& p = bp.f;
    const int sa = ATile<NST>::BYTES, sb = BTile<NST>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(bwd_tc_a_kernel<NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, sa);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(bwd_tc_b_kernel<NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, sb)) !=
        cudaSuccess)
        return e;
    const dim3 grid(static_cast<unsigned>(p.nheads * (p.chunk / R)), static_cast<unsigned>(p.nchunks),
                    static_cast<unsigned>(p.batch));
    bwd_tc_a_kernel<NST><<<grid, TPB, sa, s>>>(bp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_tc_b_kernel<NST><<<grid, TPB, sb, s>>>(bp);
    return cudaGetLastError();
}

}  // namespace

bool bwd_tc_supported(const FwdParams& p) {
    return p.headdim == PD && (p.dstate == 64 || p.dstate == 128) && (p.chunk == 128 || p.chunk == 256);
}

cudaError_t launch_bwd_tc(const BwdParams& bp, cudaStream_t s) {
    return bp.f.dstate == 64 ? launch_nst<64>(bp, s) : launch_nst<128>(bp, s);
}

cudaError_t launch_bwd_tc_dstate(const BwdParams& bp, cudaStream_t s) {
    return bp.f.dstate == 64 ? launch_ds<64>(bp, s) : launch_ds<128>(bp, s);
}

}  // namespace ssd
