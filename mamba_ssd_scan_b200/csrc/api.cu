// api.cu -- the extern "C" entry points of libssd_b200.so (declared and
// documented in include/ssd.h): argument validation, workspace carving and
// kernel dispatch.  Nothing here allocates memory or synchronises the host.
#include <atomic>
#include <stdint.h>
#include <string.h>

#include "gated_rmsnorm.h"
#include "internal.cuh"

namespace {

using ssd::DecodeParams;
using ssd::FwdParams;

constexpr size_t kAlign = 256;
inline size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// true iff the CUDA runtime knows `p` as memory of the current device
bool on_current_device(const void* p) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeManaged) return true;
    return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// A required (or optional when allow_null) device pointer, 16-byte aligned
// when need_align.
bool check_ptr(const void* p, bool allow_null, bool need_align) {
    if (!p) return allow_null;
    if (need_align && !aligned16(p)) return false;
    return on_current_device(p);
}

struct WsLayout {
    size_t status, dt, cumA, states, states_hl, total;
};

bool use_tc(int dtype, int flags) {
    return dtype == SSD_BF16 && (flags & SSD_FLAG_CUDA_CORES) == 0;
}

// Chunk states in the split-step path are fp32, except in the opt-in
// bf16-states mode (bf16 inputs with SSD_FLAG_BF16_STATES).
bool bf16_states(const ssd_fwd_args& a) {
    return a.dtype == SSD_BF16 && (a.flags & SSD_FLAG_BF16_STATES) != 0;
}

// With fp32 states and the tensor-core chunk_scan, state passing also writes
// the entering states as hi / lo bf16 halves, the operand that kernel takes.
bool states_hilo(const ssd_fwd_args& a) {
    if (!use_tc(a.dtype, a.flags) || bf16_states(a)) return false;
    ssd::FwdParams q{};  // only the sizes the support check reads
    q.headdim = a.headdim;
    q.dstate = a.dstate;
    q.chunk = a.chunk;
    return ssd::chunk_scan_tc_supported(q);
}

WsLayout ws_layout(const ssd_fwd_args& a) {
    const int64_t nc = (a.seqlen + a.chunk - 1) / a.chunk;
    const size_t vec = (size_t)a.batch * a.nheads * nc * a.chunk * sizeof(float);
    const size_t n_st = (size_t)a.batch * nc * a.nheads * a.headdim * a.dstate;
    const size_t elt = bf16_states(a) ? 2 : 4;
    WsLayout w;
    w.status = 0;
    w.dt = w.status + kAlign;
    w.cumA = w.dt + round_up(vec);
    w.states = w.cumA + round_up(vec);
    w.states_hl = w.states + round_up(n_st * elt);
    w.total = w.states_hl + (states_hilo(a) ? round_up(2 * n_st * 2) : 0);
    return w;
}

// Sizes and dtype only.
ssd_status check_fwd_sizes(const ssd_fwd_args* a) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->seqlen <= 0 || a->nheads <= 0 || a->headdim <= 0 ||
        a->dstate <= 0 || a->ngroups <= 0 || a->chunk <= 0)
        return SSD_ERR_INVALID_ARG;
    if (a->nheads % a->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->chunk > 256) return SSD_ERR_UNSUPPORTED;
    if (a->dstate % 4 != 0 || a->dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (a->headdim % 4 != 0) return SSD_ERR_UNSUPPORTED;
    const int64_t nc = (a->seqlen + a->chunk - 1) / a->chunk;
    if (a->batch > 65535 || nc * a->nheads > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

// Pointers of the inputs every step may read.
ssd_status check_fwd_inputs(const ssd_fwd_args* a) {
    if (!check_ptr(a->x, false, true) || !check_ptr(a->dt, false, false) ||
        !check_ptr(a->A, false, false) || !check_ptr(a->B, false, true) ||
        !check_ptr(a->C, false, true) || !check_ptr(a->D, true, false) ||
        !check_ptr(a->dt_bias, true, false) || !check_ptr(a->init_state, true, true) ||
        !check_ptr(a->z, true, true))
        return SSD_ERR_INVALID_ARG;
    return SSD_OK;
}

FwdParams make_params(const ssd_fwd_args* a) {
    FwdParams p;
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.nheads = a->nheads;
    p.headdim = a->headdim;
    p.dstate = a->dstate;
    p.ngroups = a->ngroups;
    p.chunk = a->chunk;
    p.nchunks = (a->seqlen + a->chunk - 1) / a->chunk;
    p.heads_per_group = a->nheads / a->ngroups;
    p.flags = a->flags;
    p.pdl = 0;
    p.fuse_cumsum = 0;
    p.states_f32 = bf16_states(*a) ? 0 : 1;
    p.x = a->x;
    p.dt_raw = a->dt;
    p.A = a->A;
    p.B = a->B;
    p.C = a->C;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.init_state = a->init_state;
    p.y = a->y;
    p.final_state = a->final_state;
    p.z = a->z;
    p.dt = p.cumA = nullptr;
    p.states = nullptr;
    p.states_hl = nullptr;
    p.status = nullptr;
    return p;
}

// The whole forward in one kernel: asked for with SSD_FLAG_SINGLE_PASS, for
// bf16 inputs in its shape range, unless the caller also asks for the CUDA
// cores, the split steps or the bf16-states mode.
bool use_fused(const ssd_fwd_args& a) {
    if (a.dtype != SSD_BF16 || !(a.flags & SSD_FLAG_SINGLE_PASS)) return false;
    if (a.flags & (SSD_FLAG_CUDA_CORES | SSD_FLAG_SPLIT_STEPS | SSD_FLAG_BF16_STATES)) return false;
    return ssd::fused_fwd_supported(make_params(&a));
}

// the last CUDA error a call of this library saw, per host thread
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

ssd_status to_status(cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    g_last_cuda_error = e;
    return SSD_ERR_CUDA;
}

cudaError_t run_cumsum(const FwdParams& p, int dtype, cudaStream_t s) {
    return dtype == SSD_BF16 ? ssd::launch_chunk_cumsum<__nv_bfloat16>(p, s)
                             : ssd::launch_chunk_cumsum<float>(p, s);
}
// The tensor-core kernels take bf16 inputs in their shape range unless the
// caller forces the CUDA-core path; everything else runs on the FFMA kernels.
// state passing is templated on the type the states are stored in
cudaError_t run_state_passing(const FwdParams& p, int dtype, cudaStream_t s) {
    return (dtype == SSD_BF16 && !p.states_f32) ? ssd::launch_state_passing<__nv_bfloat16>(p, s)
                                                : ssd::launch_state_passing<float>(p, s);
}
cudaError_t run_chunk_state(const FwdParams& p, int dtype, int flags, cudaStream_t s) {
    if (use_tc(dtype, flags) && ssd::chunk_state_tc_supported(p))
        return ssd::launch_chunk_state_tc(p, s);
    return dtype == SSD_BF16 ? ssd::launch_chunk_state_ffma<__nv_bfloat16>(p, s)
                             : ssd::launch_chunk_state_ffma<float>(p, s);
}
// The tensor-core chunk_scan takes the carried state as bf16 operands: the
// hi / lo pair that state passing wrote from the fp32 states, or, in the
// opt-in bf16-states mode, the bf16 states alone.  fp32 states without the
// pair (the step entry point) go to the CUDA-core kernel, which forms the
// state term in fp32.
cudaError_t run_chunk_scan(const FwdParams& p, int dtype, int flags, cudaStream_t s) {
    if (use_tc(dtype, flags) && (p.states_hl || !p.states_f32) && ssd::chunk_scan_tc_supported(p))
        return ssd::launch_chunk_scan_tc(p, s);
    return dtype == SSD_BF16 ? ssd::launch_chunk_scan_ffma<__nv_bfloat16>(p, s)
                             : ssd::launch_chunk_scan_ffma<float>(p, s);
}

// The forward's view of a backward call (the sizes, dtype and inputs).
ssd_fwd_args fwd_view(const ssd_bwd_args* a) {
    ssd_fwd_args f;
    memset(&f, 0, sizeof(f));
    f.batch = a->batch;
    f.seqlen = a->seqlen;
    f.nheads = a->nheads;
    f.headdim = a->headdim;
    f.dstate = a->dstate;
    f.ngroups = a->ngroups;
    f.chunk = a->chunk;
    f.dtype = a->dtype;
    f.flags = a->flags;
    f.x = a->x;
    f.dt = a->dt;
    f.A = a->A;
    f.B = a->B;
    f.C = a->C;
    f.D = a->D;
    f.dt_bias = a->dt_bias;
    f.init_state = a->init_state;
    return f;
}

struct BwdWs {
    size_t status, dt, cumA, states, dstates, xdxs, dyx, mterm, qterm, colw, roww, k4, partial, dBh,
        dCh, total;
};

BwdWs bwd_layout(const ssd_bwd_args& a) {
    const int64_t nc = (a.seqlen + a.chunk - 1) / a.chunk;
    const size_t vec = (size_t)a.batch * a.nheads * nc * a.chunk * sizeof(float);
    const size_t elt = a.dtype == SSD_BF16 ? 2 : 4;
    const size_t pn = (size_t)a.headdim * a.dstate;
    const size_t tok = (size_t)a.batch * a.nheads * a.seqlen * sizeof(float);
    const size_t per_head = a.ngroups < a.nheads
                                ? (size_t)a.batch * a.seqlen * a.nheads * a.dstate * sizeof(float)
                                : 0;
    BwdWs w;
    w.status = 0;
    w.dt = w.status + kAlign;
    w.cumA = w.dt + round_up(vec);
    w.states = w.cumA + round_up(vec);
    w.dstates = w.states + round_up((size_t)a.batch * nc * a.nheads * pn * elt);
    w.xdxs = w.dstates + round_up((size_t)a.batch * nc * a.nheads * pn * sizeof(float));
    w.dyx = w.xdxs + round_up(tok);
    w.mterm = w.dyx + round_up(tok);
    w.qterm = w.mterm + round_up(tok);
    w.colw = w.qterm + round_up(tok);
    w.roww = w.colw + round_up(tok);
    w.k4 = w.roww + round_up(tok * (size_t)(a.chunk / 64));
    w.partial = w.k4 + round_up((size_t)a.batch * a.nheads * nc * sizeof(float));
    w.dBh = w.partial + round_up((size_t)a.batch * a.nheads * nc * 3 * sizeof(float));
    w.dCh = w.dBh + round_up(per_head);
    w.total = w.dCh + round_up(per_head);
    return w;
}

ssd_status check_sel_sizes(const ssd_selective_scan_args* a) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->seqlen <= 0 || a->channels <= 0 || a->dstate <= 0 || a->chunk <= 0)
        return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->dstate % 4 != 0 || a->dstate > 32 || a->chunk * a->dstate > 4096 || a->batch > 65535)
        return SSD_ERR_UNSUPPORTED;
    const int64_t nc = (a->seqlen + a->chunk - 1) / a->chunk;
    if (nc > 65535 || (a->channels + 127) / 128 > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

struct SelWs {
    size_t S, sdt, total;
};

SelWs sel_layout(const ssd_selective_scan_args& a) {
    const int64_t nc = (a.seqlen + a.chunk - 1) / a.chunk;
    SelWs w;
    w.S = 0;
    w.sdt = round_up((size_t)a.batch * nc * a.channels * a.dstate * sizeof(float));
    w.total = w.sdt + round_up((size_t)a.batch * nc * a.channels * sizeof(float));
    return w;
}

// Largest opt-in shared memory per CTA on sm_100 (227 KB).
constexpr size_t kMaxSmemOptin = 232448;

ssd_status check_bwd_sizes(const ssd_bwd_args* a) {
    if (!a) return SSD_ERR_INVALID_ARG;
    const ssd_fwd_args f = fwd_view(a);
    const ssd_status st = check_fwd_sizes(&f);
    if (st != SSD_OK) return st;
    const int64_t nc = (a->seqlen + a->chunk - 1) / a->chunk;
    if (a->chunk % 64 != 0 || a->headdim > 128 || a->dstate > 128 || nc > 65535)
        return SSD_ERR_UNSUPPORTED;
    if (ssd::bwd_smem_bytes(a->headdim, a->dstate, a->chunk) > kMaxSmemOptin)
        return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

}  // namespace

namespace {
std::atomic<int64_t> g_withhold[3] = {{-1}, {-1}, {-1}};
}  // namespace

namespace ssd {
int64_t debug_withhold(int what) {
    return (what >= 0 && what < 3) ? g_withhold[what].load(std::memory_order_relaxed) : -1;
}
}  // namespace ssd

extern "C" {

size_t ssd_fwd_workspace_size(const ssd_fwd_args* args) {
    if (check_fwd_sizes(args) != SSD_OK) return 0;
    if (use_fused(*args)) return ssd::fused_fwd_workspace_bytes(make_params(args));
    return ws_layout(*args).total;
}

int ssd_fwd_tensor_core_steps(const ssd_fwd_args* a) {
    if (check_fwd_sizes(a) != SSD_OK || !use_tc(a->dtype, a->flags)) return 0;
    if (use_fused(*a)) return SSD_TC_CHUNK_STATE | SSD_TC_CHUNK_SCAN | SSD_TC_FUSED;
    const FwdParams p = make_params(a);
    return (ssd::chunk_state_tc_supported(p) ? SSD_TC_CHUNK_STATE : 0) |
           ((states_hilo(*a) || bf16_states(*a)) && ssd::chunk_scan_tc_supported(p) ? SSD_TC_CHUNK_SCAN : 0);
}

ssd_status ssd_fwd(const ssd_fwd_args* a, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if ((st = check_fwd_inputs(a)) != SSD_OK) return st;
    if (!check_ptr(a->y, false, true) || !check_ptr(a->final_state, true, true))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_fused(*a)) {
        FwdParams p = make_params(a);
        if (!a->workspace || a->workspace_bytes < ssd::fused_fwd_workspace_bytes(p) ||
            !check_ptr(a->workspace, false, true))
            return SSD_ERR_INVALID_ARG;
        return to_status(ssd::launch_fused_fwd(p, a->workspace, s));
    }
    const WsLayout w = ws_layout(*a);
    if (!a->workspace || a->workspace_bytes < w.total || !check_ptr(a->workspace, false, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    char* ws = static_cast<char*>(a->workspace);
    p.dt = reinterpret_cast<float*>(ws + w.dt);
    p.cumA = reinterpret_cast<float*>(ws + w.cumA);
    p.states = ws + w.states;
    p.states_hl = states_hilo(*a) ? ws + w.states_hl : nullptr;
    p.status = reinterpret_cast<int*>(ws + w.status);
    // The first kernel is a plain launch (it waits for all earlier work on
    // the stream); the later ones go out with programmatic dependent launch,
    // so their set-up overlaps the previous kernel's tail.  The tensor-core
    // chunk_state forms dt and cumA itself, which saves step 1's launch.
    cudaError_t e = cudaSuccess;
    const bool fused = use_tc(a->dtype, a->flags) && ssd::chunk_state_tc_supported(p);
    if (!fused) {
        e = run_cumsum(p, a->dtype, s);
        p.pdl = 1;
    } else {
        p.fuse_cumsum = 1;
    }
    if (e == cudaSuccess) e = run_chunk_state(p, a->dtype, a->flags, s);
    p.pdl = 1;
    p.fuse_cumsum = 0;
    if (e == cudaSuccess) e = run_state_passing(p, a->dtype, s);
    if (e == cudaSuccess) e = run_chunk_scan(p, a->dtype, a->flags, s);
    return to_status(e);
}

ssd_status ssd_fwd_check_status(const ssd_fwd_args* a, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    // both layouts keep the status word at the start of the workspace
    const size_t need = ssd_fwd_workspace_size(a);
    if (!a->workspace || a->workspace_bytes < need || !check_ptr(a->workspace, false, true))
        return SSD_ERR_INVALID_ARG;
    int v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, static_cast<char*>(a->workspace), sizeof(int),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SSD_ERR_CUDA;
    return v == 0 ? SSD_OK : static_cast<ssd_status>(v);
}

size_t ssd_bwd_workspace_size(const ssd_bwd_args* args) {
    if (check_bwd_sizes(args) != SSD_OK) return 0;
    return bwd_layout(*args).total;
}

ssd_status ssd_bwd(const ssd_bwd_args* a, void* stream) {
    ssd_status st = check_bwd_sizes(a);
    if (st != SSD_OK) return st;
    const ssd_fwd_args f = fwd_view(a);
    if ((st = check_fwd_inputs(&f)) != SSD_OK) return st;
    if (!check_ptr(a->dy, false, true) || !check_ptr(a->d_final, true, true) ||
        !check_ptr(a->dx, false, false) || !check_ptr(a->ddt, false, false) ||
        !check_ptr(a->dA, false, false) || !check_ptr(a->dB, false, false) ||
        !check_ptr(a->dC, false, false) || !check_ptr(a->dD, true, false) ||
        !check_ptr(a->ddt_bias, true, false) || !check_ptr(a->d_init, true, true))
        return SSD_ERR_INVALID_ARG;
    const BwdWs w = bwd_layout(*a);
    if (!a->workspace || a->workspace_bytes < w.total || !check_ptr(a->workspace, false, true))
        return SSD_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(a->workspace);
    FwdParams p = make_params(&f);
    p.states_f32 = 0;  // the recompute keeps its states in the input dtype
    p.dt = reinterpret_cast<float*>(ws + w.dt);
    p.cumA = reinterpret_cast<float*>(ws + w.cumA);
    p.states = ws + w.states;
    p.status = reinterpret_cast<int*>(ws + w.status);
    p.final_state = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the forward recompute: dt, cumA and the states entering each chunk
    cudaError_t e = cudaSuccess;
    const bool fused = use_tc(a->dtype, a->flags) && ssd::chunk_state_tc_supported(p);
    if (!fused) {
        e = run_cumsum(p, a->dtype, s);
        p.pdl = 1;
    } else {
        p.fuse_cumsum = 1;
    }
    if (e == cudaSuccess) e = run_chunk_state(p, a->dtype, a->flags, s);
    p.pdl = 1;
    p.fuse_cumsum = 0;
    if (e == cudaSuccess) e = run_state_passing(p, a->dtype, s);
    if (e != cudaSuccess) return to_status(e);
    ssd::BwdParams bp;
    bp.f = p;
    bp.f.pdl = 0;
    bp.dy = a->dy;
    bp.d_final = a->d_final;
    bp.dx = a->dx;
    bp.ddt = a->ddt;
    bp.dA = a->dA;
    bp.dB = a->dB;
    bp.dC = a->dC;
    bp.dD = a->dD;
    bp.ddt_bias = a->ddt_bias;
    bp.d_init = a->d_init;
    bp.dstates = reinterpret_cast<float*>(ws + w.dstates);
    const bool per_head = a->ngroups < a->nheads;
    bp.dB_h = per_head ? reinterpret_cast<float*>(ws + w.dBh) : nullptr;
    bp.dC_h = per_head ? reinterpret_cast<float*>(ws + w.dCh) : nullptr;
    bp.xdxs = reinterpret_cast<float*>(ws + w.xdxs);
    bp.dyx = reinterpret_cast<float*>(ws + w.dyx);
    bp.mterm = reinterpret_cast<float*>(ws + w.mterm);
    bp.qterm = reinterpret_cast<float*>(ws + w.qterm);
    bp.colw = reinterpret_cast<float*>(ws + w.colw);
    bp.roww = reinterpret_cast<float*>(ws + w.roww);
    bp.k4 = reinterpret_cast<float*>(ws + w.k4);
    bp.partial = reinterpret_cast<float*>(ws + w.partial);
    bp.rblk = (use_tc(a->dtype, a->flags) && ssd::bwd_tc_supported(p)) ? 128 : 64;
    return to_status(a->dtype == SSD_BF16 ? ssd::launch_ssd_bwd<__nv_bfloat16>(bp, s)
                                          : ssd::launch_ssd_bwd<float>(bp, s));
}

ssd_status ssd_bwd_check_status(const ssd_bwd_args* a, void* stream) {
    ssd_status st = check_bwd_sizes(a);
    if (st != SSD_OK) return st;
    const BwdWs w = bwd_layout(*a);
    if (!a->workspace || a->workspace_bytes < w.total || !check_ptr(a->workspace, false, true))
        return SSD_ERR_INVALID_ARG;
    int v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, static_cast<char*>(a->workspace) + w.status, sizeof(int),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SSD_ERR_CUDA;
    return v == 0 ? SSD_OK : static_cast<ssd_status>(v);
}

size_t ssd_selective_scan_workspace_size(const ssd_selective_scan_args* args) {
    if (check_sel_sizes(args) != SSD_OK) return 0;
    return sel_layout(*args).total;
}

ssd_status ssd_selective_scan(const ssd_selective_scan_args* a, void* stream) {
    const ssd_status st = check_sel_sizes(a);
    if (st != SSD_OK) return st;
    if (!check_ptr(a->x, false, false) || !check_ptr(a->dt, false, false) ||
        !check_ptr(a->A, false, true) || !check_ptr(a->B, false, false) ||
        !check_ptr(a->C, false, false) || !check_ptr(a->D, true, false) ||
        !check_ptr(a->dt_bias, true, false) || !check_ptr(a->init_state, true, true) ||
        !check_ptr(a->y, false, false) || !check_ptr(a->final_state, true, true))
        return SSD_ERR_INVALID_ARG;
    const SelWs w = sel_layout(*a);
    if (!a->workspace || a->workspace_bytes < w.total || !check_ptr(a->workspace, false, true))
        return SSD_ERR_INVALID_ARG;
    ssd::SelParams p;
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.channels = a->channels;
    p.dstate = a->dstate;
    p.chunk = a->chunk;
    p.nchunks = (a->seqlen + a->chunk - 1) / a->chunk;
    p.x = a->x;
    p.dt_raw = a->dt;
    p.A = a->A;
    p.B = a->B;
    p.C = a->C;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.init_state = a->init_state;
    p.y = a->y;
    p.final_state = a->final_state;
    char* ws = static_cast<char*>(a->workspace);
    p.S = reinterpret_cast<float*>(ws + w.S);
    p.sdt = reinterpret_cast<float*>(ws + w.sdt);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return to_status(a->dtype == SSD_BF16 ? ssd::launch_selective_scan<__nv_bfloat16>(p, false, s)
                                          : ssd::launch_selective_scan<float>(p, false, s));
}

ssd_status ssd_selective_state_update(const ssd_selective_state_update_args* a, void* stream) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->channels <= 0 || a->dstate <= 0) return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->dstate % 4 != 0 || a->dstate > 32) return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(a->state, false, true) || !check_ptr(a->x, false, false) ||
        !check_ptr(a->dt, false, false) || !check_ptr(a->A, false, true) ||
        !check_ptr(a->B, false, true) || !check_ptr(a->C, false, true) ||
        !check_ptr(a->D, true, false) || !check_ptr(a->dt_bias, true, false) ||
        !check_ptr(a->y, false, false))
        return SSD_ERR_INVALID_ARG;
    ssd::SelParams p;
    memset(&p, 0, sizeof(p));
    p.batch = a->batch;
    p.seqlen = 1;
    p.channels = a->channels;
    p.dstate = a->dstate;
    p.x = a->x;
    p.dt_raw = a->dt;
    p.A = a->A;
    p.B = a->B;
    p.C = a->C;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.y = a->y;
    p.S = a->state;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return to_status(a->dtype == SSD_BF16 ? ssd::launch_selective_scan<__nv_bfloat16>(p, true, s)
                                          : ssd::launch_selective_scan<float>(p, true, s));
}

ssd_status ssd_chunk_cumsum(const ssd_fwd_args* a, float* dt_out, float* cumA_out,
                            void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if (!check_ptr(a->dt, false, false) || !check_ptr(a->A, false, false) ||
        !check_ptr(a->dt_bias, true, false) || !check_ptr(dt_out, false, true) ||
        !check_ptr(cumA_out, false, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.dt = dt_out;
    p.cumA = cumA_out;
    return to_status(run_cumsum(p, a->dtype, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_state(const ssd_fwd_args* a, const float* dt, const float* cumA,
                           void* states, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if ((st = check_fwd_inputs(a)) != SSD_OK) return st;
    if (!check_ptr(dt, false, true) || !check_ptr(cumA, false, true) ||
        !check_ptr(states, false, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.dt = const_cast<float*>(dt);
    p.cumA = const_cast<float*>(cumA);
    p.states = states;
    return to_status(run_chunk_state(p, a->dtype, a->flags, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_state_passing(const ssd_fwd_args* a, const float* cumA, void* states,
                             void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if (!check_ptr(cumA, false, true) || !check_ptr(states, false, true) ||
        !check_ptr(a->init_state, true, true) || !check_ptr(a->final_state, true, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.cumA = const_cast<float*>(cumA);
    p.states = states;
    return to_status(run_state_passing(p, a->dtype, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_scan(const ssd_fwd_args* a, const float* dt, const float* cumA,
                          const void* states, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if ((st = check_fwd_inputs(a)) != SSD_OK) return st;
    if (!check_ptr(a->y, false, true) || !check_ptr(dt, false, true) ||
        !check_ptr(cumA, false, true) || !check_ptr(states, false, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.dt = const_cast<float*>(dt);
    p.cumA = const_cast<float*>(cumA);
    p.states = const_cast<void*>(states);
    return to_status(run_chunk_scan(p, a->dtype, a->flags, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_state_passing_hilo(const ssd_fwd_args* a, const float* cumA, const float* states,
                                  void* states_hl, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if (!states_hilo(*a)) return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(cumA, false, true) || !check_ptr(states, false, true) ||
        !check_ptr(states_hl, false, true) || !check_ptr(a->init_state, true, true) ||
        !check_ptr(a->final_state, true, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.cumA = const_cast<float*>(cumA);
    p.states = const_cast<float*>(states);
    p.states_hl = states_hl;
    return to_status(run_state_passing(p, a->dtype, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_scan_hilo(const ssd_fwd_args* a, const float* dt, const float* cumA,
                               const void* states_hl, void* stream) {
    ssd_status st = check_fwd_sizes(a);
    if (st != SSD_OK) return st;
    if (!states_hilo(*a)) return SSD_ERR_UNSUPPORTED;
    if ((st = check_fwd_inputs(a)) != SSD_OK) return st;
    if (!check_ptr(a->y, false, true) || !check_ptr(dt, false, true) ||
        !check_ptr(cumA, false, true) || !check_ptr(states_hl, false, true))
        return SSD_ERR_INVALID_ARG;
    FwdParams p = make_params(a);
    p.dt = const_cast<float*>(dt);
    p.cumA = const_cast<float*>(cumA);
    p.states_hl = const_cast<void*>(states_hl);
    return to_status(run_chunk_scan(p, a->dtype, a->flags, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_causal_conv1d(const ssd_conv1d_args* a, void* stream) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->seqlen <= 0 || a->channels <= 0 || a->width <= 0)
        return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->width > 8 || a->channels % (a->dtype == SSD_BF16 ? 8 : 4) != 0 || a->batch > 65535)
        return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(a->x, false, true) || !check_ptr(a->weight, false, false) ||
        !check_ptr(a->bias, true, false) || !check_ptr(a->init_state, true, false) ||
        !check_ptr(a->y, false, true) || !check_ptr(a->final_state, true, false))
        return SSD_ERR_INVALID_ARG;
    ssd::ConvParams p;
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.channels = a->channels;
    p.width = a->width;
    p.activation = a->activation ? 1 : 0;
    p.x = a->x;
    p.weight = a->weight;
    p.bias = a->bias;
    p.init_state = a->init_state;
    p.y = a->y;
    p.final_state = a->final_state;
    p.update_state = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return to_status(a->dtype == SSD_BF16 ? ssd::launch_conv1d<__nv_bfloat16>(p, false, s)
                                          : ssd::launch_conv1d<float>(p, false, s));
}

ssd_status ssd_conv1d_check_status(void* stream) {
    int v = 0;
    if (ssd::conv1d_take_status(&v, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return SSD_ERR_CUDA;
    return v == 0 ? SSD_OK : static_cast<ssd_status>(v);
}

ssd_status ssd_conv1d_update(const ssd_conv1d_update_args* a, void* stream) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->channels <= 0 || a->width <= 0) return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->width > 8 || a->channels % (a->dtype == SSD_BF16 ? 8 : 4) != 0)
        return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(a->state, a->width == 1, true) || !check_ptr(a->x, false, true) ||
        !check_ptr(a->weight, false, true) || !check_ptr(a->bias, true, true) ||
        !check_ptr(a->y, false, true))
        return SSD_ERR_INVALID_ARG;
    ssd::ConvParams p;
    p.batch = a->batch;
    p.seqlen = 1;
    p.channels = a->channels;
    p.width = a->width;
    p.activation = a->activation ? 1 : 0;
    p.x = a->x;
    p.weight = a->weight;
    p.bias = a->bias;
    p.init_state = nullptr;
    p.y = a->y;
    p.final_state = nullptr;
    p.update_state = a->state;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return to_status(a->dtype == SSD_BF16 ? ssd::launch_conv1d<__nv_bfloat16>(p, true, s)
                                          : ssd::launch_conv1d<float>(p, true, s));
}

ssd_status ssd_gated_rmsnorm(const ssd_gated_rmsnorm_args* a, void* stream) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->rows <= 0 || a->channels <= 0 || a->group <= 0) return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (!(a->eps >= 0.0f) || !(a->eps <= 3.4e38f)) return SSD_ERR_INVALID_ARG;
    if (a->channels % a->group != 0 || a->group % (a->dtype == SSD_BF16 ? 8 : 4) != 0)
        return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(a->y, false, true) || !check_ptr(a->z, true, true) ||
        !check_ptr(a->weight, false, true) || !check_ptr(a->out, false, true))
        return SSD_ERR_INVALID_ARG;
    ssd::NormParams p;
    p.rows = a->rows;
    p.channels = a->channels;
    p.group = a->group;
    p.eps = a->eps;
    p.y = a->y;
    p.z = a->z;
    p.weight = a->weight;
    p.out = a->out;
    return to_status(ssd::launch_gated_rmsnorm(p, a->dtype == SSD_BF16,
                                               static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_state_update(const ssd_state_update_args* a, void* stream) {
    if (!a) return SSD_ERR_INVALID_ARG;
    if (a->batch <= 0 || a->nheads <= 0 || a->headdim <= 0 || a->dstate <= 0 ||
        a->ngroups <= 0 || a->nheads % a->ngroups != 0)
        return SSD_ERR_INVALID_ARG;
    if (a->dtype != SSD_F32 && a->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (a->dstate != 16 && a->dstate != 32 && a->dstate != 64 && a->dstate != 128 &&
        a->dstate != 256)
        return SSD_ERR_UNSUPPORTED;
    if (!check_ptr(a->state, false, true) || !check_ptr(a->x, false, false) ||
        !check_ptr(a->dt, false, false) || !check_ptr(a->A, false, false) ||
        !check_ptr(a->B, false, true) || !check_ptr(a->C, false, true) ||
        !check_ptr(a->D, true, false) || !check_ptr(a->dt_bias, true, false) ||
        !check_ptr(a->y, false, false) || !check_ptr(a->z, true, false))
        return SSD_ERR_INVALID_ARG;
    DecodeParams p;
    p.batch = a->batch;
    p.nheads = a->nheads;
    p.headdim = a->headdim;
    p.dstate = a->dstate;
    p.ngroups = a->ngroups;
    p.heads_per_group = a->nheads / a->ngroups;
    p.state = a->state;
    p.x = a->x;
    p.dt_raw = a->dt;
    p.A = a->A;
    p.B = a->B;
    p.C = a->C;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.y = a->y;
    p.z = a->z;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = a->dtype == SSD_BF16 ? ssd::launch_state_update<__nv_bfloat16>(p, s)
                                         : ssd::launch_state_update<float>(p, s);
    return to_status(e);
}

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT";
        default: return "SSD_ERR_UNKNOWN";
    }
}

const char* ssd_last_cuda_error(void) {
    return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

void ssd_debug_set_withhold(int what, int64_t index) {
    if (what >= 0 && what < 3) g_withhold[what].store(index < 0 ? -1 : index, std::memory_order_relaxed);
}

const char* ssd_version(void) { return "ssd_b200 0.1.0 (sm_100a)"; }

}  // extern "C"
