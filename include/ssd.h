/*
 * ssd.h -- C ABI of libssd_b200.so: the Mamba-2 SSD selective scan forward and
 * the single-token decode state update, on NVIDIA B200 (sm_100a).
 *
 * The operation (pages: "MAMBA-2 Reference Implementations Comparison",
 * section 2.2 "SSD Mathematical Formulation" and section 3.2 "Selective Scan
 * Algorithm"; "MAMBA-2 Implementation Gaps", Gap 1 "SSD Algorithm", Gap 3
 * "dt (Time Step) Parameter", Gap 4 "D (Skip Connection) Parameter"):
 *
 *   dt_t = softplus(dt_raw_t + dt_bias_h)          (no clamp)
 *   h_t  = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T      h: [P x N]
 *   y_t  = C_t . h_t + D_h * x_t                     (h_t after the update)
 *
 * with A_h a scalar per head (normally negative), B_t, C_t shared by the heads
 * of a group (head h reads group h / (nheads / ngroups)).  The forward pass
 * computes this chunkwise, the chunked SSD of "MAMBA-2 Implementation Gaps",
 * Gap 1: chunk_cumsum -> chunk_state -> state_passing -> chunk_scan.  For bf16
 * inputs the first two steps run as one tensor-core kernel and the last as
 * another, the chunk states staying fp32 in the workspace (they reach the
 * tensor cores as bf16 hi + lo halves); SSD_FLAG_SINGLE_PASS runs all four as
 * one kernel instead (the carried state stays fp32 and crosses between tiles
 * on chip and through a small ring in the workspace).
 *
 * Layouts: row-major, innermost index last, densely packed (no strides):
 *   x, y          [batch, seqlen, nheads, headdim]     dtype
 *   dt (raw)      [batch, seqlen, nheads]              dtype
 *   B, C          [batch, seqlen, ngroups, dstate]     dtype
 *   A, D, dt_bias [nheads]                             fp32
 *   state         [batch, nheads, headdim, dstate]     fp32
 * "dtype" is SSD_F32 (fp32) or SSD_BF16 (bfloat16); arithmetic is fp32 either
 * way (bf16 operands enter the tensor cores, products accumulate in fp32) and y
 * is rounded to dtype (round to nearest even).
 *
 * Ownership and memory: every pointer is a DEVICE pointer owned by the caller
 * (cudaMalloc, a torch tensor, ...).  The library allocates no memory and keeps
 * no state between calls other than per-device kernel attributes.  Scratch
 * memory for ssd_fwd comes from the caller (ssd_fwd_workspace_size).
 * x, B, C, y, init_state, final_state and workspace must be 16-byte aligned.
 *
 * Calling convention: calls are asynchronous on `stream` (a cudaStream_t passed
 * as void*; NULL = the legacy default stream) and never synchronise the host.
 * Arguments are validated before anything is launched; on an error nothing is
 * launched and nothing is written.  There is no CPU fallback.
 *
 * Errors: SSD_ERR_INVALID_ARG for a NULL required pointer, a pointer the CUDA
 * runtime does not know as device memory, a misaligned pointer, a size <= 0 or
 * nheads % ngroups != 0, a too-small workspace; SSD_ERR_UNSUPPORTED for sizes
 * outside the kernels' range (listed per call); SSD_ERR_CUDA when a launch
 * fails (cudaGetLastError after the launch).
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,
    SSD_ERR_UNSUPPORTED = 2,
    SSD_ERR_CUDA = 3,
    SSD_ERR_TIMEOUT = 4
} ssd_status;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/* Arguments of the forward scan and of its four steps.
 *   chunk        Q, tokens per chunk; the last chunk may be shorter
 *                (nc = ceil(seqlen / chunk) chunks).
 *   D, dt_bias   may be NULL (= 0).
 *   init_state   may be NULL (= zero state): the state before token 0.
 *   y            output [batch, seqlen, nheads, headdim], dtype.
 *   final_state  may be NULL: receives h after the last token, fp32.
 *   z            may be NULL: the output gate, [batch, seqlen, nheads,
 *                headdim] in dtype; when given, y = (C h + D x) silu(z),
 *                silu(z) = z / (1 + e^-z) (the output gating of the page
 *                "MAMBA-2 Reference Implementations Comparison", sections 3
 *                and 6.1), applied in the kernel that writes y.  The gate does
 *                not touch the carried state.
 * Supported: 1 <= chunk <= 256; dstate a multiple of 4, <= 256; headdim a
 * multiple of 4.  bf16 inputs run the forward as three tensor-core (tcgen05)
 * kernels where they apply: chunk_state (with step 1 folded in; headdim in
 * {32, 64, 128}, dstate in {64, 128, 256}, 128/headdim dividing the heads per
 * group), state passing, and chunk_scan (headdim 64, dstate 64 or 128, chunk
 * 128 or 256); the chunk states stay fp32 and reach chunk_scan as hi / lo
 * bf16 halves.  Steps outside those ranges run in fp32 on the CUDA cores.
 * With SSD_FLAG_SINGLE_PASS, bf16 inputs with headdim 64 and dstate 64 or 128
 * run the whole forward as one kernel instead (its tiling is its own: the
 * result does not depend on `chunk`, which the chunked form leaves exact up
 * to rounding).  fp32 inputs always take the CUDA-core path (its exact fp32
 * arithmetic is what the 1e-4 agreement needs). */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk;
    int32_t dtype;          /* ssd_dtype of x, dt, B, C and y */
    int32_t flags;          /* SSD_FLAG_* below; 0 = defaults */
    const void* x;
    const void* dt;         /* raw dt, before bias and softplus */
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    const float* init_state;
    void* y;
    float* final_state;
    void* workspace;        /* device scratch, >= ssd_fwd_workspace_size() */
    size_t workspace_bytes;
    const void* z;          /* optional output gate (see above); NULL = none */
} ssd_fwd_args;

/* flags */
#define SSD_FLAG_CUDA_CORES 1   /* force the CUDA-core (FFMA) path */
#define SSD_FLAG_WHOLE_GROUPS 2 /* tensor-core chunk_scan (bf16-states mode): one CTA
                                   per whole group of heads */
#define SSD_FLAG_SPLIT_STEPS 4  /* bf16: the forward as its separate step kernels
                                   (the default; overrides SSD_FLAG_SINGLE_PASS) */
#define SSD_FLAG_BF16_STATES 8  /* bf16, opt-in: the split steps with the chunk
                                   states stored in bf16 and the carried state
                                   entering the tensor-core state term as one bf16
                                   operand.  Faster than the split fp32 steps but
                                   OUTSIDE the stated bf16 tolerance for some inputs
                                   (the carried state's rounding under cancellation
                                   in C . H); never the default */
#define SSD_FLAG_SINGLE_PASS 16 /* bf16, opt-in: the whole forward as one kernel
                                   (headdim 64, dstate 64 or 128): tiles of 128
                                   tokens, the carried state handed from tile to
                                   tile through the workspace.  Within the same
                                   tolerance as the default; measured slower on
                                   B200 than the three kernels (its per-tile
                                   pipeline is latency-bound) */

/* Bytes of device workspace ssd_fwd needs for these sizes (0 on invalid
 * sizes).  Only sizes, dtype and flags are read; pointers may be NULL. */
size_t ssd_fwd_workspace_size(const ssd_fwd_args* args);

/* Which steps of ssd_fwd run on the tensor cores for these sizes, dtype and
 * flags: bit 0 = chunk_state, bit 1 = chunk_scan, bit 2 = the whole forward in
 * one kernel (SSD_FLAG_SINGLE_PASS; bits 0 and 1 are then set too) (0 = all
 * on CUDA cores, or invalid sizes).  Host-only; pointers are not read. */
#define SSD_TC_CHUNK_STATE 1
#define SSD_TC_CHUNK_SCAN 2
#define SSD_TC_FUSED 4
int ssd_fwd_tensor_core_steps(const ssd_fwd_args* args);

/* The whole forward scan: y (and final_state) from x, dt, A, B, C, D,
 * dt_bias, init_state.  Stream-ordered; the workspace must not be shared with
 * another call in flight. */
ssd_status ssd_fwd(const ssd_fwd_args* args, void* stream);

/* ssd_fwd for callers that cannot allocate device memory (there is no
 * counterpart on the pages: this is a deployment variant).  Some callers only
 * hold the input and output buffers their host application hands them --
 * plugins and runtime extensions with no access to an allocator, or
 * latency-critical code that must not risk a cudaMalloc's device-wide
 * synchronisation.  This entry point ignores args->workspace and
 * args->workspace_bytes and takes the scratch from a buffer of
 * SSD_NO_ALLOC_SCRATCH_BYTES compiled into the library.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   - Sizes whose ssd_fwd_workspace_size() exceeds the buffer are rejected
 *     with SSD_ERR_UNSUPPORTED before anything is launched.
 *   - The buffer is reserved on a device when the library's device code is
 *     loaded there and is held until the process exits.  Under CUDA's lazy
 *     module loading (the default since CUDA 12.2) that happens at the first
 *     call on the device, which can then fail with SSD_ERR_CUDA for lack of
 *     device memory and may synchronise the device.  That first call also
 *     looks up the buffer's device address (cudaGetSymbolAddress, that device
 *     current) and caches it.  So make one call per device at initialisation,
 *     before any stream capture and before the latency-critical phase.
 *   - All calls share the one buffer: calls that can overlap on the GPU (on
 *     different streams without ordering between them, or from different host
 *     threads) race and give wrong results; serialise them.  The buffer keeps
 *     the last call's contents; every call writes each scratch entry before it
 *     reads it, so nothing needs clearing between calls.
 * Everything else (arguments, layouts, errors, asynchrony) is as ssd_fwd. */
#define SSD_NO_ALLOC_SCRATCH_BYTES (16u << 20)
ssd_status ssd_fwd_no_alloc(const ssd_fwd_args* args, void* stream);

/* SSD_NO_ALLOC_SCRATCH_BYTES as compiled into this library (bindings read the
 * limit from here rather than repeating the constant). */
size_t ssd_fwd_no_alloc_scratch_bytes(void);

/* ssd_fwd_check_status for ssd_fwd_no_alloc: synchronises `stream` and returns
 * the device status of the last ssd_fwd_no_alloc call on the current device
 * (SSD_OK, or SSD_ERR_TIMEOUT when a kernel gave up on a bounded wait and the
 * outputs are invalid).  Only sizes, dtype and flags of `args` are read; they
 * must be those of that call.  SSD_ERR_UNSUPPORTED for sizes beyond the
 * buffer, SSD_ERR_INVALID_ARG for invalid sizes. */
ssd_status ssd_fwd_no_alloc_check_status(const ssd_fwd_args* args, void* stream);

/* Synchronises `stream` and returns the device status of the last ssd_fwd
 * call that used this workspace: SSD_OK, or SSD_ERR_TIMEOUT when a kernel gave
 * up on a bounded wait (it then stops early and its outputs are invalid).
 * Each ssd_fwd call resets the status at its start.  The status word is the
 * workspace's first 4 bytes in every path. */
ssd_status ssd_fwd_check_status(const ssd_fwd_args* args, void* stream);

/* ---- the four steps of ssd_fwd, exported one by one -------------------- */
/* Each reads the fields of `args` it needs and the intermediate buffers named
 * in its signature (device, caller-owned, 16-byte aligned):
 *   dt_out, cumA_out  [batch, nheads, nc, chunk]                 fp32
 *   states            [batch, nc, nheads, headdim, dstate]       fp32
 * (with SSD_FLAG_BF16_STATES and bf16 inputs, `states` is bf16 instead; the
 * carry across chunks is fp32 in registers either way).
 */

/* Step 1: dt = softplus(dt_raw + dt_bias) and the inclusive in-chunk
 * cumulative sum of dt * A_h.  Entries past the end of a short last chunk hold
 * dt = 0 and the chunk's last cumulative value. */
ssd_status ssd_chunk_cumsum(const ssd_fwd_args* args, float* dt_out, float* cumA_out,
                            void* stream);

/* Step 2: each chunk's local state, as if the chunk started from zero:
 * S_c[p,n] = sum_{l in c} exp(cumA[last] - cumA[l]) * dt[l] * x[l,p] * B[l,n]. */
ssd_status ssd_chunk_state(const ssd_fwd_args* args, const float* dt, const float* cumA,
                           void* states, void* stream);

/* Step 3: in place over `states`: reads the local states S_c and replaces each
 * with the state entering chunk c, H_{c-1} = exp(cumA_{c-1}[last]) H_{c-2} +
 * S_{c-1} (H before chunk 0 = init_state or 0); writes final_state if given. */
ssd_status ssd_state_passing(const ssd_fwd_args* args, const float* cumA, void* states,
                             void* stream);

/* Step 4: y[l,p] = sum_{j<=l in chunk} exp(cumA[l]-cumA[j]) (C_l.B_j) dt[j] x[j,p]
 *                 + exp(cumA[l]) sum_n C_l[n] H_in[p,n] + D x[l,p],
 * with H_in the state entering the chunk (states after step 3).  With fp32
 * states the state term is formed in fp32 on the CUDA cores; the tensor-core
 * kernel takes the _hilo form below. */
ssd_status ssd_chunk_scan(const ssd_fwd_args* args, const float* dt, const float* cumA,
                          const void* states, void* stream);

/* Steps 3 and 4 as ssd_fwd runs them for bf16 inputs on the tensor cores
 * (ssd_fwd_tensor_core_steps reports SSD_TC_CHUNK_SCAN; SSD_ERR_UNSUPPORTED
 * otherwise).  The state entering each chunk goes to chunk_scan as two bf16
 * halves, hi = bf16(H) and lo = bf16(H - hi), so that the tensor-core state
 * term C . (hi + lo) carries the fp32 state to about 2^-17 of its size:
 *   states_hl  [2][batch, nc, nheads, headdim, dstate] bf16 (hi, then lo),
 *              device, caller-owned, 16-byte aligned.
 * ssd_state_passing_hilo reads the fp32 local states of step 2 (`states`, not
 * modified) and writes the entering states to states_hl (and final_state if
 * given); ssd_chunk_scan_hilo writes y from states_hl. */
ssd_status ssd_state_passing_hilo(const ssd_fwd_args* args, const float* cumA,
                                  const float* states, void* states_hl, void* stream);
ssd_status ssd_chunk_scan_hilo(const ssd_fwd_args* args, const float* dt, const float* cumA,
                               const void* states_hl, void* stream);

/* ---- backward --------------------------------------------------------------- */
/* The backward pass of ssd_fwd (without the output gate): the gradients of
 *   J = sum_t dy_t . y_t + d_final : final_state
 * with respect to every input, i.e. what reverse-mode differentiation of the
 * recurrence of "MAMBA-2 Reference Implementations Comparison", section 2.2
 * returns (the page "Agent 230: Comprehensive MAMBA-2 Implementation
 * Comparison", section 6, Gradient Computation, takes the gradients of A, B,
 * C and delta (dt); x, D, dt_bias and the initial state are the other
 * inputs).  The forward is recomputed inside the call (dt, the
 * chunk states) from the same inputs.
 *   sizes, dtype, x, dt, A, B, C, D, dt_bias, init_state: as ssd_fwd_args.
 *   dy        [batch, seqlen, nheads, headdim] dtype: dJ/dy.
 *   d_final   [batch, nheads, headdim, dstate] fp32, or NULL (= 0).
 *   dx        [batch, seqlen, nheads, headdim] dtype.
 *   ddt       [batch, seqlen, nheads] dtype: the gradient of the RAW dt.
 *   dB, dC    [batch, seqlen, ngroups, dstate] dtype (summed over the heads of
 *             a group).
 *   dA [nheads] fp32; dD, ddt_bias [nheads] fp32 or NULL (not written); all
 *             three summed over batch and time.
 *   d_init    [batch, nheads, headdim, dstate] fp32, or NULL (not written).
 * All gradients are accumulated in fp32 and rounded once to their dtype; sums
 * over heads and batch rows run in a fixed order, so repeated calls give
 * bitwise-identical results.
 * Supported: as ssd_fwd, and chunk a multiple of 64, headdim and dstate at
 * most 128 with the per-chunk tiles fitting the device's shared memory
 * (else SSD_ERR_UNSUPPORTED); dy, d_final and d_init 16-byte aligned.
 * Errors, stream ordering and the workspace rules as for ssd_fwd. */
typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups, chunk;
    int32_t dtype;
    int32_t flags;          /* SSD_FLAG_* for the forward recompute */
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    const float* init_state;
    const void* dy;
    const float* d_final;
    void* dx;
    void* ddt;
    float* dA;
    void* dB;
    void* dC;
    float* dD;
    float* ddt_bias;
    float* d_init;
    void* workspace;        /* device scratch, >= ssd_bwd_workspace_size() */
    size_t workspace_bytes;
} ssd_bwd_args;

/* Bytes of device workspace ssd_bwd needs for these sizes (0 on invalid or
 * unsupported sizes).  Only sizes, dtype and flags are read. */
size_t ssd_bwd_workspace_size(const ssd_bwd_args* args);

/* The backward pass (see above).  Stream-ordered. */
ssd_status ssd_bwd(const ssd_bwd_args* args, void* stream);

/* Synchronises `stream` and returns the device status of the last ssd_bwd
 * call that used this workspace: SSD_OK, or SSD_ERR_TIMEOUT when a kernel of
 * its forward recompute gave up on a wait. */
ssd_status ssd_bwd_check_status(const ssd_bwd_args* args, void* stream);

/* ---- diagonal-A selective scan (Mamba-1 form) ------------------------------ */
/* The selective scan with A diagonal per channel and state, the Mamba-1 form
 * the page "MAMBA-2 Reference Implementations Comparison" sets beside SSD
 * (section 2.3; A_log [d_inner, d_state] in the block parameter list of
 * section 1.3; dt per channel and B * dt in "MAMBA-2 Implementation Gaps",
 * Gap 3):
 *   dt_t[d]  = softplus(dt_raw_t[d] + dt_bias[d])
 *   h_t[d,n] = exp(dt_t[d] A[d,n]) h_{t-1}[d,n] + dt_t[d] B_t[n] x_t[d]
 *   y_t[d]   = sum_n C_t[n] h_t[d,n] + D[d] x_t[d]
 * Layouts: x, dt (raw), y [batch, seqlen, channels] dtype; A [channels,
 * dstate] fp32 (the negative values themselves, i.e. -exp(A_log)); B, C
 * [batch, seqlen, dstate] dtype (shared by all channels); D, dt_bias
 * [channels] fp32 or NULL; init_state, final_state [batch, channels, dstate]
 * fp32 or NULL.  `chunk` cuts the sequence for parallelism (the result does
 * not depend on it beyond rounding).
 * Supported: dstate a multiple of 4 up to 32; 1 <= chunk, chunk * dstate <=
 * 4096; batch <= 65535 (else SSD_ERR_UNSUPPORTED); A, init_state,
 * final_state and the workspace 16-byte aligned.  Errors and stream ordering
 * as for ssd_fwd. */
typedef struct {
    int64_t batch, seqlen, channels, dstate, chunk;
    int32_t dtype;
    int32_t flags;          /* reserved, 0 */
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    const float* init_state;
    void* y;
    float* final_state;
    void* workspace;        /* device scratch, >= ssd_selective_scan_workspace_size() */
    size_t workspace_bytes;
} ssd_selective_scan_args;

/* Bytes of workspace for these sizes (0 if invalid or unsupported). */
size_t ssd_selective_scan_workspace_size(const ssd_selective_scan_args* args);

ssd_status ssd_selective_scan(const ssd_selective_scan_args* args, void* stream);

/* One decode step of the same scan on a carried state [batch, channels,
 * dstate] fp32, updated in place; x, dt, y [batch, channels] dtype; B, C
 * [batch, dstate] dtype.  state, A, B and C 16-byte aligned (else
 * SSD_ERR_INVALID_ARG); dstate as above.  Consecutive calls on one stream go
 * out with programmatic dependent launch. */
typedef struct {
    int64_t batch, channels, dstate;
    int32_t dtype;
    int32_t flags;          /* reserved, 0 */
    float* state;
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    void* y;
} ssd_selective_state_update_args;

ssd_status ssd_selective_state_update(const ssd_selective_state_update_args* args, void* stream);

/* ---- decode ------------------------------------------------------------- */
/* One token per sequence against a carried state (the SSM half of the
 * Mamba2Cache the page "MAMBA-2 Reference Implementations Comparison",
 * section 1.3, mentions):
 *   dt = softplus(dt_raw + dt_bias_h);  a = exp(dt A_h)
 *   state[p,n] <- a state[p,n] + dt x[p] B[n];   y[p] = sum_n state[p,n] C[n] + D x[p]
 * Layouts: state [batch, nheads, headdim, dstate] fp32, updated in place;
 *   x, y [batch, nheads, headdim] dtype; dt [batch, nheads] dtype;
 *   B, C [batch, ngroups, dstate] dtype; A, D, dt_bias [nheads] fp32
 *   (D, dt_bias may be NULL); z may be NULL, else the output gate
 *   [batch, nheads, headdim] dtype: y = (sum_n state C + D x) silu(z).
 * Supported: dstate in {16, 32, 64, 128, 256}; headdim >= 1. */
typedef struct {
    int64_t batch, nheads, headdim, dstate, ngroups;
    int32_t dtype;
    int32_t flags;          /* reserved, 0 */
    float* state;
    const void* x;
    const void* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    const float* dt_bias;
    void* y;
    const void* z;          /* optional output gate; NULL = none */
} ssd_state_update_args;

ssd_status ssd_state_update(const ssd_state_update_args* args, void* stream);

/* ---- causal depthwise convolution (before the scan) ---------------------- */
/* The layer the page "MAMBA-2 Implementation Gaps" (Gap 2, "Convolution
 * Layer") puts in front of the scan: a Conv1d with one filter per channel,
 * kernel width K, causal padding K - 1 and the output cut to the sequence
 * length, then SiLU:
 *   out[t, c] = bias[c] + sum_{k<K} w[c, k] xin[t - (K-1) + k, c];  y = silu(out)
 * where xin extends x backwards with the carried inputs (init_state).
 * Layouts: x, y [batch, seqlen, channels] dtype; weight [channels, width]
 *   fp32; bias [channels] fp32 or NULL; init_state, final_state [batch,
 *   channels, width - 1] fp32, the inputs before token 0 / the last width - 1
 *   inputs, oldest first; NULL = zeros / not returned.
 * Supported: 1 <= width <= 8; channels a multiple of 8 (bf16) or 4 (fp32);
 *   batch <= 65535; x and y 16-byte aligned (else SSD_ERR_UNSUPPORTED /
 *   SSD_ERR_INVALID_ARG).  Errors as for ssd_fwd; a kernel that gave up on a
 *   wait is reported by ssd_conv1d_check_status. */
typedef struct {
    int64_t batch, seqlen, channels, width;
    int32_t dtype;
    int32_t activation;     /* 1 = SiLU, 0 = none */
    const void* x;
    const float* weight;
    const float* bias;
    const float* init_state;
    void* y;
    float* final_state;
} ssd_conv1d_args;

ssd_status ssd_causal_conv1d(const ssd_conv1d_args* args, void* stream);

/* Synchronises `stream` and returns SSD_ERR_TIMEOUT if a ssd_causal_conv1d
 * launch on this device timed out on an internal wait since the last check
 * (the flag is cleared), else SSD_OK. */
ssd_status ssd_conv1d_check_status(void* stream);

/* One decode step of the same convolution (its half of the Mamba2Cache):
 * state [batch, channels, width - 1] fp32 holds the previous width - 1 inputs,
 * oldest first, and is shifted in place to end with x;
 *   y[c] = silu(bias[c] + sum_{k<width-1} w[c, k] state[c, k] + w[c, width-1] x[c]).
 * x, y [batch, channels] dtype; weight, bias as for ssd_causal_conv1d.
 * Supported: 1 <= width <= 8; channels a multiple of 8 (bf16) or 4 (fp32)
 *   (else SSD_ERR_UNSUPPORTED); every pointer 16-byte aligned (else
 *   SSD_ERR_INVALID_ARG). */
typedef struct {
    int64_t batch, channels, width;
    int32_t dtype;
    int32_t activation;     /* 1 = SiLU, 0 = none */
    float* state;
    const void* x;
    const float* weight;
    const float* bias;
    void* y;
} ssd_conv1d_update_args;

ssd_status ssd_conv1d_update(const ssd_conv1d_update_args* args, void* stream);

/* ---- gated RMSNorm (after the scan) ------------------------------------- */
/* The normalisation "MAMBA-2 Implementation Gaps" (section 7.3, items 9 and
 * 11) puts between the scan and the output projection, with the output gate
 * y * silu(z) applied inside it: for each row and each group of `group`
 * consecutive channels,
 *   g = y * silu(z)  (g = y when z is NULL),
 *   out = g / sqrt(mean over the group of g^2 + eps) * weight.
 * Use it on the ungated y of ssd_fwd (z = NULL there) with the same z here.
 * Layouts: y, z, out [rows, channels] dtype (rows = batch * seqlen for the
 *   scan's y viewed as [batch * seqlen, nheads * headdim]); weight [channels]
 *   fp32.  out may be y (in place).  Arithmetic in fp32; out rounded to dtype.
 * Supported: channels % group == 0; group a multiple of 8 (bf16) or 4 (fp32)
 *   (else SSD_ERR_UNSUPPORTED); eps >= 0 and finite, sizes > 0, y, weight,
 *   out non-NULL (else SSD_ERR_INVALID_ARG); every pointer 16-byte aligned
 *   (else SSD_ERR_INVALID_ARG). */
typedef struct {
    int64_t rows, channels, group;
    int32_t dtype;
    float eps;
    const void* y;
    const void* z;           /* optional gate; NULL = none */
    const float* weight;
    void* out;
} ssd_gated_rmsnorm_args;

ssd_status ssd_gated_rmsnorm(const ssd_gated_rmsnorm_args* args, void* stream);

/* ---- misc --------------------------------------------------------------- */
/* Static, human-readable name of a status code. */
const char* ssd_status_string(ssd_status status);

/* Name of the last CUDA error behind an SSD_ERR_CUDA returned to this host
 * thread (static string; "no CUDA error" if none). */
const char* ssd_last_cuda_error(void);

/* Library version string (static). */
const char* ssd_version(void);

/* Test hook for the failure paths, off by default: makes one producer withhold
 * one hand-off, so the consumers' bounded waits run out and the kernel reports
 * SSD_ERR_TIMEOUT through its status word instead of hanging (no fault, no
 * trap).  `what` = SSD_DEBUG_CONV_TILE: the convolution's producer stops before
 * tile `index`; SSD_DEBUG_FWD_CARRY: the single-pass forward does not publish the
 * state leaving run `index` (a run is the group of up to four consecutive
 * 128-token tiles one cluster of CTAs takes; the next run's wait gives up
 * after about a second; SSD_FLAG_SINGLE_PASS only); SSD_DEBUG_SCAN_DECAYS: the
 * tensor-core chunk_scan does not hand the decays of the first head of chunk
 * `index` to its workers, whose waits give up.  index < 0 turns the hook off.
 * Process-wide; read on the host when a kernel is launched.  Other values of
 * `what` are ignored. */
#define SSD_DEBUG_CONV_TILE 0
#define SSD_DEBUG_FWD_CARRY 1
#define SSD_DEBUG_SCAN_DECAYS 2
void ssd_debug_set_withhold(int what, int64_t index);

#ifdef __cplusplus
}
#endif
#endif /* SSD_B200_H */
