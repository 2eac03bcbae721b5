/*
 * ssd_oracle.c -- fp64 CPU oracle for the Mamba-2 SSD selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; its inputs arrive as plain double arrays.
 *
 * What it computes (sources are the five pages this project is built from):
 *
 *   dt_t  = softplus(dt_raw_t + dt_bias_h)
 *           ("MAMBA-2 Reference Implementations Comparison", section 3.2
 *            "Selective Scan Algorithm"; "MAMBA-2 Implementation Gaps",
 *            Gap 3 "dt (Time Step) Parameter")
 *   a_t   = exp(dt_t * A_h), A_h a scalar per head
 *           (same passages; scalar-times-identity A per "MAMBA-2 Reference
 *            Implementations Comparison", section 2.2)
 *   h_t   = a_t * h_{t-1} + dt_t * x_t B_t^T      (Euler input, B * dt)
 *   y_t   = C_t . h_t + D_h * x_t
 *           (D skip: "MAMBA-2 Implementation Gaps", Gap 4)
 *
 * and, around the scan, the output gate y * silu(z) (oracle_gate) and the causal
 * depthwise convolution before it with its decode step (oracle_causal_conv1d,
 * oracle_conv1d_update).
 *
 * Layouts (row-major, innermost last):
 *   x, y       [batch, seqlen, nheads, headdim]
 *   dt_raw     [batch, seqlen, nheads]
 *   B, C       [batch, seqlen, ngroups, dstate]
 *   A, D, bias [nheads]
 *   state      [batch, nheads, headdim, dstate]
 * Head h reads group g = h / (nheads / ngroups).
 *
 * Functions:
 *   oracle_ssd_fwd       the plain token-by-token recurrence (the definition)
 *   oracle_ssd_chunked   the chunked restatement (local chunk states, carry
 *                        of the last state across chunks, per-chunk output)
 *                        that also returns each step's intermediates
 *   oracle_state_update  one decode step on a carried state (the recurrence
 *                        body applied once; the page "MAMBA-2 Reference
 *                        Implementations Comparison", section 1.3, names the
 *                        Mamba2Cache this state lives in)
 *   oracle_ssd_bwd       the gradients of oracle_ssd_fwd (reverse-mode
 *                        differentiation of the recurrence, token by token)
 *   oracle_selective_scan, oracle_selective_state_update
 *                        the diagonal-A (per channel and state) selective
 *                        scan and its decode step
 *   oracle_gated_rmsnorm the RMSNorm of y * silu(z) per channel group
 *
 * Pins (tests/, CPU only): the masked-attention (quadratic) dual form by brute
 * force, the A = 0 cumulative-sum closed form, chunk-size invariance, split /
 * resume, decode == forward, special cases (C = 0, x = 0, full decay, L = 1),
 * causality, and a hand-derived half-decay example.
 *
 * ORACLE_MUTANT selects a deliberately wrong variant for the test that checks
 * the pins catch plausible mistakes; the default build (0) is the oracle.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* softplus(u) = log(1 + e^u), evaluated without overflow. */
double oracle_softplus(double u) {
#if ORACLE_MUTANT == 8
    return exp(u);
#else
    return (u > 0.0 ? u : 0.0) + log1p(exp(-fabs(u)));
#endif
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the following calls (timing on one core or all of them); no
 * effect on the arithmetic. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

static double dt_of(const double* dt_raw, const double* dt_bias,
                    int64_t i, int64_t h) {
#if ORACLE_MUTANT == 5
    (void)dt_bias; (void)h;
    return oracle_softplus(dt_raw[i]);
#else
    return oracle_softplus(dt_raw[i] + (dt_bias ? dt_bias[h] : 0.0));
#endif
}

static int64_t group_of(int64_t h, int64_t H, int64_t G) {
#if ORACLE_MUTANT == 6
    (void)H;
    return h % G;
#else
    return h / (H / G);
#endif
}

/* The output gate applied after the scan, y <- y * silu(z) with
 * silu(z) = z * sigmoid(z) = z / (1 + e^-z) ("MAMBA-2 Reference
 * Implementations Comparison", section 3 (the forward listing) and section 6.1
 * item 5, output gating).  n elements, in place on y. */
void oracle_gate(double* y, const double* z, int64_t n) {
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i) {
#if ORACLE_MUTANT == 10
        y[i] = y[i] / (1.0 + exp(-z[i]));
#else
        y[i] = y[i] * (z[i] / (1.0 + exp(-z[i])));
#endif
    }
}

/* The recurrence, token by token.  init may be NULL (zero state); D and
 * dt_bias may be NULL (zero); final_state may be NULL. */
void oracle_ssd_fwd(int64_t batch, int64_t L, int64_t H, int64_t P,
                    int64_t N, int64_t G,
                    const double* x, const double* dt_raw, const double* A,
                    const double* B, const double* C, const double* D,
                    const double* dt_bias, const double* init,
                    double* y, double* final_state) {
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < batch * H; ++bh) {
        const int64_t b = bh / H, h = bh % H, g = group_of(h, H, G);
        double* S = (double*)malloc(sizeof(double) * (size_t)(P * N));
        const double Dh = D ? D[h] : 0.0;
        if (init && ORACLE_MUTANT != 9)
            memcpy(S, init + bh * P * N, sizeof(double) * (size_t)(P * N));
        else
            memset(S, 0, sizeof(double) * (size_t)(P * N));
        for (int64_t t = 0; t < L; ++t) {
            const int64_t it = (b * L + t) * H + h;
            const double dt = dt_of(dt_raw, dt_bias, it, h);
#if ORACLE_MUTANT == 4
            const double a = exp(-dt * A[h]);
#else
            const double a = exp(dt * A[h]);
#endif
            const double* xt = x + it * P;
            const double* Bt = B + ((b * L + t) * G + g) * N;
            const double* Ct = C + ((b * L + t) * G + g) * N;
#if ORACLE_MUTANT == 3
            { const double* tmp = Bt; Bt = Ct; Ct = tmp; }
#endif
            double* yt = y + it * P;
            for (int64_t p = 0; p < P; ++p) {
                double* Sp = S + p * N;
                double acc = 0.0;
#if ORACLE_MUTANT == 2
                for (int64_t n = 0; n < N; ++n) acc += Sp[n] * Ct[n];
#endif
                for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 7
                    Sp[n] = a * Sp[n] + xt[p] * Bt[n];
#else
                    Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];
#endif
                }
#if ORACLE_MUTANT != 2
                for (int64_t n = 0; n < N; ++n) acc += Sp[n] * Ct[n];
#endif
#if ORACLE_MUTANT == 1
                yt[p] = acc;
#else
                yt[p] = acc + Dh * xt[p];
#endif
            }
        }
        if (final_state)
            memcpy(final_state + bh * P * N, S, sizeof(double) * (size_t)(P * N));
        free(S);
    }
}

/*
 * The backward pass of oracle_ssd_fwd: the gradients of the scalar
 *   J = sum_t dy_t . y_t + d_final : h_L
 * with respect to every input, by reverse-mode differentiation of the
 * recurrence one line at a time.  With g_t = dJ/dh_t (P x N), a_t = dt_t A_h
 * the log decay and h_0 the initial state:
 *   g_L = d_final + dy_L C_L^T,   g_t = e^{a_{t+1}} g_{t+1} + dy_t C_t^T
 *   dC_t      = h_t^T dy_t                      (from y_t = C_t . h_t)
 *   dx_t      = D_h dy_t + dt_t g_t B_t          (h_t receives dt_t x_t B_t^T)
 *   dB_t      = dt_t g_t^T x_t
 *   da_t      = e^{a_t} <g_t, h_{t-1}>           (h_t = e^{a_t} h_{t-1} + ...)
 *   ddt_t     = x_t . (g_t B_t) + A_h da_t,   dA_h += dt_t da_t
 *   ddt_raw_t = ddt_t sigmoid(dt_raw_t + dt_bias_h),   ddt_bias_h += ddt_raw_t
 *   dD_h     += dy_t . x_t,   d_init = dJ/dh_0 = e^{a_1} g_1
 * The recurrence is the one of "MAMBA-2 Reference Implementations
 * Comparison", section 2.2; the page "Agent 230: Comprehensive MAMBA-2
 * Implementation Comparison", section 6 (Gradient Computation), takes the
 * gradients of A, B, C and delta (dt) after its backward pass but gives no
 * formulas; all of them follow from the chain rule alone
 * (softplus'(u) = sigmoid(u)).
 *
 * dy [b,L,H,P]; d_final [b,H,P,N] or NULL (zero).  Outputs shaped like the
 * inputs: dx, ddt_raw, dB, dC (dB, dC summed over the heads of a group),
 * d_init [b,H,P,N]; dA, dD, ddt_bias [H] summed over batch and time.  d_init,
 * dD and ddt_bias may be NULL.  Sums over heads and batch rows are taken in a
 * fixed order after the parallel part.
 */
void oracle_ssd_bwd(int64_t batch, int64_t L, int64_t H, int64_t P,
                    int64_t N, int64_t G,
                    const double* x, const double* dt_raw, const double* A,
                    const double* B, const double* C, const double* D,
                    const double* dt_bias, const double* init,
                    const double* dy, const double* d_final,
                    double* dx, double* ddt_raw, double* dA, double* dB,
                    double* dC, double* dD, double* ddt_bias, double* d_init) {
    const int64_t PN = P * N;
    double* dBh = (double*)calloc((size_t)(batch * H * L * N), sizeof(double));
    double* dCh = (double*)calloc((size_t)(batch * H * L * N), sizeof(double));
    double* sums = (double*)calloc((size_t)(batch * H * 3), sizeof(double));
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < batch * H; ++bh) {
        const int64_t b = bh / H, h = bh % H, g = group_of(h, H, G);
        const double Dh = D ? D[h] : 0.0;
        double* hs = (double*)malloc(sizeof(double) * (size_t)((L + 1) * PN));
        double* gr = (double*)malloc(sizeof(double) * (size_t)PN);
        double* dxs = (double*)malloc(sizeof(double) * (size_t)P);
        /* forward, keeping every state: hs[t] = h_t, hs[0] = h_0 */
        if (init)
            memcpy(hs, init + bh * PN, sizeof(double) * (size_t)PN);
        else
            memset(hs, 0, sizeof(double) * (size_t)PN);
        for (int64_t t = 0; t < L; ++t) {
            const int64_t it = (b * L + t) * H + h;
            const double dt = dt_of(dt_raw, dt_bias, it, h);
            const double a = exp(dt * A[h]);
            const double* xt = x + it * P;
            const double* Bt = B + ((b * L + t) * G + g) * N;
            const double* hp = hs + t * PN;
            double* hn = hs + (t + 1) * PN;
            for (int64_t p = 0; p < P; ++p)
                for (int64_t n = 0; n < N; ++n)
                    hn[p * N + n] = a * hp[p * N + n] + dt * xt[p] * Bt[n];
        }
        /* backward */
        if (d_final)
            memcpy(gr, d_final + bh * PN, sizeof(double) * (size_t)PN);
        else
            memset(gr, 0, sizeof(double) * (size_t)PN);
        double sA = 0.0, sD = 0.0, sbias = 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
            const int64_t it = (b * L + t) * H + h;
            const double u = dt_raw[it] + (dt_bias ? dt_bias[h] : 0.0);
            const double dt = dt_of(dt_raw, dt_bias, it, h);
            const double a = exp(dt * A[h]);
            const double* xt = x + it * P;
            const double* Bt = B + ((b * L + t) * G + g) * N;
            const double* Ct = C + ((b * L + t) * G + g) * N;
            const double* dyt = dy + it * P;
            const double* ht = hs + (t + 1) * PN;
            const double* hp = hs + t * PN;
            double* dBt = dBh + (bh * L + t) * N;
            double* dCt = dCh + (bh * L + t) * N;
#if ORACLE_MUTANT != 17
            for (int64_t p = 0; p < P; ++p)          /* g_t = ... + dy_t C_t^T */
                for (int64_t n = 0; n < N; ++n) gr[p * N + n] += dyt[p] * Ct[n];
#endif
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t p = 0; p < P; ++p) acc += dyt[p] * ht[p * N + n];
                dCt[n] = acc;
            }
            for (int64_t p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) acc += gr[p * N + n] * Bt[n];
                dxs[p] = acc;
                dx[it * P + p] = Dh * dyt[p] + dt * acc;
            }
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t p = 0; p < P; ++p) acc += gr[p * N + n] * xt[p];
                dBt[n] = dt * acc;
            }
            double gh = 0.0, xdxs = 0.0, dyx = 0.0;
            for (int64_t k = 0; k < PN; ++k) gh += gr[k] * hp[k];
            for (int64_t p = 0; p < P; ++p) {
                xdxs += xt[p] * dxs[p];
                dyx += dyt[p] * xt[p];
            }
            const double da = a * gh;
#if ORACLE_MUTANT == 15
            const double ddt = xdxs;
#else
            const double ddt = xdxs + A[h] * da;
#endif
            sA += dt * da;
#if ORACLE_MUTANT == 16
            const double dr = ddt;
            (void)u;
#else
            const double dr = ddt / (1.0 + exp(-u));
#endif
            ddt_raw[it] = dr;
            sbias += dr;
            sD += dyx;
#if ORACLE_MUTANT == 17
            for (int64_t p = 0; p < P; ++p)
                for (int64_t n = 0; n < N; ++n) gr[p * N + n] += dyt[p] * Ct[n];
#endif
#if ORACLE_MUTANT != 14
            for (int64_t k = 0; k < PN; ++k) gr[k] *= a;   /* now dJ/dh_{t-1} */
#endif
        }
        if (d_init) memcpy(d_init + bh * PN, gr, sizeof(double) * (size_t)PN);
        sums[bh * 3 + 0] = sA;
        sums[bh * 3 + 1] = sD;
        sums[bh * 3 + 2] = sbias;
        free(dxs);
        free(gr);
        free(hs);
    }
    for (int64_t h = 0; h < H; ++h) {
        double sA = 0.0, sD = 0.0, sb = 0.0;
        for (int64_t b = 0; b < batch; ++b) {
            sA += sums[(b * H + h) * 3 + 0];
            sD += sums[(b * H + h) * 3 + 1];
            sb += sums[(b * H + h) * 3 + 2];
        }
        dA[h] = sA;
        if (dD) dD[h] = sD;
        if (ddt_bias) ddt_bias[h] = sb;
    }
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t t = 0; t < L; ++t)
            for (int64_t g = 0; g < G; ++g)
                for (int64_t n = 0; n < N; ++n) {
                    double sb = 0.0, sc = 0.0;
                    for (int64_t h = 0; h < H; ++h) {
                        if (group_of(h, H, G) != g) continue;
                        sb += dBh[((b * H + h) * L + t) * N + n];
                        sc += dCh[((b * H + h) * L + t) * N + n];
                    }
                    dB[((b * L + t) * G + g) * N + n] = sb;
                    dC[((b * L + t) * G + g) * N + n] = sc;
                }
    free(sums);
    free(dCh);
    free(dBh);
}

/*
 * The selective scan with a diagonal A per channel (the Mamba-1 form the pages
 * set beside SSD: "MAMBA-2 Reference Implementations Comparison", section 2.3,
 * Mamba-1 vs SSD; A_log of shape [d_inner, d_state] in the block's parameter
 * list of section 1.3, and dt per channel from dt_proj with B * dt as the
 * input term in "MAMBA-2 Implementation Gaps", Gap 3).  Per channel d and state n:
 *   dt_t[d]   = softplus(dt_raw_t[d] + dt_bias[d])
 *   h_t[d,n]  = exp(dt_t[d] A[d,n]) h_{t-1}[d,n] + dt_t[d] B_t[n] x_t[d]
 *   y_t[d]    = sum_n C_t[n] h_t[d,n] + D[d] x_t[d]
 * Layouts: x, dt_raw, y [b, L, Dc]; A [Dc, N]; B, C [b, L, N]; D, dt_bias
 * [Dc]; state [b, Dc, N].  init, D, dt_bias, final_state may be NULL.
 */
void oracle_selective_scan(int64_t batch, int64_t L, int64_t Dc, int64_t N,
                           const double* x, const double* dt_raw, const double* A,
                           const double* B, const double* C, const double* D,
                           const double* dt_bias, const double* init,
                           double* y, double* final_state) {
    int64_t bd;
#pragma omp parallel for schedule(dynamic, 16)
    for (bd = 0; bd < batch * Dc; ++bd) {
        const int64_t b = bd / Dc, d = bd % Dc;
        double* h = (double*)malloc(sizeof(double) * (size_t)N);
        for (int64_t n = 0; n < N; ++n) h[n] = init ? init[bd * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const int64_t it = (b * L + t) * Dc + d;
            const double dt = oracle_softplus(dt_raw[it] + (dt_bias ? dt_bias[d] : 0.0));
#if ORACLE_MUTANT == 19
            const double xt = x[(b * L + t) * Dc];
#else
            const double xt = x[it];
#endif
            const double* Bt = B + (b * L + t) * N;
            const double* Ct = C + (b * L + t) * N;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 18
                const double a = exp(dt * A[d * N]);
#else
                const double a = exp(dt * A[d * N + n]);
#endif
                h[n] = a * h[n] + dt * Bt[n] * xt;
                acc += Ct[n] * h[n];
            }
            y[it] = acc + (D ? D[d] : 0.0) * x[it];
        }
        if (final_state) memcpy(final_state + bd * N, h, sizeof(double) * (size_t)N);
        free(h);
    }
}

/* One decode step of oracle_selective_scan on a carried state [b, Dc, N]:
 * x, dt_raw, y [b, Dc]; B, C [b, N]. */
void oracle_selective_state_update(int64_t batch, int64_t Dc, int64_t N, double* state,
                                   const double* x, const double* dt_raw, const double* A,
                                   const double* B, const double* C, const double* D,
                                   const double* dt_bias, double* y) {
    int64_t bd;
#pragma omp parallel for schedule(static)
    for (bd = 0; bd < batch * Dc; ++bd) {
        const int64_t b = bd / Dc, d = bd % Dc;
        const double dt = oracle_softplus(dt_raw[bd] + (dt_bias ? dt_bias[d] : 0.0));
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double* h = state + bd * N + n;
            *h = exp(dt * A[d * N + n]) * *h + dt * B[b * N + n] * x[bd];
            acc += C[b * N + n] * *h;
        }
        y[bd] = acc + (D ? D[d] : 0.0) * x[bd];
    }
}

/*
 * The gated RMSNorm after the scan ("MAMBA-2 Implementation Gaps" lists an
 * RMSNorm before the final projection; the gated form normalises the gated
 * output): for each row and each group of `group` consecutive channels,
 *   g = y * silu(z)   (g = y when z is NULL)
 *   out = g / sqrt(mean over the group of g^2 + eps) * weight
 * y, z, out [rows, channels]; weight [channels].
 */
void oracle_gated_rmsnorm(int64_t rows, int64_t channels, int64_t group, double eps,
                          const double* y, const double* z, const double* weight, double* out) {
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; ++r) {
        for (int64_t g0 = 0; g0 < channels; g0 += group) {
            double ss = 0.0;
            for (int64_t k = 0; k < group; ++k) {
                const int64_t i = r * channels + g0 + k;
#if ORACLE_MUTANT == 20
                const double g = y[i];
#else
                const double g = z ? y[i] * (z[i] / (1.0 + exp(-z[i]))) : y[i];
#endif
                out[i] = g;
                ss += g * g;
            }
#if ORACLE_MUTANT == 21
            const double inv = 1.0 / sqrt(ss + eps);
#else
            const double inv = 1.0 / sqrt(ss / (double)group + eps);
#endif
            for (int64_t k = 0; k < group; ++k) {
                const int64_t i = r * channels + g0 + k;
#if ORACLE_MUTANT == 20
                out[i] = out[i] * inv * (z ? z[i] / (1.0 + exp(-z[i])) : 1.0) * weight[g0 + k];
#else
                out[i] = out[i] * inv * weight[g0 + k];
#endif
            }
        }
    }
}

/*
 * The chunked restatement: the sequence is cut into chunks of Q tokens (the
 * last one may be shorter) and processed in the three phases the SSD chunk
 * scan describes ("MAMBA-2 Implementation Gaps", Gap 1: a local, parallel
 * "diagonal block" per chunk, an inter-chunk carry of the last state, then the
 * output), with dt and the in-chunk cumulative sum of dt * A made explicit.
 *
 * Outputs (any may be NULL except y):
 *   dt_out, cumA_out  [batch, H, nc, Q]  (entries past a short tail are 0)
 *   S_out             [batch, nc, H, P, N] local state of each chunk
 *   Hin_out           [batch, nc, H, P, N] state entering each chunk
 *   final_state       [batch, H, P, N]
 */
void oracle_ssd_chunked(int64_t batch, int64_t L, int64_t H, int64_t P,
                        int64_t N, int64_t G, int64_t Q,
                        const double* x, const double* dt_raw, const double* A,
                        const double* B, const double* C, const double* D,
                        const double* dt_bias, const double* init,
                        double* dt_out, double* cumA_out, double* S_out,
                        double* Hin_out, double* y, double* final_state) {
    const int64_t nc = (L + Q - 1) / Q;
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < batch * H; ++bh) {
        const int64_t b = bh / H, h = bh % H, g = group_of(h, H, G);
        const double Dh = D ? D[h] : 0.0;
        double* dt = (double*)calloc((size_t)Q, sizeof(double));
        double* cumA = (double*)calloc((size_t)Q, sizeof(double));
        double* S = (double*)malloc(sizeof(double) * (size_t)(P * N));
        double* Hc = (double*)malloc(sizeof(double) * (size_t)(P * N));
        if (init)
            memcpy(Hc, init + bh * P * N, sizeof(double) * (size_t)(P * N));
        else
            memset(Hc, 0, sizeof(double) * (size_t)(P * N));
        for (int64_t c = 0; c < nc; ++c) {
            const int64_t t0 = c * Q;
            const int64_t Lc = (L - t0 < Q) ? (L - t0) : Q;
            /* step 1: dt and the inclusive in-chunk cumulative sum of dt*A */
            double run = 0.0;
            for (int64_t l = 0; l < Q; ++l) {
                if (l < Lc) {
                    dt[l] = dt_of(dt_raw, dt_bias, (b * L + t0 + l) * H + h, h);
                    run += dt[l] * A[h];
                    cumA[l] = run;
                } else {
                    dt[l] = 0.0;
                    cumA[l] = 0.0;
                }
            }
            if (dt_out)
                memcpy(dt_out + (bh * nc + c) * Q, dt, sizeof(double) * (size_t)Q);
            if (cumA_out)
                memcpy(cumA_out + (bh * nc + c) * Q, cumA, sizeof(double) * (size_t)Q);
            /* step 2: the chunk's local state, as if it started from zero */
            memset(S, 0, sizeof(double) * (size_t)(P * N));
            for (int64_t l = 0; l < Lc; ++l) {
                const double w = exp(cumA[Lc - 1] - cumA[l]) * dt[l];
                const double* xl = x + ((b * L + t0 + l) * H + h) * P;
                const double* Bl = B + ((b * L + t0 + l) * G + g) * N;
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n)
                        S[p * N + n] += w * xl[p] * Bl[n];
            }
            if (S_out)
                memcpy(S_out + ((b * nc + c) * H + h) * P * N, S,
                       sizeof(double) * (size_t)(P * N));
            if (Hin_out)
                memcpy(Hin_out + ((b * nc + c) * H + h) * P * N, Hc,
                       sizeof(double) * (size_t)(P * N));
            /* step 4 (uses the state entering the chunk): the output */
            for (int64_t l = 0; l < Lc; ++l) {
                const double* Cl = C + ((b * L + t0 + l) * G + g) * N;
                const double* xl = x + ((b * L + t0 + l) * H + h) * P;
                double* yl = y + ((b * L + t0 + l) * H + h) * P;
                const double carry = exp(cumA[l]);
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) acc += Cl[n] * Hc[p * N + n];
                    yl[p] = carry * acc + Dh * xl[p];
                }
                for (int64_t j = 0; j <= l; ++j) {
                    const double* Bj = B + ((b * L + t0 + j) * G + g) * N;
                    const double* xj = x + ((b * L + t0 + j) * H + h) * P;
                    double cb = 0.0;
                    for (int64_t n = 0; n < N; ++n) cb += Cl[n] * Bj[n];
                    const double m = exp(cumA[l] - cumA[j]) * cb * dt[j];
                    for (int64_t p = 0; p < P; ++p) yl[p] += m * xj[p];
                }
            }
            /* step 3: carry the state across the chunk boundary */
            const double decay = exp(cumA[Lc - 1]);
            for (int64_t i = 0; i < P * N; ++i) Hc[i] = decay * Hc[i] + S[i];
        }
        if (final_state)
            memcpy(final_state + bh * P * N, Hc, sizeof(double) * (size_t)(P * N));
        free(dt); free(cumA); free(S); free(Hc);
    }
}

/* One decode step: state [batch, H, P, N] is updated in place and y [batch,
 * H, P] receives the step's output.  x [batch, H, P], dt_raw [batch, H],
 * B, C [batch, G, N]. */
void oracle_state_update(int64_t batch, int64_t H, int64_t P, int64_t N,
                         int64_t G, double* state,
                         const double* x, const double* dt_raw,
                         const double* A, const double* B, const double* C,
                         const double* D, const double* dt_bias, double* y) {
    int64_t bh;
#pragma omp parallel for schedule(static)
    for (bh = 0; bh < batch * H; ++bh) {
        const int64_t b = bh / H, h = bh % H, g = group_of(h, H, G);
        const double dt = dt_of(dt_raw, dt_bias, bh, h);
        const double a = exp(dt * A[h]);
        const double* xt = x + bh * P;
        const double* Bt = B + (b * G + g) * N;
        const double* Ct = C + (b * G + g) * N;
        double* S = state + bh * P * N;
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                S[p * N + n] = a * S[p * N + n] + dt * xt[p] * Bt[n];
                acc += S[p * N + n] * Ct[n];
            }
            y[bh * P + p] = acc + (D ? D[h] : 0.0) * xt[p];
        }
    }
}

/*
 * Causal depthwise convolution over time with an optional SiLU, the layer the
 * page "MAMBA-2 Implementation Gaps" (Gap 2, "Convolution Layer") puts before
 * the scan: a Conv1d with one filter per channel, kernel width K, padding K-1
 * and the output cut to the sequence length, so
 *
 *   out[t, c] = bias[c] + sum_{k=0}^{K-1} w[c, k] * xin[t - (K-1) + k, c]
 *   y[t, c]   = silu(out[t, c])  (or out when act == 0)
 *
 * where xin[i] = x[i] for i >= 0 and, for -(K-1) <= i < 0, the carried
 * inputs before token 0: init[c, K-1+i] (oldest first), zero when init is
 * NULL.  final (may be NULL) receives the last K-1 entries of xin, the state
 * the next call (or a decode step) continues from.
 * x, y [batch, L, Cn]; w [Cn, K]; bias [Cn] or NULL; init, final [batch, Cn, K-1].
 */
static double conv_in(const double* x, const double* init, int64_t L, int64_t Cn,
                      int64_t K, int64_t b, int64_t c, int64_t i) {
    if (i >= 0) return x[(b * L + i) * Cn + c];
#if ORACLE_MUTANT == 13
    (void)init;
    return 0.0;
#else
    return init ? init[(b * Cn + c) * (K - 1) + (K - 1 + i)] : 0.0;
#endif
}

void oracle_causal_conv1d(int64_t batch, int64_t L, int64_t Cn, int64_t K,
                          const double* x, const double* w, const double* bias,
                          const double* init, int act, double* y, double* final) {
    int64_t bc;
#pragma omp parallel for schedule(static)
    for (bc = 0; bc < batch * Cn; ++bc) {
        const int64_t b = bc / Cn, c = bc % Cn;
        for (int64_t t = 0; t < L; ++t) {
            double acc = bias ? bias[c] : 0.0;
            for (int64_t k = 0; k < K; ++k) {
#if ORACLE_MUTANT == 11
                const int64_t i = t - k;                 /* kernel reversed */
#elif ORACLE_MUTANT == 12
                const int64_t i = t - (K - 1) + k + 1;   /* one token ahead */
                if (i >= L) continue;
#else
                const int64_t i = t - (K - 1) + k;
#endif
                acc += w[c * K + k] * conv_in(x, init, L, Cn, K, b, c, i);
            }
            y[(b * L + t) * Cn + c] = act ? acc / (1.0 + exp(-acc)) : acc;
        }
        if (final)
            for (int64_t j = 0; j < K - 1; ++j)
                final[(b * Cn + c) * (K - 1) + j] = conv_in(x, init, L, Cn, K, b, c, L - (K - 1) + j);
    }
}

/* One decode step of the same convolution: state [batch, Cn, K-1] holds the
 * previous K-1 inputs (oldest first) and is shifted in place to end with
 * x [batch, Cn]; y [batch, Cn] receives the step's output. */
void oracle_conv1d_update(int64_t batch, int64_t Cn, int64_t K, double* state,
                          const double* x, const double* w, const double* bias,
                          int act, double* y) {
    int64_t bc;
#pragma omp parallel for schedule(static)
    for (bc = 0; bc < batch * Cn; ++bc) {
        const int64_t c = bc % Cn;
        double* s = state + bc * (K - 1);
        double acc = bias ? bias[c] : 0.0;
        for (int64_t k = 0; k < K - 1; ++k) acc += w[c * K + k] * s[k];
        acc += w[c * K + K - 1] * x[bc];
        for (int64_t k = 0; k + 1 < K - 1; ++k) s[k] = s[k + 1];
        if (K > 1) s[K - 2] = x[bc];
        y[bc] = act ? acc / (1.0 + exp(-acc)) : acc;
    }
}
