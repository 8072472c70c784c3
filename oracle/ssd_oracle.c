/*
 * ssd_oracle.c -- plain fp64 CPU oracle for the SSD (structured state space
 * duality) layer.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark load this library; the product
 * path (the CUDA library and its Python binding) never does.  It shares no
 * code, header or table with the CUDA path.
 *
 * What it computes.  The scalar-times-identity selective SSM, run as the
 * textbook linear recurrence, one token at a time, in double precision:
 *
 *     a_t      = exp(dt_t * A_h)                       (discretised A)
 *     S_t      = a_t * S_{t-1} + dt_t * x_t B_t^T       (P x N state)
 *     y_t[p]   = sum_n S_t[p][n] * C_t[n] + D_h * x_t[p]
 *
 * with S_{-1} = the initial state (or zero) and the final state = S_{L-1}.
 * The chunked (block-decomposed) algorithm of the CUDA path reaches exactly
 * this result up to rounding order.
 *
 * Passages followed:
 *  - "论文解读：Mamba: Linear-Time Sequence Modeling with Selective State
 *    Spaces", section 状态空间模型 (State Space Models): the continuous
 *    parameters (Delta, A, B, C) are discretised to (A-bar, B-bar) and the
 *    discrete model is evaluated either as a linear recurrence (the
 *    autoregressive form used here) or as a global convolution.  The
 *    discretisation formula itself is lost from that page; the reading taken
 *    is A-bar = exp(dt*A) and B-bar = dt*B.
 *  - Same page, section 选择性状态空间模型 (Selective State Space Models):
 *    dt, B and C vary with the token (time-varying, input-dependent).
 *  - "Transformers are SSMs: Generalized Models and Efficient Algorithms
 *    Through Structured State Space Duality" (CiteArk), AI research summary:
 *    the layer is a 1-semiseparable selective SSM; "what this means": the
 *    same map has a constant-memory recurrent (inference) form -- ssd_oracle_step.
 *
 * Layouts (row-major, contiguous):
 *   x, y         (batch, seqlen, nheads, headdim)
 *   dt           (batch, seqlen, nheads)
 *   A, D         (nheads)
 *   B, C         (batch, seqlen, ngroups, dstate)
 *   init, final  (batch, nheads, headdim, dstate)
 * Head h reads group g = h * ngroups / nheads (contiguous blocks of heads).
 *
 * Return value: 0 on success, -1 on an invalid argument (nothing written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int dims_ok(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                   int64_t dstate, int64_t ngroups) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
        return 0;
    if (nheads % ngroups != 0) return 0;
    return 1;
}

/* One (batch, head) pair of the recurrence.  S is a caller-provided
 * headdim*dstate scratch array. */
static void recur_one(int64_t b, int64_t h, int64_t seqlen, int64_t nheads, int64_t P,
                      int64_t N, int64_t G, const double* x, const double* dt,
                      const double* A, const double* B, const double* C, const double* D,
                      const double* init, double* y, double* final_state, double* S) {
    const int64_t g = h * G / nheads;
    if (init)
        memcpy(S, init + (b * nheads + h) * P * N, sizeof(double) * (size_t)(P * N));
    else
        memset(S, 0, sizeof(double) * (size_t)(P * N));

    for (int64_t t = 0; t < seqlen; ++t) {
        const double dtv = dt[(b * seqlen + t) * nheads + h];
        const double a = exp(dtv * A[h]);
        const double* xt = x + ((b * seqlen + t) * nheads + h) * P;
        const double* Bt = B + ((b * seqlen + t) * G + g) * N;
        const double* Ct = C + ((b * seqlen + t) * G + g) * N;
        double* yt = y + ((b * seqlen + t) * nheads + h) * P;
        for (int64_t p = 0; p < P; ++p) {
            double* Sp = S + p * N;
            const double u = dtv * xt[p];
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                Sp[n] = a * Sp[n] + u * Bt[n];
                acc += Sp[n] * Ct[n];
            }
            yt[p] = acc + D[h] * xt[p];
        }
    }
    if (final_state)
        memcpy(final_state + (b * nheads + h) * P * N, S, sizeof(double) * (size_t)(P * N));
}

/* The full forward: y for every token, final state per (batch, head). */
int ssd_oracle_recurrence(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                          int64_t dstate, int64_t ngroups, const double* x, const double* dt,
                          const double* A, const double* B, const double* C, const double* D,
                          const double* init, double* y, double* final_state, int nthreads) {
    if (!dims_ok(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!A || !D || (seqlen > 0 && batch > 0 && (!x || !dt || !B || !C || !y))) return -1;
    const int64_t pairs = batch * nheads;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)(headdim * dstate));
        if (!S) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < pairs; ++bh)
                recur_one(bh / nheads, bh % nheads, seqlen, nheads, headdim, dstate, ngroups, x,
                          dt, A, B, C, D, init, y, final_state, S);
            free(S);
        }
    }
    return failed ? -1 : 0;
}

/* One decode step: state (batch, nheads, headdim, dstate) updated in place,
 * x/y (batch, nheads, headdim), dt (batch, nheads), B/C (batch, ngroups,
 * dstate).  Same arithmetic as one iteration of the recurrence above. */
int ssd_oracle_step(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                    int64_t ngroups, double* state, const double* x, const double* dt,
                    const double* A, const double* B, const double* C, const double* D,
                    double* y) {
    if (!dims_ok(batch, 1, nheads, headdim, dstate, ngroups)) return -1;
    if (!state || !x || !dt || !A || !B || !C || !D || !y) return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t h = 0; h < nheads; ++h) {
            const int64_t g = h * ngroups / nheads;
            const double dtv = dt[b * nheads + h];
            const double a = exp(dtv * A[h]);
            const double* Bt = B + (b * ngroups + g) * dstate;
            const double* Ct = C + (b * ngroups + g) * dstate;
            for (int64_t p = 0; p < headdim; ++p) {
                double* Sp = state + ((b * nheads + h) * headdim + p) * dstate;
                const double xv = x[(b * nheads + h) * headdim + p];
                double acc = 0.0;
                for (int64_t n = 0; n < dstate; ++n) {
                    Sp[n] = a * Sp[n] + dtv * xv * Bt[n];
                    acc += Sp[n] * Ct[n];
                }
                y[(b * nheads + h) * headdim + p] = acc + D[h] * xv;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ backward
 * Gradients of the recurrence above for a loss whose derivatives with respect
 * to the outputs are dy (like y) and dfinal (like the final state; NULL = 0).
 * "Transformers are SSMs" (CiteArk), AI research summary: training is the
 * use the layer is built for; the gradients below are the chain rule applied
 * to the same token-by-token recurrence, in reverse token order:
 *
 *     G      = dL/dS_t          (starts at dfinal, then G += dy_t C_t^T)
 *     dC_t  += S_t^T dy_t        dx_t = D_h dy_t + dt_t G B_t
 *     dB_t  += dt_t G^T x_t      ddt_t = x_t^T G B_t + A_h a_t <G, S_{t-1}>
 *     dA_h  += dt_t a_t <G, S_{t-1}>     dD_h += dy_t . x_t
 *     G      = a_t G            (dL/dS_{t-1}); dinit = G after token 0
 *
 * The states S_t are kept from a forward sweep (test sizes only).  dB and dC
 * sum over the heads of a group, dA and dD over batch and tokens.  Outputs
 * are overwritten (not accumulated into).  Return 0, or -1 on an invalid
 * argument or allocation failure. */
static void bwd_one(int64_t b, int64_t h, int64_t L, int64_t H, int64_t P, int64_t N,
                    int64_t G, const double* x, const double* dt, const double* A,
                    const double* B, const double* C, const double* D, const double* init,
                    const double* dy, const double* dfinal, double* dx, double* ddt,
                    double* dA_part, double* dB, double* dC, double* dD_part, double* dinit,
                    double* Sall, double* Gm) {
    const int64_t g = h * G / H;
    const int64_t PN = P * N;
    /* forward sweep: Sall[0] = initial state, Sall[t + 1] = S_t */
    if (init != NULL)
        memcpy(Sall, init + (b * H + h) * PN, sizeof(double) * (size_t)PN);
    else
        memset(Sall, 0, sizeof(double) * (size_t)PN);
    for (int64_t t = 0; t < L; ++t) {
        const double dtv = dt[(b * L + t) * H + h];
        const double at = exp(A[h] * dtv);
        const double* xt = x + ((b * L + t) * H + h) * P;
        const double* Bt = B + ((b * L + t) * G + g) * N;
        const double* Sp = Sall + t * PN;
        double* Sn = Sall + (t + 1) * PN;
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n)
                Sn[p * N + n] = at * Sp[p * N + n] + dtv * xt[p] * Bt[n];
    }
    /* reverse sweep */
    if (dfinal != NULL)
        memcpy(Gm, dfinal + (b * H + h) * PN, sizeof(double) * (size_t)PN);
    else
        memset(Gm, 0, sizeof(double) * (size_t)PN);
    for (int64_t t = L - 1; t >= 0; --t) {
        const double dtv = dt[(b * L + t) * H + h];
        const double at = exp(A[h] * dtv);
        const double* xt = x + ((b * L + t) * H + h) * P;
        const double* Bt = B + ((b * L + t) * G + g) * N;
        const double* Ct = C + ((b * L + t) * G + g) * N;
        const double* dyt = dy + ((b * L + t) * H + h) * P;
        const double* St = Sall + (t + 1) * PN;   /* S_t */
        const double* Sp = Sall + t * PN;         /* S_{t-1} */
        double* dxt = dx + ((b * L + t) * H + h) * P;
        double* dBt = dB + ((b * L + t) * G + g) * N;
        double* dCt = dC + ((b * L + t) * G + g) * N;
        /* y_t = S_t C_t + D x_t */
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n) {
                Gm[p * N + n] += dyt[p] * Ct[n];
                dCt[n] += St[p * N + n] * dyt[p];
            }
        double xgb = 0.0, gs = 0.0, dydx = 0.0;
        for (int64_t p = 0; p < P; ++p) {
            double gb = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                gb += Gm[p * N + n] * Bt[n];
                dBt[n] += dtv * Gm[p * N + n] * xt[p];
                gs += Gm[p * N + n] * Sp[p * N + n];
            }
            dxt[p] = D[h] * dyt[p] + dtv * gb;
            xgb += xt[p] * gb;
            dydx += dyt[p] * xt[p];
        }
        /* S_t = a_t S_{t-1} + dt_t x_t B_t^T,  a_t = exp(dt_t A_h) */
        ddt[(b * L + t) * H + h] = xgb + A[h] * at * gs;
        dA_part[h] += dtv * at * gs;
        dD_part[h] += dydx;
        for (int64_t k = 0; k < PN; ++k) Gm[k] *= at;
    }
    if (dinit) memcpy(dinit + (b * H + h) * PN, Gm, sizeof(double) * (size_t)PN);
}

int ssd_oracle_backward(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                        int64_t dstate, int64_t ngroups, const double* x, const double* dt,
                        const double* A, const double* B, const double* C, const double* D,
                        const double* init, const double* dy, const double* dfinal,
                        double* dx, double* ddt, double* dA, double* dB, double* dC,
                        double* dD, double* dinit) {
    if (!dims_ok(batch, seqlen, nheads, headdim, dstate, ngroups)) return -1;
    if (!A || !D || !dA || !dD) return -1;
    const int have_tokens = seqlen > 0 && batch > 0;
    if (have_tokens && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC)) return -1;
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    const int64_t PN = P * N;
    if (have_tokens) {
        memset(dx, 0, sizeof(double) * (size_t)(batch * L * H * P));
        memset(ddt, 0, sizeof(double) * (size_t)(batch * L * H));
        memset(dB, 0, sizeof(double) * (size_t)(batch * L * G * N));
        memset(dC, 0, sizeof(double) * (size_t)(batch * L * G * N));
    }
    memset(dA, 0, sizeof(double) * (size_t)H);
    memset(dD, 0, sizeof(double) * (size_t)H);
    double* Sall = (double*)malloc(sizeof(double) * (size_t)((L + 1) * PN));
    double* Gm = (double*)malloc(sizeof(double) * (size_t)PN);
    if (!Sall || !Gm) {
        free(Sall);
        free(Gm);
        return -1;
    }
    /* sequential over (batch, head): dB, dC are shared by a group's heads and
     * dA, dD by the batch, so one order of summation, no races */
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t h = 0; h < H; ++h)
            bwd_one(b, h, L, H, P, N, G, x, dt, A, B, C, D, init, dy, dfinal, dx, ddt, dA, dB,
                    dC, dD, dinit, Sall, Gm);
    free(Sall);
    free(Gm);
    return 0;
}
