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
