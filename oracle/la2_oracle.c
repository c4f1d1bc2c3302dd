/*
 * la2_oracle.c -- CPU fp64 oracle for Lightning Attention-2 (causal linear
 * attention with per-head decay), forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (per independent sequence of length T, identity feature
 * map, no normaliser, no 1/sqrt(d) scale):
 *
 *     o_t = sum_{s<=t} lambda^(t-s) (q_t . k_s) v_s
 *
 * This is causal linear attention as the "Lightning Attention" explainer page
 * (lizeman.github.io llm-arch-kb, section 1 "Premise") writes it, with the
 * feature map phi set to the identity (section 2, "Let phi ... Qin et al. use
 * the identity"), the denominator dropped (the default configuration pairs the
 * identity map with a normalisation gate instead of a divisor), and a per-head
 * decay lambda in (0,1] on the term of lag t-s, lambda = 1 giving the plain
 * prefix sum of section 1.
 *
 * Functions:
 *   la2o_forward            serial prefix-sum recurrence of section 1,
 *                           S_t = lambda S_{t-1} + k_t v_t^T,  o_t = S_t^T q_t.
 *   la2o_backward           gradients of L = sum_t do_t . o_t by the two
 *                           recurrences that differentiate the one above:
 *                           dq_t = S_t do_t (forward sweep);
 *                           R_t = lambda R_{t+1} + q_t do_t^T,
 *                           dk_t = R_t v_t, dv_t = R_t^T k_t (reverse sweep).
 *   la2o_forward_blocked    the tiled algorithm of section 2 (steps 1-4:
 *                           intra-tile masked product, inter-tile product with
 *                           the running state, state update), with the decay
 *                           folded into each step.  The decay exponents are not
 *                           printed on the pages; they are derived from the
 *                           definition above:
 *                             intra weight   lambda^(r-c), r >= c
 *                             inter weight   lambda^(r+1) on row r
 *                             state update   KV <- lambda^TB KV
 *                                                  + sum_r lambda^(TB-1-r) k_r v_r^T
 *   la2o_forward_state      la2o_forward from a given state: S_{-1} = S0 instead
 *                           of 0, and the state after the last token returned
 *                           (the state is the only thing a sequence carries,
 *                           section 2 "Memory footprint", so a long sequence
 *                           can be processed in consecutive pieces).
 *   la2o_backward_state     gradients of L = sum_t do_t . o_t + <G, S_{T-1}>
 *                           for the forward from a given state S_{-1} = S0:
 *                           dq, dk, dv, and dS0.  G (the gradient arriving at
 *                           the final state) enters the reverse sweep at the
 *                           last position: R_{T-1} = q_{T-1} do_{T-1}^T + G,
 *                           R_t = lambda R_{t+1} + q_t do_t^T; dq_t = S_t do_t
 *                           with S_t started from S0; dS0 = lambda R_0 (G
 *                           when T = 0).  This is what a sequence trained in
 *                           consecutive pieces needs (section 2, "Memory
 *                           footprint": the state is all a piece carries).
 *   la2o_dlambda            the gradient of the same L with respect to lambda
 *                           (one scalar per sequence), by differentiating the
 *                           recurrence: U_t = dS_t/dlambda obeys
 *                           U_t = lambda U_{t-1} + S_{t-1} (U_{-1} = 0), and
 *                           dL/dlambda = sum_t q_t^T U_t do_t + <G, U_{T-1}>.
 *   la2o_forward_norm       the normalised form of section 1 (feature map
 *                           identity, as section 2 says the default is; any
 *                           other phi is applied to q and k beforehand), with
 *                           the same decay on the denominator's running sum:
 *                           z_t = lambda z_{t-1} + k_t, den_t = q_t . z_t,
 *                           y_t = (S_t^T q_t) / den_t.
 *   la2o_backward_norm      gradients of L = sum_t dy_t . y_t through it:
 *                           dnum_t = dy_t / den_t, dden_t = -(dy_t . num_t) / den_t^2,
 *                           dq_t = S_t dnum_t + dden_t z_t; reverse sweep
 *                           R_t = lambda R_{t+1} + q_t dnum_t^T,
 *                           r_t = lambda r_{t+1} + dden_t q_t,
 *                           dk_t = R_t v_t + r_t, dv_t = R_t^T k_t.
 *   la2o_decode_step        one step of the same recurrence for one new token
 *                           per sequence: S <- lambda S + k v^T, o = S^T q.
 *   la2o_backward_blocked   the mirrored tiling for the backward (the pages say
 *                           only that tiling covers the backward too): dq by a
 *                           forward-direction blocked scan, dk and dv by a
 *                           reverse-direction blocked scan with
 *                             intra weight   lambda^(c-r), c >= r
 *                             inter weight   lambda^(TB-r) on row r
 *                             state update   R <- lambda^TB R
 *                                                 + sum_r lambda^r q_r do_r^T
 *
 * Layout: sequence-major, row-major: x[n][t][j] for sequence n, position t,
 * feature j.  lam[n] is the decay of sequence n.  All arithmetic is double.
 * Sequences are independent; they are split across OpenMP threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int la2o_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* lambda^n for an integer n >= 0, by the C library's pow in double. */
static double lpow(double lam, int n) { return pow(lam, (double)n); }

/* ---------------------------------------------------------------- forward */

void la2o_forward(int NS, int T, int d, int e, const double *lam,
                  const double *q, const double *k, const double *v,
                  double *o, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d;
        const double *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        double *on = o + (size_t)n * T * e;
        double *S = (double *)calloc((size_t)d * e, sizeof(double)); /* S[i][j] */
        const double l = lam[n];
        for (int t = 0; t < T; ++t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e;
            /* S_t = lambda S_{t-1} + k_t v_t^T */
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            /* o_t = S_t^T q_t */
            double *ot = on + (size_t)t * e;
            for (int j = 0; j < e; ++j) ot[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) ot[j] += qt[i] * S[(size_t)i * e + j];
        }
        free(S);
    }
}

/* ------------------------------------------------- state in / state out */

void la2o_forward_state(int NS, int T, int d, int e, const double *lam,
                        const double *q, const double *k, const double *v,
                        const double *s0, double *o, double *sT, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d;
        const double *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        double *on = o + (size_t)n * T * e;
        double *S = sT + (size_t)n * d * e; /* S[i][j], starts as S0 (or 0) */
        if (s0) memcpy(S, s0 + (size_t)n * d * e, sizeof(double) * (size_t)d * e);
        else memset(S, 0, sizeof(double) * (size_t)d * e);
        const double l = lam[n];
        for (int t = 0; t < T; ++t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            double *ot = on + (size_t)t * e;
            for (int j = 0; j < e; ++j) ot[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) ot[j] += qt[i] * S[(size_t)i * e + j];
        }
    }
}

void la2o_decode_step(int NS, int d, int e, const double *lam, const double *q,
                      const double *k, const double *v, double *S, double *o)
{
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * d, *kn = k + (size_t)n * d, *vn = v + (size_t)n * e;
        double *Sn = S + (size_t)n * d * e, *on = o + (size_t)n * e;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < e; ++j)
                Sn[(size_t)i * e + j] = lam[n] * Sn[(size_t)i * e + j] + kn[i] * vn[j];
        for (int j = 0; j < e; ++j) on[j] = 0.0;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < e; ++j) on[j] += qn[i] * Sn[(size_t)i * e + j];
    }
}

/* --------------------------------------------------------------- backward */

void la2o_backward(int NS, int T, int d, int e, const double *lam,
                   const double *q, const double *k, const double *v,
                   const double *dout, double *dq, double *dk, double *dv,
                   int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d;
        const double *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        const double *gn = dout + (size_t)n * T * e;
        double *dqn = dq + (size_t)n * T * d;
        double *dkn = dk + (size_t)n * T * d;
        double *dvn = dv + (size_t)n * T * e;
        double *S = (double *)calloc((size_t)d * e, sizeof(double));
        const double l = lam[n];

        /* forward sweep: dq_t = S_t do_t, S_t as in the forward pass */
        for (int t = 0; t < T; ++t) {
            const double *kt = kn + (size_t)t * d, *vt = vn + (size_t)t * e;
            const double *gt = gn + (size_t)t * e;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            double *dqt = dqn + (size_t)t * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < e; ++j) acc += S[(size_t)i * e + j] * gt[j];
                dqt[i] = acc;
            }
        }

        /* reverse sweep: R_t = lambda R_{t+1} + q_t do_t^T,
           dk_t = R_t v_t, dv_t = R_t^T k_t                     */
        double *R = S;
        memset(R, 0, sizeof(double) * (size_t)d * e);
        for (int t = T - 1; t >= 0; --t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e, *gt = gn + (size_t)t * e;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    R[(size_t)i * e + j] = l * R[(size_t)i * e + j] + qt[i] * gt[j];
            double *dkt = dkn + (size_t)t * d, *dvt = dvn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < e; ++j) acc += R[(size_t)i * e + j] * vt[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < e; ++j) dvt[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) dvt[j] += R[(size_t)i * e + j] * kt[i];
        }
        free(S);
    }
}

/* ------------------------------------------- backward with carried state */

void la2o_backward_state(int NS, int T, int d, int e, const double *lam,
                         const double *q, const double *k, const double *v,
                         const double *dout, const double *s0, const double *dsT,
                         double *dq, double *dk, double *dv, double *ds0,
                         int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d;
        const double *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        const double *gn = dout + (size_t)n * T * e;
        double *dqn = dq + (size_t)n * T * d;
        double *dkn = dk + (size_t)n * T * d;
        double *dvn = dv + (size_t)n * T * e;
        double *S = (double *)calloc((size_t)d * e, sizeof(double));
        const double l = lam[n];

        /* forward sweep from S_{-1} = S0: dq_t = S_t do_t */
        if (s0) memcpy(S, s0 + (size_t)n * d * e, sizeof(double) * (size_t)d * e);
        for (int t = 0; t < T; ++t) {
            const double *kt = kn + (size_t)t * d, *vt = vn + (size_t)t * e;
            const double *gt = gn + (size_t)t * e;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            double *dqt = dqn + (size_t)t * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < e; ++j) acc += S[(size_t)i * e + j] * gt[j];
                dqt[i] = acc;
            }
        }

        /* reverse sweep: R starts as G at the last position (no decay there),
           R_t = lambda R_{t+1} + q_t do_t^T before it; dk_t = R_t v_t,
           dv_t = R_t^T k_t */
        double *R = S;
        if (dsT) memcpy(R, dsT + (size_t)n * d * e, sizeof(double) * (size_t)d * e);
        else memset(R, 0, sizeof(double) * (size_t)d * e);
        for (int t = T - 1; t >= 0; --t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e, *gt = gn + (size_t)t * e;
            const double f = (t == T - 1) ? 1.0 : l;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    R[(size_t)i * e + j] = f * R[(size_t)i * e + j] + qt[i] * gt[j];
            double *dkt = dkn + (size_t)t * d, *dvt = dvn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < e; ++j) acc += R[(size_t)i * e + j] * vt[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < e; ++j) dvt[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) dvt[j] += R[(size_t)i * e + j] * kt[i];
        }
        /* S_0 = lambda S_{-1} + k_0 v_0^T, so dS_{-1} = lambda R_0; with no
           position at all, S_{T-1} is S_{-1} itself */
        double *g0 = ds0 + (size_t)n * d * e;
        for (size_t z = 0; z < (size_t)d * e; ++z) g0[z] = T > 0 ? l * R[z] : R[z];
        free(S);
    }
}

/* ------------------------------------------------- gradient in lambda */

void la2o_dlambda(int NS, int T, int d, int e, const double *lam,
                  const double *q, const double *k, const double *v,
                  const double *dout, const double *s0, const double *dsT,
                  double *dlam, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d;
        const double *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        const double *gn = dout + (size_t)n * T * e;
        double *S = (double *)calloc((size_t)d * e, sizeof(double));
        double *U = (double *)calloc((size_t)d * e, sizeof(double));
        const double l = lam[n];
        if (s0) memcpy(S, s0 + (size_t)n * d * e, sizeof(double) * (size_t)d * e);
        double acc = 0.0;
        for (int t = 0; t < T; ++t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e, *gt = gn + (size_t)t * e;
            /* U_t = lambda U_{t-1} + S_{t-1}, then S_t = lambda S_{t-1} + k_t v_t^T */
            for (size_t z = 0; z < (size_t)d * e; ++z) U[z] = l * U[z] + S[z];
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            /* q_t^T U_t do_t */
            for (int i = 0; i < d; ++i) {
                double r = 0.0;
                for (int j = 0; j < e; ++j) r += U[(size_t)i * e + j] * gt[j];
                acc += qt[i] * r;
            }
        }
        if (dsT && T > 0) {
            const double *g = dsT + (size_t)n * d * e;
            for (size_t z = 0; z < (size_t)d * e; ++z) acc += g[z] * U[z];
        }
        dlam[n] = acc;
        free(S);
        free(U);
    }
}

/* ------------------------------------------------- normalised variant */

void la2o_forward_norm(int NS, int T, int d, int e, const double *lam,
                       const double *q, const double *k, const double *v,
                       double *y, double *den, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d, *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e;
        double *yn = y + (size_t)n * T * e, *dn = den + (size_t)n * T;
        double *S = (double *)calloc((size_t)d * e, sizeof(double));
        double *z = (double *)calloc((size_t)d, sizeof(double));
        const double l = lam[n];
        for (int t = 0; t < T; ++t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                z[i] = l * z[i] + kt[i];
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            }
            double dd = 0.0;
            for (int i = 0; i < d; ++i) dd += qt[i] * z[i];
            dn[t] = dd;
            double *yt = yn + (size_t)t * e;
            for (int j = 0; j < e; ++j) yt[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) yt[j] += qt[i] * S[(size_t)i * e + j];
            for (int j = 0; j < e; ++j) yt[j] /= dd;
        }
        free(S);
        free(z);
    }
}

void la2o_backward_norm(int NS, int T, int d, int e, const double *lam,
                        const double *q, const double *k, const double *v,
                        const double *dy, double *dq, double *dk, double *dv,
                        int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d, *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e, *gn = dy + (size_t)n * T * e;
        double *dqn = dq + (size_t)n * T * d, *dkn = dk + (size_t)n * T * d;
        double *dvn = dv + (size_t)n * T * e;
        double *S = (double *)calloc((size_t)d * e, sizeof(double));
        double *z = (double *)calloc((size_t)d, sizeof(double));
        double *dnum = (double *)malloc(sizeof(double) * ((size_t)T * e + 1));
        double *dden = (double *)malloc(sizeof(double) * ((size_t)T + 1));
        const double l = lam[n];
        /* forward sweep: S_t, z_t, num_t, den_t; dq_t = S_t dnum_t + dden_t z_t */
        for (int t = 0; t < T; ++t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e, *gt = gn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                z[i] = l * z[i] + kt[i];
                for (int j = 0; j < e; ++j)
                    S[(size_t)i * e + j] = l * S[(size_t)i * e + j] + kt[i] * vt[j];
            }
            double den = 0.0;
            for (int i = 0; i < d; ++i) den += qt[i] * z[i];
            double gnum = 0.0;
            for (int j = 0; j < e; ++j) {
                double num = 0.0;
                for (int i = 0; i < d; ++i) num += qt[i] * S[(size_t)i * e + j];
                gnum += gt[j] * num;
                dnum[(size_t)t * e + j] = gt[j] / den;
            }
            dden[t] = -gnum / (den * den);
            double *dqt = dqn + (size_t)t * d;
            for (int i = 0; i < d; ++i) {
                double acc = dden[t] * z[i];
                for (int j = 0; j < e; ++j) acc += S[(size_t)i * e + j] * dnum[(size_t)t * e + j];
                dqt[i] = acc;
            }
        }
        /* reverse sweep: R_t = lambda R_{t+1} + q_t dnum_t^T, r_t = lambda r_{t+1} + dden_t q_t */
        double *R = S, *r = z;
        memset(R, 0, sizeof(double) * (size_t)d * e);
        memset(r, 0, sizeof(double) * (size_t)d);
        for (int t = T - 1; t >= 0; --t) {
            const double *qt = qn + (size_t)t * d, *kt = kn + (size_t)t * d;
            const double *vt = vn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                r[i] = l * r[i] + dden[t] * qt[i];
                for (int j = 0; j < e; ++j)
                    R[(size_t)i * e + j] = l * R[(size_t)i * e + j] + qt[i] * dnum[(size_t)t * e + j];
            }
            double *dkt = dkn + (size_t)t * d, *dvt = dvn + (size_t)t * e;
            for (int i = 0; i < d; ++i) {
                double acc = r[i];
                for (int j = 0; j < e; ++j) acc += R[(size_t)i * e + j] * vt[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < e; ++j) dvt[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < e; ++j) dvt[j] += R[(size_t)i * e + j] * kt[i];
        }
        free(S);
        free(z);
        free(dnum);
        free(dden);
    }
}

/* ------------------------------------------------------- blocked variants */

/*
 * One blocked scan, used for the forward pass and for every backward output:
 *
 *   dir = +1:  x_t = sum_{s<=t} lambda^(t-s) (a_t . b_s) c_s
 *   dir = -1:  x_t = sum_{s>=t} lambda^(s-t) (a_t . b_s) c_s
 *
 * a, b are [T][da]; c, x are [T][dc].  Tiles are the contiguous ranges
 * [i*TB, min((i+1)*TB, T)); the last one may be short.  For dir = +1 the tiles
 * are visited first to last, for dir = -1 last to first.  Within tile i, with
 * local row r and local column c:
 *
 *   dir = +1:  x_r = sum_{c<=r} lambda^(r-c) (a_r . b_c) c_c  +  lambda^(r+1) a_r^T W
 *              W  <- lambda^TB W + sum_c lambda^(TB-1-c) b_c c_c^T
 *   dir = -1:  x_r = sum_{c>=r} lambda^(c-r) (a_r . b_c) c_c  +  lambda^(TB-r) a_r^T W
 *              W  <- lambda^TB W + sum_c lambda^c b_c c_c^T
 *
 * W (da x dc) starts at zero.  Every exponent is measured from a tile's first
 * row, so a short last tile needs no special case: in the forward direction
 * the state after it is never used, and in the reverse direction it is the
 * first tile visited, where W is still zero, and the state it leaves behind is
 * sum_c lambda^c b_c c_c^T, exactly the lag from the start of the tile.
 */
static void blocked_scan(int T, int da, int dc, int TB, int dir, double lam,
                         const double *a, const double *b, const double *c,
                         double *x)
{
    const int nb = (T + TB - 1) / TB;
    double *W = (double *)calloc((size_t)da * dc, sizeof(double));
    double *Wn = (double *)calloc((size_t)da * dc, sizeof(double));
    const double lTB = lpow(lam, TB);
    for (int step = 0; step < nb; ++step) {
        const int i = dir > 0 ? step : nb - 1 - step;
        const int t0 = i * TB;
        const int len = (t0 + TB <= T) ? TB : T - t0;
        for (int r = 0; r < len; ++r) {
            const double *ar = a + (size_t)(t0 + r) * da;
            double *xr = x + (size_t)(t0 + r) * dc;
            for (int j = 0; j < dc; ++j) xr[j] = 0.0;
            /* intra-tile: masked, decayed left product */
            for (int cc = 0; cc < len; ++cc) {
                int lag = dir > 0 ? r - cc : cc - r;
                if (lag < 0) continue;
                const double *bc = b + (size_t)(t0 + cc) * da;
                double s = 0.0;
                for (int u = 0; u < da; ++u) s += ar[u] * bc[u];
                s *= lpow(lam, lag);
                const double *ccv = c + (size_t)(t0 + cc) * dc;
                for (int j = 0; j < dc; ++j) xr[j] += s * ccv[j];
            }
            /* inter-tile: right product with the running state */
            const double w = dir > 0 ? lpow(lam, r + 1) : lpow(lam, TB - r);
            for (int u = 0; u < da; ++u) {
                const double au = w * ar[u];
                for (int j = 0; j < dc; ++j) xr[j] += au * W[(size_t)u * dc + j];
            }
        }
        /* state update, using the unmasked tile */
        for (size_t z = 0; z < (size_t)da * dc; ++z) Wn[z] = lTB * W[z];
        for (int cc = 0; cc < len; ++cc) {
            const double w = dir > 0 ? lpow(lam, TB - 1 - cc) : lpow(lam, cc);
            const double *bc = b + (size_t)(t0 + cc) * da;
            const double *ccv = c + (size_t)(t0 + cc) * dc;
            for (int u = 0; u < da; ++u) {
                const double bu = w * bc[u];
                for (int j = 0; j < dc; ++j) Wn[(size_t)u * dc + j] += bu * ccv[j];
            }
        }
        double *tmp = W; W = Wn; Wn = tmp;
    }
    free(W);
    free(Wn);
}

void la2o_forward_blocked(int NS, int T, int d, int e, int TB, const double *lam,
                          const double *q, const double *k, const double *v,
                          double *o, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n)
        blocked_scan(T, d, e, TB, +1, lam[n], q + (size_t)n * T * d,
                     k + (size_t)n * T * d, v + (size_t)n * T * e,
                     o + (size_t)n * T * e);
}

/*
 * Blocked backward.  Differentiating o_t = sum_{s<=t} lambda^(t-s)(q_t.k_s) v_s
 * against L = sum_t do_t . o_t gives
 *   dq_t = sum_{s<=t} lambda^(t-s) (do_t . v_s) k_s   forward scan (a=do, b=v, c=k)
 *   dk_s = sum_{t>=s} lambda^(t-s) (v_s . do_t) q_t   reverse scan (a=v, b=do, c=q)
 *   dv_s = sum_{t>=s} lambda^(t-s) (k_s . q_t) do_t   reverse scan (a=k, b=q, c=do)
 */
void la2o_backward_blocked(int NS, int T, int d, int e, int TB, const double *lam,
                           const double *q, const double *k, const double *v,
                           const double *dout, double *dq, double *dk, double *dv,
                           int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < NS; ++n) {
        const double *qn = q + (size_t)n * T * d, *kn = k + (size_t)n * T * d;
        const double *vn = v + (size_t)n * T * e, *gn = dout + (size_t)n * T * e;
        blocked_scan(T, e, d, TB, +1, lam[n], gn, vn, kn, dq + (size_t)n * T * d);
        blocked_scan(T, e, d, TB, -1, lam[n], vn, gn, qn, dk + (size_t)n * T * d);
        blocked_scan(T, d, e, TB, -1, lam[n], kn, qn, gn, dv + (size_t)n * T * e);
    }
}
