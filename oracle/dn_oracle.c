/*
 * dn_oracle.c -- plain, slow, fp64 CPU oracle for the causal delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library; both sides only see the same seeded inputs.
 *
 * What it computes (one independent problem per (b, h)):
 *
 *   state S is d_k x d_v, row-major [i][j] (row i = key channel, column j =
 *   value channel), starting from S0 (or zero).  For t = 0 .. T-1:
 *
 *     1. forget   Sd = decay(S)        none:      Sd = S
 *                                      scalar:    Sd = exp(g_t) * S
 *                                      per-key:   Sd[i][:] = exp(g_t[i]) * S[i][:]
 *     2. predict  p  = Sd^T k_t
 *     3. correct  e  = beta_t * (v_t - p)
 *     4. write    S  = Sd + k_t e^T
 *     5. read     o_t = S^T (scale * q_t)
 *
 *   This is the error form of the delta rule: "Linear attention and Gated
 *   DeltaNet" (inference.shantanugoel.com, ch. 28), sections "Correct: the
 *   delta rule" and "Gated DeltaNet" (displayed update equations) and "The
 *   recurrent form"; D2L section 12.5 "DeltaNet", slide "One rule, two
 *   readings" (error form); and for the per-key decay, "A walk through of the
 *   DeltaNet family of linear attention variants" (selinyilmaz.dev), the KDA
 *   update (forget each key channel, predict, correct, write, read) and its
 *   five-line reference recurrence.  The output is read after the write.
 *
 * Second form (transition, then write), D2L section 12.5, "One rule, two
 * readings" (matrix form) and slide "Gating: the modern cell":
 *
 *     M_t = (I - beta_t k_t k_t^T) Diag(alpha_t),  S = M_t S + beta_t k_t v_t^T
 *
 *   built as an explicit d_k x d_k matrix, so it shares no arithmetic shape
 *   with the error form.
 *
 * Additive rule (no correction, no decay), ch. 28 "Removing the softmax":
 *
 *     S = S + k_t v_t^T,  o_t = S^T (scale * q_t)
 *
 * All arrays are fp64, contiguous, [B][H][T][d] for tokens, [B][H][T] (scalar
 * gate, beta) or [B][H][T][d_k] (per-key gate), [B][H][d_k][d_v] for states.
 * OpenMP threads run over the B*H independent problems only; within a problem
 * the loops run in the order written above.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { DNO_GATE_NONE = 0, DNO_GATE_SCALAR = 1, DNO_GATE_PER_KEY = 2 };

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int dno_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Error form.  Returns 0, or -1 on a bad argument. */
int dno_delta_error_form(const double *q, const double *k, const double *v,
                         const double *beta, const double *g, int gate,
                         const double *S0, double *o, double *ST,
                         long B, long H, long T, long dk, long dv,
                         double scale, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if (gate != DNO_GATE_NONE && g == NULL) return -1;
    set_threads(nthreads);
    long nbh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < nbh; ++bh) {
        double *S = (double *)malloc(sizeof(double) * dk * dv);
        double *p = (double *)malloc(sizeof(double) * dv);
        double *e = (double *)malloc(sizeof(double) * dv);
        if (S0) memcpy(S, S0 + bh * dk * dv, sizeof(double) * dk * dv);
        else memset(S, 0, sizeof(double) * dk * dv);
        for (long t = 0; t < T; ++t) {
            long tok = bh * T + t;
            const double *qt = q + tok * dk, *kt = k + tok * dk, *vt = v + tok * dv;
            double bt = beta[tok];
            /* 1. forget */
            if (gate == DNO_GATE_SCALAR) {
                double a = exp(g[tok]);
                for (long x = 0; x < dk * dv; ++x) S[x] *= a;
            } else if (gate == DNO_GATE_PER_KEY) {
                const double *gt = g + tok * dk;
                for (long i = 0; i < dk; ++i) {
                    double a = exp(gt[i]);
                    for (long j = 0; j < dv; ++j) S[i * dv + j] *= a;
                }
            }
            /* 2. predict: p = Sd^T k */
            for (long j = 0; j < dv; ++j) p[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) p[j] += kt[i] * S[i * dv + j];
            /* 3. correct */
            for (long j = 0; j < dv; ++j) e[j] = bt * (vt[j] - p[j]);
            /* 4. write */
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * e[j];
            /* 5. read, after the write */
            double *ot = o + tok * dv;
            for (long j = 0; j < dv; ++j) ot[j] = 0.0;
            for (long i = 0; i < dk; ++i) {
                double qi = scale * qt[i];
                for (long j = 0; j < dv; ++j) ot[j] += qi * S[i * dv + j];
            }
        }
        if (ST) memcpy(ST + bh * dk * dv, S, sizeof(double) * dk * dv);
        free(S); free(p); free(e);
    }
    return 0;
}

/* Transition-then-write form with an explicit d_k x d_k transition. */
int dno_delta_transition_form(const double *q, const double *k, const double *v,
                              const double *beta, const double *g, int gate,
                              const double *S0, double *o, double *ST,
                              long B, long H, long T, long dk, long dv,
                              double scale, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if (gate != DNO_GATE_NONE && g == NULL) return -1;
    set_threads(nthreads);
    long nbh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < nbh; ++bh) {
        double *S = (double *)malloc(sizeof(double) * dk * dv);
        double *Sn = (double *)malloc(sizeof(double) * dk * dv);
        double *M = (double *)malloc(sizeof(double) * dk * dk);
        double *alpha = (double *)malloc(sizeof(double) * dk);
        if (S0) memcpy(S, S0 + bh * dk * dv, sizeof(double) * dk * dv);
        else memset(S, 0, sizeof(double) * dk * dv);
        for (long t = 0; t < T; ++t) {
            long tok = bh * T + t;
            const double *qt = q + tok * dk, *kt = k + tok * dk, *vt = v + tok * dv;
            double bt = beta[tok];
            for (long c = 0; c < dk; ++c) {
                if (gate == DNO_GATE_SCALAR) alpha[c] = exp(g[tok]);
                else if (gate == DNO_GATE_PER_KEY) alpha[c] = exp(g[tok * dk + c]);
                else alpha[c] = 1.0;
            }
            /* M = (I - beta k k^T) Diag(alpha): entry (r, c) */
            for (long r = 0; r < dk; ++r)
                for (long c = 0; c < dk; ++c)
                    M[r * dk + c] = ((r == c ? 1.0 : 0.0) - bt * kt[r] * kt[c]) * alpha[c];
            /* Sn = M S + beta k v^T */
            for (long r = 0; r < dk; ++r)
                for (long j = 0; j < dv; ++j) {
                    double acc = bt * kt[r] * vt[j];
                    for (long c = 0; c < dk; ++c) acc += M[r * dk + c] * S[c * dv + j];
                    Sn[r * dv + j] = acc;
                }
            memcpy(S, Sn, sizeof(double) * dk * dv);
            double *ot = o + tok * dv;
            for (long j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (long i = 0; i < dk; ++i) acc += S[i * dv + j] * (scale * qt[i]);
                ot[j] = acc;
            }
        }
        if (ST) memcpy(ST + bh * dk * dv, S, sizeof(double) * dk * dv);
        free(S); free(Sn); free(M); free(alpha);
    }
    return 0;
}

/* Additive (Hebbian) linear attention: no correction, no decay. */
int dno_additive(const double *q, const double *k, const double *v,
                 const double *S0, double *o, double *ST,
                 long B, long H, long T, long dk, long dv, double scale,
                 int nthreads) {
    if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    set_threads(nthreads);
    long nbh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < nbh; ++bh) {
        double *S = (double *)malloc(sizeof(double) * dk * dv);
        if (S0) memcpy(S, S0 + bh * dk * dv, sizeof(double) * dk * dv);
        else memset(S, 0, sizeof(double) * dk * dv);
        for (long t = 0; t < T; ++t) {
            long tok = bh * T + t;
            const double *qt = q + tok * dk, *kt = k + tok * dk, *vt = v + tok * dv;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * vt[j];
            double *ot = o + tok * dv;
            for (long j = 0; j < dv; ++j) ot[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) ot[j] += scale * qt[i] * S[i * dv + j];
        }
        if (ST) memcpy(ST + bh * dk * dv, S, sizeof(double) * dk * dv);
        free(S);
    }
    return 0;
}
