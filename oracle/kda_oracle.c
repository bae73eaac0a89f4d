/*
 * kda_oracle.c -- plain fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this
 * library: only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark call it.  It shares no code, header or constant with the
 * CUDA kernels.
 *
 * What it computes (source: "Kimi K3" open-weights field notes,
 * ailearn.mscapital.top/kimi-k3.html, panel "KDA 单头递归" -- KDA single-head
 * recurrence):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     alpha_t = exp(g_t)  (one forgetting factor per key channel),
 *     o_t     = S_t^T q_t (the query reads the UPDATED state).
 *
 * S is d_k x d_v; Diag(alpha_t) scales the rows (key channels) of S.  Every
 * (sequence, head) chain is independent, so the chains are spread over OpenMP
 * threads; the arithmetic inside a chain is the recurrence above, token by
 * token, in the printed order: decay first, then the delta-rule erase/write,
 * then the read.  No chunking, blocking or reassociation.
 *
 * Layouts (row-major, contiguous, fp64):
 *   q, k, g : [T_total, H, d_k]     v, o : [T_total, H, d_v]
 *   beta    : [T_total, H]
 *   h0, hT  : [N, H, d_k, d_v]      (h0 may be NULL: zero initial state)
 *   cu      : [N + 1] token offsets of the N packed sequences (int64)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Run one (sequence, head) chain over tokens [t0, t1).  S holds the d_k x d_v
 * state on entry and the final state on exit.  u is d_v scratch. */
static void kda_chain(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, int64_t t0,
                      int64_t t1, int64_t H, int64_t h, int64_t dk, int64_t dv,
                      double *S, double *o, double *u) {
    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = q + (t * H + h) * dk;
        const double *kt = k + (t * H + h) * dk;
        const double *gt = g + (t * H + h) * dk;
        const double *vt = v + (t * H + h) * dv;
        const double bt = beta[t * H + h];
        double *ot = o + (t * H + h) * dv;

        /* Diag(alpha_t) S_{t-1}: row i of S is scaled by exp(g_t[i]). */
        for (int64_t i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
        /* (I - beta k k^T) S' + beta k v^T, with S' the decayed state:
         * u = k^T S' (a d_v row), then S'_{ij} - beta k_i u_j + beta k_i v_j. */
        for (int64_t j = 0; j < dv; ++j) u[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) u[j] += kt[i] * S[i * dv + j];
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j)
                S[i * dv + j] = S[i * dv + j] - bt * kt[i] * u[j] + bt * kt[i] * vt[j];
        /* o_t = S_t^T q_t. */
        for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) ot[j] += qt[i] * S[i * dv + j];
    }
}

/* Returns the number of OpenMP threads that ran chains (>= 1), or -1 on a bad
 * argument.  cu must be non-decreasing with cu[0] == 0. */
int kda_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *g, const double *beta, const double *h0,
                   const int64_t *cu, int64_t N, int64_t H, int64_t dk,
                   int64_t dv, int nthreads, double *o, double *hT) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu || !hT) return -1;
    for (int64_t n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return -1;
    if (cu[0] != 0) return -1;
    const int64_t units = N * H;
    int used = 1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    if ((int64_t)nthreads > units) nthreads = (int)(units > 0 ? units : 1);
#else
    nthreads = 1;
#endif
    used = nthreads;
    int bad = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!u) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t w = 0; w < units; ++w) {
            if (!u) continue;
            const int64_t n = w / H, h = w % H;
            double *S = hT + (n * H + h) * dk * dv;
            if (h0) {
                const double *src = h0 + (n * H + h) * dk * dv;
                if (src != S) memmove(S, src, sizeof(double) * (size_t)(dk * dv));
            } else
                memset(S, 0, sizeof(double) * (size_t)(dk * dv));
            kda_chain(q, k, v, g, beta, cu[n], cu[n + 1], H, h, dk, dv, S, o, u);
        }
        free(u);
    }
    return bad ? -1 : used;
}
