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

/* ------------------------------------------------------------------------------
 * Gradient of the recurrence: reverse accumulation through the token loop above.
 *
 * The loss is any L whose gradients with respect to the outputs are given:
 * dO = dL/do_t for every token and dhT = dL/dS_T for each chain's final state
 * (NULL: zero).  Returned: dL/dq, dL/dk, dL/dv, dL/dg, dL/dbeta and dL/dh0 (the
 * last only if dh0 != NULL).  Per token t, with S' = Diag(exp g_t) S_{t-1},
 * u = S'^T k, delta = v - u, S_t = S' + beta k delta^T and o_t = S_t^T q, the
 * chain rule walked from the last token to the first, G being dL/dS_t:
 *   G     += q do_t^T          (the read o_t = S_t^T q)
 *   dq     = S_t do_t
 *   w      = G delta;   dbeta = k . w
 *   ddelta = beta G^T k;  dv = ddelta;  du = -ddelta
 *   dk     = beta w + S' du    (the write beta k delta^T and the erase u = S'^T k)
 *   G'     = G + k du^T        (everything reaching S')
 *   dg_i   = sum_j S'_ij G'_ij (S'_ij = exp(g_i) S_{t-1,ij})
 *   G      = Diag(exp g_t) G'  (reaching S_{t-1})
 * and dh0 = G at the end.  The states S_{t-1} are needed in reverse order: they are
 * recomputed forward, segment by segment, from states stored every SEG tokens, with
 * exactly the arithmetic of kda_chain (so they equal the forward pass's states).
 * ------------------------------------------------------------------------------ */
#define KDA_ORACLE_SEG 64

/* One token of the recurrence on S (no read-out), as in kda_chain. */
static void kda_step(const double *kt, const double *gt, const double *vt, double bt,
                     int64_t dk, int64_t dv, double *S, double *u) {
    for (int64_t i = 0; i < dk; ++i) {
        const double a = exp(gt[i]);
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    for (int64_t j = 0; j < dv; ++j) u[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) u[j] += kt[i] * S[i * dv + j];
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j)
            S[i * dv + j] = S[i * dv + j] - bt * kt[i] * u[j] + bt * kt[i] * vt[j];
}

/* Reverse pass of one (sequence, head) chain over tokens [t0, t1).  G holds dL/dS_T
 * on entry and dL/dh0 on exit.  S0 is the initial state (NULL: zero).  Scratch:
 * ck ((nseg + 1) states), st (SEG + 1 states), Sp (one state), vectors of d_k / d_v. */
static void kda_chain_bwd(const double *q, const double *k, const double *v, const double *g,
                          const double *beta, const double *dO, const double *S0, int64_t t0,
                          int64_t t1, int64_t H, int64_t h, int64_t dk, int64_t dv, double *G,
                          double *dq, double *dkk, double *dvv, double *dg, double *db,
                          double *ck, double *st, double *Sp, double *u, double *w,
                          double *dd) {
    const int64_t n = dk * dv, L = t1 - t0, nseg = (L + KDA_ORACLE_SEG - 1) / KDA_ORACLE_SEG;
    /* forward: the state at the start of every segment */
    double *S = st;
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)n);
    else memset(S, 0, sizeof(double) * (size_t)n);
    for (int64_t s = 0; s < nseg; ++s) {
        memcpy(ck + s * n, S, sizeof(double) * (size_t)n);
        const int64_t a = t0 + s * KDA_ORACLE_SEG, b = a + KDA_ORACLE_SEG < t1 ? a + KDA_ORACLE_SEG : t1;
        for (int64_t t = a; t < b; ++t)
            kda_step(k + (t * H + h) * dk, g + (t * H + h) * dk, v + (t * H + h) * dv,
                     beta[t * H + h], dk, dv, S, u);
    }
    for (int64_t s = nseg - 1; s >= 0; --s) {
        const int64_t a = t0 + s * KDA_ORACLE_SEG, b = a + KDA_ORACLE_SEG < t1 ? a + KDA_ORACLE_SEG : t1;
        /* st[i] = state before token a + i, st[b - a] = state after the segment */
        memcpy(st, ck + s * n, sizeof(double) * (size_t)n);
        for (int64_t t = a; t < b; ++t) {
            double *nx = st + (t - a + 1) * n;
            memcpy(nx, st + (t - a) * n, sizeof(double) * (size_t)n);
            kda_step(k + (t * H + h) * dk, g + (t * H + h) * dk, v + (t * H + h) * dv,
                     beta[t * H + h], dk, dv, nx, u);
        }
        for (int64_t t = b - 1; t >= a; --t) {
            const double *qt = q + (t * H + h) * dk, *kt = k + (t * H + h) * dk;
            const double *gt = g + (t * H + h) * dk, *vt = v + (t * H + h) * dv;
            const double *dot = dO + (t * H + h) * dv;
            const double bt = beta[t * H + h];
            const double *Sprev = st + (t - a) * n, *St = st + (t - a + 1) * n;
            double *dqt = dq + (t * H + h) * dk, *dkt = dkk + (t * H + h) * dk;
            double *dvt = dvv + (t * H + h) * dv, *dgt = dg + (t * H + h) * dk;
            /* S' = Diag(exp g) S_{t-1}; u = S'^T k; delta (in u) = v - u */
            for (int64_t i = 0; i < dk; ++i) {
                const double a_i = exp(gt[i]);
                for (int64_t j = 0; j < dv; ++j) Sp[i * dv + j] = Sprev[i * dv + j] * a_i;
            }
            for (int64_t j = 0; j < dv; ++j) u[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) u[j] += kt[i] * Sp[i * dv + j];
            for (int64_t j = 0; j < dv; ++j) u[j] = vt[j] - u[j];
            /* G += q do^T */
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) G[i * dv + j] += qt[i] * dot[j];
            /* dq = S_t do */
            for (int64_t i = 0; i < dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < dv; ++j) x += St[i * dv + j] * dot[j];
                dqt[i] = x;
            }
            /* w = G delta; dbeta = k . w */
            double dbt = 0.0;
            for (int64_t i = 0; i < dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < dv; ++j) x += G[i * dv + j] * u[j];
                w[i] = x;
                dbt += kt[i] * x;
            }
            db[t * H + h] = dbt;
            /* ddelta = beta G^T k = dv; du = -ddelta */
            for (int64_t j = 0; j < dv; ++j) dd[j] = 0.0;
            for (int64_t i = 0; i < dk; ++i)
                for (int64_t j = 0; j < dv; ++j) dd[j] += G[i * dv + j] * kt[i];
            for (int64_t j = 0; j < dv; ++j) {
                dd[j] *= bt;
                dvt[j] = dd[j];
            }
            /* dk = beta w + S' du = beta w - S' ddelta */
            for (int64_t i = 0; i < dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < dv; ++j) x += Sp[i * dv + j] * dd[j];
                dkt[i] = bt * w[i] - x;
            }
            /* G' = G + k du^T = G - k ddelta^T; dg_i = sum_j S'_ij G'_ij; G = Diag(exp g) G' */
            for (int64_t i = 0; i < dk; ++i) {
                const double a_i = exp(gt[i]);
                double x = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    const double gp = G[i * dv + j] - kt[i] * dd[j];
                    x += Sp[i * dv + j] * gp;
                    G[i * dv + j] = a_i * gp;
                }
                dgt[i] = x;
            }
        }
    }
}

/* Returns the number of OpenMP threads used (>= 1), or -1 on a bad argument.
 * dO: [T_total, H, d_v]; dhT: [N, H, d_k, d_v] or NULL; outputs dq, dk, dg
 * [T_total, H, d_k], dv [T_total, H, d_v], dbeta [T_total, H], dh0 [N, H, d_k, d_v]
 * (may be NULL). */
int kda_oracle_bwd(const double *q, const double *k, const double *v, const double *g,
                   const double *beta, const double *h0, const int64_t *cu, int64_t N,
                   int64_t H, int64_t dk, int64_t dv, const double *dO, const double *dhT,
                   int nthreads, double *dq, double *dkk, double *dvv, double *dg,
                   double *db, double *dh0) {
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu || !dO) return -1;
    for (int64_t n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return -1;
    if (cu[0] != 0) return -1;
    int64_t maxlen = 0;
    for (int64_t n = 0; n < N; ++n)
        if (cu[n + 1] - cu[n] > maxlen) maxlen = cu[n + 1] - cu[n];
    const int64_t units = N * H, sz = dk * dv;
    const int64_t nseg_max = (maxlen + KDA_ORACLE_SEG - 1) / KDA_ORACLE_SEG;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
    if ((int64_t)nthreads > units) nthreads = (int)(units > 0 ? units : 1);
#else
    nthreads = 1;
#endif
    int bad = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double *ck = (double *)malloc(sizeof(double) * (size_t)((nseg_max + 1) * sz));
        double *st = (double *)malloc(sizeof(double) * (size_t)((KDA_ORACLE_SEG + 1) * sz));
        double *Sp = (double *)malloc(sizeof(double) * (size_t)sz);
        double *G = (double *)malloc(sizeof(double) * (size_t)sz);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *dd = (double *)malloc(sizeof(double) * (size_t)dv);
        double *w = (double *)malloc(sizeof(double) * (size_t)dk);
        const int ok = ck && st && Sp && G && u && dd && w;
        if (!ok) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t un = 0; un < units; ++un) {
            if (!ok) continue;
            const int64_t n = un / H, h = un % H;
            if (dhT) memcpy(G, dhT + (n * H + h) * sz, sizeof(double) * (size_t)sz);
            else memset(G, 0, sizeof(double) * (size_t)sz);
            kda_chain_bwd(q, k, v, g, beta, dO, h0 ? h0 + (n * H + h) * sz : NULL, cu[n],
                          cu[n + 1], H, h, dk, dv, G, dq, dkk, dvv, dg, db, ck, st, Sp, u, w,
                          dd);
            if (dh0) memcpy(dh0 + (n * H + h) * sz, G, sizeof(double) * (size_t)sz);
        }
        free(ck); free(st); free(Sp); free(G); free(u); free(dd); free(w);
    }
    return bad ? -1 : nthreads;
}
