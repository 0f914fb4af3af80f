/*
 * KDA oracle: the plain, sequential, fp64 CPU form of the Kimi Delta Attention
 * recurrence.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; no product code path may.  It shares no
 * code, header or constant with the CUDA path.
 *
 * What it computes (page "Kimi Linear" on docsaid.org, section "KDA : une
 * decroissance propre a chaque canal", the KDA update equation; the same
 * equation on the course page "Attention lineaire et recurrence", section
 * "Kimi Delta Attention = les trois remedes combines"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t          (read-out with the updated state)
 *
 * with alpha_t = exp(g_t) given per key channel as g = log(alpha) <= 0.
 * The read-out S^T q is the associative read of the course page, section
 * "Le probleme de la memoire associative saturee" (S^T k returns v).
 *
 * Each step is taken in the order the equation reads from right to left:
 *   1. D S      : row c of S (key channel c) is scaled by exp(g_t[c]);
 *   2. r = (D S)^T k_t ;
 *   3. u = beta_t (v_t - r) ;
 *   4. S = D S + k_t u^T     which equals (I - beta k k^T) D S + beta k v^T;
 *   5. o_t = S^T q_t.
 * Step 4 is the same matrix as the printed equation, expanded:
 * (I - b k k^T) D S + b k v^T = D S + k (b v - b (D S)^T k)^T.
 *
 * Layouts (all row-major, contiguous, double):
 *   q, k, g : [T_total, H, d_k]     v, o : [T_total, H, d_v]
 *   beta    : [T_total, H]
 *   init_state / final_state : [num_seqs, H, d_k, d_v]  (d_v fastest)
 *   cu_seqlens : [num_seqs + 1] token offsets, cu_seqlens[0] = 0.
 * init_state may be NULL (zero state); final_state may be NULL.
 * Work is split over independent (sequence, head) pairs with OpenMP.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One (sequence, head) chain.  S is d_k x d_v scratch owned by the caller. */
static void kda_oracle_chain(const double *q, const double *k, const double *v,
                             const double *g, const double *beta,
                             int64_t t0, int64_t t1, int H, int h, int dk,
                             int dv, double *S, double *r, double *o)
{
    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = q + (t * H + h) * (int64_t)dk;
        const double *kt = k + (t * H + h) * (int64_t)dk;
        const double *gt = g + (t * H + h) * (int64_t)dk;
        const double *vt = v + (t * H + h) * (int64_t)dv;
        const double bt = beta[t * H + h];
        double *ot = o + (t * H + h) * (int64_t)dv;

        /* 1. Diag(alpha_t) S : decay row c by alpha_t[c] = exp(g_t[c]). */
        for (int c = 0; c < dk; ++c) {
            const double a = exp(gt[c]);
            double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* 2. r = (D S)^T k_t */
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) r[j] += row[j] * kt[c];
        }
        /* 3. u = beta_t (v_t - r), kept in r */
        for (int j = 0; j < dv; ++j) r[j] = bt * (vt[j] - r[j]);
        /* 4. S = D S + k_t u^T */
        for (int c = 0; c < dk; ++c) {
            double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kt[c] * r[j];
        }
        /* 5. o_t = S_t^T q_t */
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) ot[j] += row[j] * qt[c];
        }
    }
}

/* Returns 0 on success, -1 on a bad argument, -2 when scratch allocation fails. */
int kda_oracle_recurrence(const double *q, const double *k, const double *v,
                          const double *g, const double *beta,
                          const double *init_state, const int64_t *cu_seqlens,
                          int num_seqs, int H, int dk, int dv, double *o,
                          double *final_state, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o) return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    const int64_t units = (int64_t)num_seqs * H;
    const int64_t state_elems = (int64_t)dk * dv;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t u = 0; u < units; ++u) {
        const int s = (int)(u / H);
        const int h = (int)(u % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)(state_elems + dv));
        if (!S) { failed |= 1; continue; }
        double *r = S + state_elems;
        if (init_state)
            memcpy(S, init_state + u * state_elems, sizeof(double) * (size_t)state_elems);
        else
            memset(S, 0, sizeof(double) * (size_t)state_elems);
        kda_oracle_chain(q, k, v, g, beta, cu_seqlens[s], cu_seqlens[s + 1], H,
                         h, dk, dv, S, r, o);
        if (final_state)
            memcpy(final_state + u * state_elems, S, sizeof(double) * (size_t)state_elems);
        free(S);
    }
    return failed ? -2 : 0;
}

/*
 * Gated DeltaNet: the same memory with one scalar forget gate per token and
 * head (page "Kimi Linear" on docsaid.org, section "KDA : une decroissance
 * propre a chaque canal", the Gated DeltaNet update printed before the KDA
 * one; news digest page on Kimi Linear, section "De l'attention lineaire a
 * Gated DeltaNet"):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,   alpha_t = exp(g_t), g : [T_total, H].
 *
 * Taken as printed, the erase first and the scalar decay outside it:
 *   1. r = S_{t-1}^T k_t ;
 *   2. S = alpha_t (S_{t-1} - k_t (beta_t r)^T) + k_t (beta_t v_t)^T ;
 *   3. o_t = S_t^T q_t.
 * (Not the KDA loop with a repeated gate: the KDA loop decays first and
 * reads the decayed state; the two agree only because a scalar commutes with
 * I - beta k k^T, which the tests check.)
 */
static void gdn_oracle_chain(const double *q, const double *k, const double *v,
                             const double *g, const double *beta,
                             int64_t t0, int64_t t1, int H, int h, int dk,
                             int dv, double *S, double *r, double *o)
{
    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = q + (t * H + h) * (int64_t)dk;
        const double *kt = k + (t * H + h) * (int64_t)dk;
        const double *vt = v + (t * H + h) * (int64_t)dv;
        const double a = exp(g[t * H + h]);
        const double bt = beta[t * H + h];
        double *ot = o + (t * H + h) * (int64_t)dv;

        /* 1. r = S_{t-1}^T k_t */
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) r[j] += row[j] * kt[c];
        }
        /* 2. S = a (S - k (b r)^T) + k (b v)^T */
        for (int c = 0; c < dk; ++c) {
            double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j)
                row[j] = a * (row[j] - kt[c] * bt * r[j]) + kt[c] * bt * vt[j];
        }
        /* 3. o_t = S_t^T q_t */
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double *row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) ot[j] += row[j] * qt[c];
        }
    }
}

/* As kda_oracle_recurrence, with g : [T_total, H] (one gate per token and head). */
int gdn_oracle_recurrence(const double *q, const double *k, const double *v,
                          const double *g, const double *beta,
                          const double *init_state, const int64_t *cu_seqlens,
                          int num_seqs, int H, int dk, int dv, double *o,
                          double *final_state, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o) return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    const int64_t units = (int64_t)num_seqs * H;
    const int64_t state_elems = (int64_t)dk * dv;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t u = 0; u < units; ++u) {
        const int s = (int)(u / H);
        const int h = (int)(u % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)(state_elems + dv));
        if (!S) { failed |= 1; continue; }
        double *r = S + state_elems;
        if (init_state)
            memcpy(S, init_state + u * state_elems, sizeof(double) * (size_t)state_elems);
        else
            memset(S, 0, sizeof(double) * (size_t)state_elems);
        gdn_oracle_chain(q, k, v, g, beta, cu_seqlens[s], cu_seqlens[s + 1], H,
                         h, dk, dv, S, r, o);
        if (final_state)
            memcpy(final_state + u * state_elems, S, sizeof(double) * (size_t)state_elems);
        free(S);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
