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

/*
 * Backward pass: the reverse-mode derivative of the KDA recurrence above, for
 * training (news digest page on Kimi Linear, section "Algorithme parallele
 * par chunks": the chunk algebra is organised for training throughput; the
 * derivative itself is the chain rule through each step of the recurrence).
 *
 * Given dL/do for every token and dL/dS_T for every sequence (NULL = 0), it
 * returns dL/dq, dL/dk, dL/dv, dL/dg, dL/dbeta and dL/dS_0.  Step t of the
 * forward, with Sp = Diag(exp(g_t)) S_{t-1}:
 *     r = Sp^T k,   u = beta (v - r),   S_t = Sp + k u^T,   o_t = S_t^T q
 * read backwards, with dS holding dL/dS_t on entry (the later steps' share):
 *     dS   += q do^T                      (o_t = S_t^T q)
 *     dq    = S_t do
 *     du    = dS^T k,  dk = dS u          (S_t = Sp + k u^T)
 *     dbeta = du . (v - r),  dv = beta du,  dr = -beta du
 *     dSp   = dS + k dr^T,  dk += Sp dr   (r = Sp^T k)
 *     dg[c] = sum_j Sp[c][j] dSp[c][j]    (Sp[c][.] = exp(g[c]) S_{t-1}[c][.])
 *     dS    = Diag(exp(g_t)) dSp          -> dL/dS_{t-1}
 * The states entering each step are recomputed from the state entering each
 * block of 64 steps, which the forward keeps (so memory is one state per 64
 * tokens plus 64 states).  Outputs use the forward's layouts; every gradient is
 * written (not accumulated).
 */

/* One forward step on S (the recurrence above, without the read-out). */
static void kda_oracle_step(double *S, double *r, const double *kt, const double *gt,
                            const double *vt, double bt, int dk, int dv)
{
    for (int c = 0; c < dk; ++c) {
        const double a = exp(gt[c]);
        for (int j = 0; j < dv; ++j) S[(int64_t)c * dv + j] *= a;
    }
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) r[j] += S[(int64_t)c * dv + j] * kt[c];
    for (int j = 0; j < dv; ++j) r[j] = bt * (vt[j] - r[j]);
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(int64_t)c * dv + j] += kt[c] * r[j];
}

enum { kOracleBlock = 64 };

/* One (sequence, head): S holds S_0 on entry, dS holds dL/dS_T on entry and
 * dL/dS_0 on return.  Returns 0, or -2 when scratch allocation fails. */
static int kda_oracle_chain_backward(const double *q, const double *k, const double *v,
                                     const double *g, const double *beta, const double *d_o,
                                     int64_t t0, int64_t t1, int H, int h, int dk, int dv,
                                     double *S, double *dS, double *dq, double *dk_out,
                                     double *dv_out, double *dg, double *dbeta)
{
    const int64_t L = t1 - t0, se = (int64_t)dk * dv;
    const int64_t nb = (L + kOracleBlock - 1) / kOracleBlock;
    double *ck = (double *)malloc(sizeof(double) * (size_t)((nb > 0 ? nb : 1) * se));
    double *prev = (double *)malloc(sizeof(double) * (size_t)(kOracleBlock * se));
    double *Sp = (double *)malloc(sizeof(double) * (size_t)(2 * se + 4 * dv));
    if (!ck || !prev || !Sp) { free(ck); free(prev); free(Sp); return -2; }
    double *St = Sp + se, *r = St + se, *u = r + dv, *du = u + dv, *dr = du + dv;

    /* forward: keep the state entering every block */
    for (int64_t b = 0; b < nb; ++b) {
        memcpy(ck + b * se, S, sizeof(double) * (size_t)se);
        const int64_t te = (t0 + (b + 1) * kOracleBlock < t1) ? t0 + (b + 1) * kOracleBlock : t1;
        for (int64_t t = t0 + b * kOracleBlock; t < te; ++t)
            kda_oracle_step(S, r, k + (t * H + h) * (int64_t)dk, g + (t * H + h) * (int64_t)dk,
                            v + (t * H + h) * (int64_t)dv, beta[t * H + h], dk, dv);
    }
    /* backward, block by block from the end */
    for (int64_t b = nb - 1; b >= 0; --b) {
        const int64_t tb = t0 + b * kOracleBlock;
        const int64_t te = (tb + kOracleBlock < t1) ? tb + kOracleBlock : t1;
        memcpy(Sp, ck + b * se, sizeof(double) * (size_t)se);
        for (int64_t t = tb; t < te; ++t) {   /* the state entering each step */
            memcpy(prev + (t - tb) * se, Sp, sizeof(double) * (size_t)se);
            kda_oracle_step(Sp, r, k + (t * H + h) * (int64_t)dk, g + (t * H + h) * (int64_t)dk,
                            v + (t * H + h) * (int64_t)dv, beta[t * H + h], dk, dv);
        }
        for (int64_t t = te - 1; t >= tb; --t) {
            const double *qt = q + (t * H + h) * (int64_t)dk;
            const double *kt = k + (t * H + h) * (int64_t)dk;
            const double *gt = g + (t * H + h) * (int64_t)dk;
            const double *vt = v + (t * H + h) * (int64_t)dv;
            const double *dot = d_o + (t * H + h) * (int64_t)dv;
            const double bt = beta[t * H + h];
            const double *Sprev = prev + (t - tb) * se;
            double *dqt = dq + (t * H + h) * (int64_t)dk;
            double *dkt = dk_out + (t * H + h) * (int64_t)dk;
            double *dgt = dg + (t * H + h) * (int64_t)dk;
            double *dvt = dv_out + (t * H + h) * (int64_t)dv;

            /* the forward step again, keeping Sp, r, u and S_t */
            for (int c = 0; c < dk; ++c) {
                const double a = exp(gt[c]);
                for (int j = 0; j < dv; ++j) Sp[(int64_t)c * dv + j] = a * Sprev[(int64_t)c * dv + j];
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += Sp[(int64_t)c * dv + j] * kt[c];
                r[j] = acc;
                u[j] = bt * (vt[j] - acc);
            }
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j)
                    St[(int64_t)c * dv + j] = Sp[(int64_t)c * dv + j] + kt[c] * u[j];

            /* o_t = S_t^T q_t */
            for (int c = 0; c < dk; ++c)
                for (int j = 0; j < dv; ++j) dS[(int64_t)c * dv + j] += qt[c] * dot[j];
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += St[(int64_t)c * dv + j] * dot[j];
                dqt[c] = acc;
            }
            /* S_t = Sp + k u^T */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c) acc += dS[(int64_t)c * dv + j] * kt[c];
                du[j] = acc;
            }
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += dS[(int64_t)c * dv + j] * u[j];
                dkt[c] = acc;
            }
            /* u = beta (v - r) */
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                db += du[j] * (vt[j] - r[j]);
                dvt[j] = bt * du[j];
                dr[j] = -bt * du[j];
            }
            dbeta[t * H + h] = db;
            /* r = Sp^T k */
            for (int c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    dS[(int64_t)c * dv + j] += kt[c] * dr[j];
                    acc += Sp[(int64_t)c * dv + j] * dr[j];
                }
                dkt[c] += acc;
            }
            /* Sp = Diag(exp(g_t)) S_{t-1} */
            for (int c = 0; c < dk; ++c) {
                const double a = exp(gt[c]);
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += Sp[(int64_t)c * dv + j] * dS[(int64_t)c * dv + j];
                    dS[(int64_t)c * dv + j] *= a;
                }
                dgt[c] = acc;
            }
        }
    }
    free(ck); free(prev); free(Sp);
    return 0;
}

/* Returns 0 on success, -1 on a bad argument, -2 when scratch allocation fails.
 * d_final_state and init_state may be NULL (zeros); d_init_state may be NULL. */
int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *g, const double *beta,
                        const double *init_state, const int64_t *cu_seqlens,
                        int num_seqs, int H, int dk, int dv, const double *d_o,
                        const double *d_final_state, double *dq, double *dk_out,
                        double *dv_out, double *dg, double *dbeta, double *d_init_state,
                        int nthreads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !d_o || !dq || !dk_out ||
        !dv_out || !dg || !dbeta)
        return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    const int64_t units = (int64_t)num_seqs * H;
    const int64_t se = (int64_t)dk * dv;
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
        double *S = (double *)malloc(sizeof(double) * (size_t)(2 * se));
        if (!S) { failed |= 1; continue; }
        double *dS = S + se;
        if (init_state) memcpy(S, init_state + u * se, sizeof(double) * (size_t)se);
        else memset(S, 0, sizeof(double) * (size_t)se);
        if (d_final_state) memcpy(dS, d_final_state + u * se, sizeof(double) * (size_t)se);
        else memset(dS, 0, sizeof(double) * (size_t)se);
        if (kda_oracle_chain_backward(q, k, v, g, beta, d_o, cu_seqlens[s], cu_seqlens[s + 1],
                                      H, h, dk, dv, S, dS, dq, dk_out, dv_out, dg, dbeta) != 0)
            failed |= 1;
        else if (d_init_state)
            memcpy(d_init_state + u * se, dS, sizeof(double) * (size_t)se);
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
