/*
 * kda_oracle.c -- CPU fp64 reference for the Kimi Delta Attention (KDA)
 * forward recurrence.  TEST INFRASTRUCTURE ONLY: the product path never
 * links, loads or calls this file; only tests/, the smoke check and the
 * bench's CPU-baseline leg do.
 *
 * What it computes (plain token-by-token definition, no chunking):
 *
 *   For each sequence n and head h, S starts at S0[n,h] (zeros if absent),
 *   S is a dk x dv matrix (rows = key channels, columns = value channels).
 *   For every token t of the sequence, in order:
 *     1. gt  = max(g_t, g_floor);  alpha = exp(gt)          (natural log)
 *     2. P   = Diag(alpha) . S          -- each key row forgets at its own
 *                                          rate ("per-channel diagonal gate":
 *                                          page "Kimi-K3 为什么这么强？", §① ②)
 *     3. u   = P^T k_t                  -- what the state recalls for k_t
 *     4. S   = P + beta_t k_t (v_t - u)^T
 *             == (I - beta_t k_t k_t^T) P + beta_t k_t v_t^T
 *                                       -- the current key's row is weakened
 *                                          to (1-beta) and the new value is
 *                                          written in, leaving an
 *                                          interpolation (same page and
 *                                          section, the three-step figure)
 *     5. o_t = scale . S^T q_t          -- read-out with the state AFTER
 *                                          token t; then o_t *= sigmoid(z_t)
 *                                          when a gate is given (fupanwang.com
 *                                          Kimi K3 report digest, section
 *                                          "KDA：百万上下文先要过「数值 算子」
 *                                          这一关": the output gate is a
 *                                          channel-wise switch)
 *   S_T[n,h] = S after the last token.
 *
 *   The transition (I - beta k k^T) Diag(alpha) is diagonal-plus-low-rank
 *   (page "Kimi K3 深度拆解", 突破一).  The floor in step 1 bounds the
 *   per-step log-decay from below (fupanwang.com digest, KDA section, Fig. 3a);
 *   the page's formula for it is lost, so the floor is a parameter.
 *
 * Layouts (row-major, contiguous): q,k,g [T_tot,H,dk]; v,o,gate [T_tot,H,dv];
 * beta [T_tot,H]; S0,S_T [N,H,dk,dv].  Sequence n covers packed tokens
 * [cu_seqlens[n], cu_seqlens[n+1]).
 *
 * Every (n,h) unit is independent; OpenMP spreads units over host threads.
 * Within a unit the arithmetic is exactly steps 1-5 above in that order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns 0 on success, a negative value on bad arguments or allocation
 * failure. */
int kda_oracle_fwd(int32_t num_seqs, const int64_t *cu_seqlens, int32_t H,
                   int32_t dk, int32_t dv, const double *q, const double *k,
                   const double *v, const double *g, const double *beta,
                   const double *gate, const double *S0, double scale,
                   double g_floor, double *o, double *S_T, int32_t nthreads)
{
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens)
        return -1;
    for (int32_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n])
            return -2;
    if (cu_seqlens[num_seqs] > cu_seqlens[0] && (!q || !k || !v || !g || !beta || !o))
        return -3;

    const int64_t units = (int64_t)num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : failed)
#endif
    for (int64_t unit = 0; unit < units; ++unit) {
        const int32_t n = (int32_t)(unit / H);
        const int32_t h = (int32_t)(unit % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !u || !alpha) {
            free(S); free(u); free(alpha);
            failed |= 1;
            continue;
        }
        const size_t sdim = (size_t)dk * dv;
        if (S0)
            memcpy(S, S0 + (size_t)unit * sdim, sizeof(double) * sdim);
        else
            memset(S, 0, sizeof(double) * sdim);

        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const size_t rk = ((size_t)t * H + h) * dk;   /* row of q,k,g */
            const size_t rv = ((size_t)t * H + h) * dv;   /* row of v,o,z */
            const double *qt = q + rk, *kt = k + rk, *gt = g + rk;
            const double *vt = v + rv;
            const double bt = beta[(size_t)t * H + h];

            /* 1. retention factors with the floor */
            for (int32_t i = 0; i < dk; ++i) {
                double gi = gt[i] > g_floor ? gt[i] : g_floor;
                alpha[i] = exp(gi);
            }
            /* 2. P = Diag(alpha) S */
            for (int32_t i = 0; i < dk; ++i)
                for (int32_t j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] *= alpha[i];
            /* 3. u = P^T k */
            for (int32_t j = 0; j < dv; ++j)
                u[j] = 0.0;
            for (int32_t i = 0; i < dk; ++i)
                for (int32_t j = 0; j < dv; ++j)
                    u[j] += S[(size_t)i * dv + j] * kt[i];
            /* 4. S = P + beta k (v - u)^T */
            for (int32_t i = 0; i < dk; ++i)
                for (int32_t j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] += bt * kt[i] * (vt[j] - u[j]);
            /* 5. o = scale S^T q, then the optional sigmoid gate */
            double *ot = o + rv;
            for (int32_t j = 0; j < dv; ++j)
                ot[j] = 0.0;
            for (int32_t i = 0; i < dk; ++i)
                for (int32_t j = 0; j < dv; ++j)
                    ot[j] += S[(size_t)i * dv + j] * qt[i];
            for (int32_t j = 0; j < dv; ++j) {
                ot[j] *= scale;
                if (gate)
                    ot[j] *= 1.0 / (1.0 + exp(-gate[rv + j]));
            }
        }
        if (S_T)
            memcpy(S_T + (size_t)unit * sdim, S, sizeof(double) * sdim);
        free(S); free(u); free(alpha);
    }
    return failed ? -4 : 0;
}

/* Number of host threads OpenMP would use by default (1 without OpenMP). */
int32_t kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}
