/*
 * kda_oracle.c -- fp64 CPU oracle for the Kimi Delta Attention recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain statement of what the
 * KDA hot path computes.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header or constant with the
 * CUDA library under gated_delta_rule_108_b200/csrc, and neither side includes
 * or links the other.
 *
 * What it computes, token by token, for every (sequence, head) pair:
 *
 *   daiw.net "Kimi Delta Attention", section "KDA 的更新式" (the update equation):
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   with S in R^{d_k x d_v}, alpha_t in (0,1)^{d_k} one decay per key channel
 *   (section "一、Diag(alpha_t)：通道级遗忘") and beta_t a scalar write strength
 *   (section "二、I - beta_t k_t k_t^T：delta 规则").
 *
 *   news.bugfactory.tech/news/3610 (the paragraphs on DeltaNet, Gated DeltaNet
 *   and KDA) fixes the order of the steps the equation folds together:
 *   forget per channel, predict on the decayed state with the same key, form
 *   the error scaled by beta, write the error along the key, then read the
 *   query with the d_k^{-1/2} scale.  The read uses the state after the write
 *   (o_t = S_t^T q_t, as in the linear-attention recurrence on the kongchang.com
 *   page, section "循环视角下的线性注意力").
 *
 *   alpha_t = exp(log_alpha_t): the library takes the log of the decay, which
 *   keeps products of many decays representable.
 *
 * Layouts (all row-major, C order), Ttot = total packed tokens, N = sequences:
 *   q, k       [Ttot, H, dk]        v [Ttot, H, dv]
 *   log_alpha  [Ttot, H, dk]        beta [Ttot, H]
 *   S0         [N, H, dk, dv]  (NULL means zeros)
 *   cu_seqlens [N + 1], int64, cu_seqlens[0] = 0, non-decreasing, last = Ttot
 *   o          [Ttot, H, dv]        S_final [N, H, dk, dv] (NULL: not written)
 *
 * Work is split over (sequence, head) pairs with OpenMP when compiled with
 * -fopenmp; each pair runs its own serial token loop, so the result does not
 * depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns 0 on success, -1 on bad arguments, -2 if scratch allocation fails. */
int oracle_kda_forward(const double* q, const double* k, const double* v,
                       const double* log_alpha, const double* beta,
                       const double* S0, const int64_t* cu_seqlens,
                       int num_seqs, int H, int dk, int dv,
                       double* o, double* S_final)
{
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    const double scale = 1.0 / sqrt((double)dk);
    const long units = (long)num_seqs * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long unit = 0; unit < units; ++unit) {
        const int s = (int)(unit / H);
        const int h = (int)(unit % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* p = (double*)malloc(sizeof(double) * (size_t)dv);
        double* u = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!S || !p || !u) { free(S); free(p); free(u); failed |= 1; continue; }

        const size_t state_off = ((size_t)s * H + h) * (size_t)dk * dv;
        if (S0) memcpy(S, S0 + state_off, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);

        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            const double* kt = k + ((size_t)t * H + h) * dk;
            const double* qt = q + ((size_t)t * H + h) * dk;
            const double* vt = v + ((size_t)t * H + h) * dv;
            const double* lat = log_alpha + ((size_t)t * H + h) * dk;
            const double bt = beta[(size_t)t * H + h];
            double* ot = o + ((size_t)t * H + h) * dv;

            /* forget: each key channel (row i of S) decays by its own alpha */
            for (int i = 0; i < dk; ++i) {
                const double a = exp(lat[i]);
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
            }
            /* predict: what the decayed memory returns for key k_t */
            for (int j = 0; j < dv; ++j) p[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) p[j] += S[(size_t)i * dv + j] * kt[i];
            /* correct: the beta-scaled prediction error */
            for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - p[j]);
            /* write: add the error along the key direction */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kt[i] * u[j];
            /* read: the query against the updated memory, scaled by dk^-1/2 */
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)i * dv + j] * qt[i];
            for (int j = 0; j < dv; ++j) ot[j] *= scale;
        }
        if (S_final) memcpy(S_final + state_off, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(p); free(u);
    }
    return failed ? -2 : 0;
}

/* Number of threads the OpenMP loop above would use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
