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

/*
 * Reverse-mode derivative of the same recurrence (the chunkwise form is the
 * training mode on news.bugfactory.tech/news/3610, KDA paragraph, so its
 * gradients are part of what the path computes).
 *
 * For the scalar loss  L = sum_t <d_o_t, o_t> + <dS_final, S_final>  this returns
 * dL/dq, dL/dk, dL/dv, dL/dlog_alpha, dL/dbeta and dL/dS0.  It walks the
 * tokens of each sequence backwards, undoing the five steps of the forward
 * loop in reverse order (read, write, correct, predict, forget) by the chain
 * rule, with G = dL/dS_t carried from token to token:
 *
 *   read    o = c S_t^T q          dq = c S_t d_o          G += c q d_o^T
 *   write   S_t = X + k u^T        du = G^T k              dk += G u,  dX = G
 *   correct u = beta (v - p)       dbeta = <du, v - p>     dv = beta du,  dp = -beta du
 *   predict p = X^T k              dX += k dp^T            dk += X dp
 *   forget  X = Diag(a) S_{t-1}    dlog_alpha_i = sum_j dX_ij X_ij,  G = Diag(a) dX
 *
 * (X is the decayed state, c = dk^{-1/2}, a = exp(log_alpha_t).)  The states
 * S_{t-1} are recomputed from a copy of the state kept every kSegment tokens,
 * so memory stays at two segments of states per (sequence, head).
 *
 * Layouts as oracle_kda_forward; d_o like o; dS_final like S_final (NULL means
 * zeros); gradients like their inputs (dS0 like S0, always written).
 * Returns 0 on success, -1 on bad arguments, -2 if scratch allocation fails.
 */
enum { kSegment = 64 };

int oracle_kda_backward(const double* q, const double* k, const double* v,
                        const double* log_alpha, const double* beta,
                        const double* S0, const int64_t* cu_seqlens,
                        int num_seqs, int H, int dk, int dv,
                        const double* d_o, const double* dS_final,
                        double* dq, double* dk_out, double* dv_out,
                        double* dlog_alpha, double* dbeta, double* dS0)
{
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return -1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    const double c = pow((double)dk, -0.5);
    const size_t DD = (size_t)dk * dv;
    const long units = (long)num_seqs * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long unit = 0; unit < units; ++unit) {
        const int s = (int)(unit / H);
        const int h = (int)(unit % H);
        const int64_t t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
        const int64_t nseg = (t1 - t0 + kSegment - 1) / kSegment;
        /* ckpt[n]: state before token t0 + n*kSegment; prev[i]: S_{t-1} of segment token i */
        double* ckpt = (double*)malloc(sizeof(double) * DD * (size_t)(nseg > 0 ? nseg : 1));
        double* prev = (double*)malloc(sizeof(double) * DD * kSegment);
        double* cur = (double*)malloc(sizeof(double) * DD);   /* running state */
        double* X = (double*)malloc(sizeof(double) * DD);     /* decayed state of token t */
        double* G = (double*)malloc(sizeof(double) * DD);     /* dL/dS_t */
        double* pp = (double*)malloc(sizeof(double) * dv);
        double* uu = (double*)malloc(sizeof(double) * dv);
        double* du = (double*)malloc(sizeof(double) * dv);
        double* dp = (double*)malloc(sizeof(double) * dv);
        double* St = (double*)malloc(sizeof(double) * DD);
        if (!ckpt || !prev || !cur || !X || !G || !pp || !uu || !du || !dp || !St) {
            free(ckpt); free(prev); free(cur); free(X); free(G);
            free(pp); free(uu); free(du); free(dp); free(St);
            failed |= 1;
            continue;
        }
        const size_t state_off = ((size_t)s * H + h) * DD;

        /* forward sweep: keep the state entering every segment */
        if (S0) memcpy(cur, S0 + state_off, sizeof(double) * DD);
        else memset(cur, 0, sizeof(double) * DD);
        for (int64_t t = t0; t < t1; ++t) {
            if ((t - t0) % kSegment == 0) memcpy(ckpt + DD * (size_t)((t - t0) / kSegment), cur, sizeof(double) * DD);
            const double* kv = k + ((size_t)t * H + h) * dk;
            const double* vv = v + ((size_t)t * H + h) * dv;
            const double* lv = log_alpha + ((size_t)t * H + h) * dk;
            const double bv = beta[(size_t)t * H + h];
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) cur[(size_t)i * dv + j] *= exp(lv[i]);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += cur[(size_t)i * dv + j] * kv[i];
                uu[j] = bv * (vv[j] - acc);
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) cur[(size_t)i * dv + j] += kv[i] * uu[j];
        }

        /* backward sweep */
        if (dS_final) memcpy(G, dS_final + state_off, sizeof(double) * DD);
        else memset(G, 0, sizeof(double) * DD);
        for (int64_t n = nseg - 1; n >= 0; --n) {
            const int64_t ts = t0 + n * kSegment;
            const int64_t te = (ts + kSegment < t1) ? ts + kSegment : t1;
            /* recompute S_{t-1} for every token of the segment */
            memcpy(cur, ckpt + DD * (size_t)n, sizeof(double) * DD);
            for (int64_t t = ts; t < te; ++t) {
                memcpy(prev + DD * (size_t)(t - ts), cur, sizeof(double) * DD);
                const double* kv = k + ((size_t)t * H + h) * dk;
                const double* vv = v + ((size_t)t * H + h) * dv;
                const double* lv = log_alpha + ((size_t)t * H + h) * dk;
                const double bv = beta[(size_t)t * H + h];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) cur[(size_t)i * dv + j] *= exp(lv[i]);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += cur[(size_t)i * dv + j] * kv[i];
                    uu[j] = bv * (vv[j] - acc);
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) cur[(size_t)i * dv + j] += kv[i] * uu[j];
            }
            for (int64_t t = te - 1; t >= ts; --t) {
                const size_t tk = ((size_t)t * H + h) * dk, tv = ((size_t)t * H + h) * dv;
                const double* kv = k + tk;
                const double* qv = q + tk;
                const double* vv = v + tv;
                const double* lv = log_alpha + tk;
                const double bv = beta[(size_t)t * H + h];
                const double* Sp = prev + DD * (size_t)(t - ts);
                /* the forward step again: X, p, u and S_t of this token */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) X[(size_t)i * dv + j] = exp(lv[i]) * Sp[(size_t)i * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += X[(size_t)i * dv + j] * kv[i];
                    pp[j] = acc;
                    uu[j] = bv * (vv[j] - acc);
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) St[(size_t)i * dv + j] = X[(size_t)i * dv + j] + kv[i] * uu[j];

                /* read */
                const double* dot = d_o + tv;
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * dot[j];
                    dq[tk + i] = c * acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += c * qv[i] * dot[j];
                /* write */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += G[(size_t)i * dv + j] * kv[i];
                    du[j] = acc;
                }
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += G[(size_t)i * dv + j] * uu[j];
                    dk_out[tk + i] = acc;
                }
                /* correct */
                double db = 0.0;
                for (int j = 0; j < dv; ++j) {
                    db += du[j] * (vv[j] - pp[j]);
                    dv_out[tv + j] = bv * du[j];
                    dp[j] = -bv * du[j];
                }
                dbeta[(size_t)t * H + h] = db;
                /* predict: G becomes dL/dX */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += X[(size_t)i * dv + j] * dp[j];
                    dk_out[tk + i] += acc;
                }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += kv[i] * dp[j];
                /* forget: G becomes dL/dS_{t-1} */
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += G[(size_t)i * dv + j] * X[(size_t)i * dv + j];
                    dlog_alpha[tk + i] = acc;
                    const double ai = exp(lv[i]);
                    for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= ai;
                }
            }
        }
        memcpy(dS0 + state_off, G, sizeof(double) * DD);
        free(ckpt); free(prev); free(cur); free(X); free(G);
        free(pp); free(uu); free(du); free(dp); free(St);
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
