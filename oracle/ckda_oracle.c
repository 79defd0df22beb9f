/*
 * CKDA recurrence, fp64, one plain sequential loop per (batch, head).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the correctness oracle for the CUDA
 * library; only the test suite, the package's smoke check and the bench's CPU
 * baseline load it. It shares no code, header or constant with the CUDA side.
 *
 * What it computes (Complex KDA: Understanding and Enhancing the Expressivity of
 * Kimi Delta Attention; blog post "One update, one quarter-turn", section
 * "The mirror", update rule S' = (I - b k k^T) Diag(a) S + b k v^T, and section
 * "How it works: the spectrum argument", transition A = (I - b k k^T) Diag(a)):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                      (read after the update; no q scale)
 *
 * written in the algebraically identical delta form
 *
 *     S <- Diag(alpha_t) S;  u = beta_t (v_t - S^T k_t);  S <- S + k_t u^T;
 *     o_t = S^T q_t.
 *
 * The ranges alpha in [-1,1]^dk and beta in [0,2] (ai.info summary, "What This
 * Paper Is About") and ||k|| = 1 (same page, "Key Contributions", Theorem 1)
 * are the caller's business: nothing is clamped or renormalised here.
 *
 * Layouts (row-major, contiguous):
 *   q, k, alpha : [B, T, H, dk]     v, o : [B, T, H, dv]     beta : [B, T, H]
 *   S0, ST      : [B, H, dk, dv]    (S0 == NULL: zero state; ST == NULL: not written)
 */
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int ckda_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void ckda_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Returns 0 on success, 1 on a bad size, 2 on allocation failure. */
int ckda_oracle_fwd(const double* q, const double* k, const double* v,
                    const double* alpha, const double* beta, const double* S0,
                    double* o, double* ST,
                    long B, long T, long H, long dk, long dv) {
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1) return 1;
    long nseq = B * H;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (long bh = 0; bh < nseq; ++bh) {
        long b = bh / H, h = bh % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)(dk * dv));
        double* u = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!S || !u) { free(S); free(u); failed |= 1; continue; }
        if (S0) memcpy(S, S0 + bh * dk * dv, sizeof(double) * (size_t)(dk * dv));
        else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
        for (long t = 0; t < T; ++t) {
            long tok = (b * T + t) * H + h;           /* token-head index */
            const double* qt = q + tok * dk;
            const double* kt = k + tok * dk;
            const double* vt = v + tok * dv;
            const double* at = alpha + tok * dk;
            double bt = beta[tok];
            double* ot = o + tok * dv;
            /* S <- Diag(alpha_t) S */
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) S[i * dv + j] *= at[i];
            /* u = beta_t (v_t - S^T k_t) */
            for (long j = 0; j < dv; ++j) u[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) u[j] += S[i * dv + j] * kt[i];
            for (long j = 0; j < dv; ++j) u[j] = bt * (vt[j] - u[j]);
            /* S <- S + k_t u^T */
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * u[j];
            /* o_t = S_t^T q_t */
            for (long j = 0; j < dv; ++j) ot[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];
        }
        if (ST) memcpy(ST + bh * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
        free(S);
        free(u);
    }
    return failed ? 2 : 0;
}
