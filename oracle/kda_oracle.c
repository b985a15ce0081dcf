/*
 * kda_oracle.c -- plain fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * forward pass.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and
 * the bench's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, no chunking, no blocking, no
 * re-association):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = S_t^T q_t,
 *
 * per (sequence, head), with S in R^{dk x dv}, alpha_t = exp(log_alpha_t) in
 * (0,1)^{dk}, beta_t in (0,1).  Sources:
 *   - "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)" (GeekNews
 *     topic 31936), sections "선형 어텐션에서 Gated DeltaNet까지" (delta rule,
 *     scalar forget gate, Householder view) and "Kimi Delta Attention의 세밀한
 *     메모리 제어" (the scalar decay replaced by a channel-wise diagonal gate);
 *   - "From GPT-2 to Kimi K3, Explained" (seosoyoung digest), sections
 *     "DeltaNet -- 유한한 캐시의 덮어쓰기" (read the old value with the current
 *     key, subtract it from the new value, write the difference back) and
 *     "Kimi Linear (KDA) -- 채널별 세밀한 게이팅" (alpha becomes Diag(alpha)).
 *
 * The transition is applied in the order the product is written: first the
 * channel-wise decay Diag(alpha_t) on the key axis (the dk rows of S), then the
 * delta read r = S'^T k_t on the decayed state S', then the write
 * S = S' + beta_t k_t (v_t - r)^T, and the output is read after the write.
 *
 * RULE_ADDITIVE replaces the delta write by the plain additive write
 * S = Diag(alpha_t) S_{t-1} + k_t v_t^T (linear attention / GLA form).  It is
 * used only by the oracle's own closed-form checks.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_RULE_DELTA 0
#define KDA_ORACLE_RULE_ADDITIVE 1

/*
 * One (sequence, head) unit of length L.
 *   q, k, log_alpha : row t at q + t*sq (dk contiguous doubles), etc.
 *   v               : row t at v + t*sv (dv contiguous doubles)
 *   beta            : beta_t at beta[t*sb]
 *   S               : dk x dv row-major, in: initial state, out: final state
 *   o               : row t at o + t*so (dv doubles)
 *   r               : caller-provided scratch of dv doubles
 */
static void unit_recurrence(int64_t L, int dk, int dv,
                            const double* q, const double* k, const double* v,
                            const double* log_alpha, const double* beta,
                            int64_t sq, int64_t sk, int64_t sv, int64_t sa, int64_t sb,
                            double* S, double* o, int64_t so, int rule, double* r)
{
    for (int64_t t = 0; t < L; ++t) {
        const double* qt = q + t * sq;
        const double* kt = k + t * sk;
        const double* vt = v + t * sv;
        const double* at = log_alpha + t * sa;
        const double bt = beta[t * sb];
        double* ot = o + t * so;

        /* 1. S <- Diag(alpha_t) S: row c (key channel c) scaled by alpha_{t,c}. */
        for (int c = 0; c < dk; ++c) {
            const double alpha = exp(at[c]);
            double* row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] *= alpha;
        }

        if (rule == KDA_ORACLE_RULE_DELTA) {
            /* 2. read the value the decayed state returns for key k_t: r = S^T k_t */
            for (int j = 0; j < dv; ++j) r[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double kc = kt[c];
                const double* row = S + (int64_t)c * dv;
                for (int j = 0; j < dv; ++j) r[j] += row[j] * kc;
            }
            /* 3. write back the correction: S <- S + beta_t k_t (v_t - r)^T */
            for (int c = 0; c < dk; ++c) {
                const double w = bt * kt[c];
                double* row = S + (int64_t)c * dv;
                for (int j = 0; j < dv; ++j) row[j] += w * (vt[j] - r[j]);
            }
        } else {
            /* additive write: S <- S + k_t v_t^T */
            for (int c = 0; c < dk; ++c) {
                const double kc = kt[c];
                double* row = S + (int64_t)c * dv;
                for (int j = 0; j < dv; ++j) row[j] += kc * vt[j];
            }
        }

        /* 4. output after the write: o_t = S^T q_t */
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double qc = qt[c];
            const double* row = S + (int64_t)c * dv;
            for (int j = 0; j < dv; ++j) ot[j] += row[j] * qc;
        }
    }
}

/*
 * Packed variable-length batch.
 *   q, k, log_alpha : [T_total, H, dk]   v, o : [T_total, H, dv]   beta : [T_total, H]
 *   cu_seqlens      : [N+1] token offsets, cu_seqlens[0] = 0, non-decreasing
 *   S0              : [N, H, dk, dv] or NULL (zeros)
 *   S_final         : [N, H, dk, dv] (written; may not be NULL)
 *   nthreads        : OpenMP threads over the independent (sequence, head) units (<=0: default)
 * Returns 0 on success, -1 on an invalid argument, -2 on allocation failure.
 */
int kda_oracle_forward(const double* q, const double* k, const double* v,
                       const double* log_alpha, const double* beta,
                       const double* S0, const int64_t* cu_seqlens,
                       int64_t N, int64_t H, int dk, int dv,
                       double* o, double* S_final, int rule, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o || !S_final) return -1;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (rule != KDA_ORACLE_RULE_DELTA && rule != KDA_ORACLE_RULE_ADDITIVE) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;

    const int64_t units = N * H;
    const int64_t state_elems = (int64_t)dk * dv;
    int status = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* r = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!r) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t u = 0; u < units; ++u) {
            if (!r) continue;
            const int64_t n = u / H, h = u % H;
            const int64_t t0 = cu_seqlens[n];
            const int64_t L = cu_seqlens[n + 1] - t0;
            double* S = S_final + u * state_elems;
            if (S0)
                memcpy(S, S0 + u * state_elems, sizeof(double) * (size_t)state_elems);
            else
                memset(S, 0, sizeof(double) * (size_t)state_elems);
            unit_recurrence(L, dk, dv,
                            q + (t0 * H + h) * dk, k + (t0 * H + h) * dk, v + (t0 * H + h) * dv,
                            log_alpha + (t0 * H + h) * dk, beta + (t0 * H + h),
                            H * dk, H * dk, H * dv, H * dk, H,
                            S, o + (t0 * H + h) * dv, H * dv, rule, r);
        }
        free(r);
    }
    return status;
}

/*
 * One recurrent decode step for B sequences (one token each), state in place.
 *   q, k, log_alpha : [B, H, dk]  v, o : [B, H, dv]  beta : [B, H]  S : [B, H, dk, dv]
 * Identical to kda_oracle_forward with every sequence of length 1.
 */
int kda_oracle_decode(const double* q, const double* k, const double* v,
                      const double* log_alpha, const double* beta, double* S,
                      int64_t B, int64_t H, int dk, int dv, double* o, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return -1;
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    const int64_t units = B * H;
    const int64_t state_elems = (int64_t)dk * dv;
    int status = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* r = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!r) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = -2;
        }
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
        for (int64_t u = 0; u < units; ++u) {
            if (!r) continue;
            unit_recurrence(1, dk, dv, q + u * dk, k + u * dk, v + u * dv, log_alpha + u * dk,
                            beta + u, dk, dk, dv, dk, 1, S + u * state_elems, o + u * dv, dv,
                            KDA_ORACLE_RULE_DELTA, r);
        }
        free(r);
    }
    return status;
}

/* Number of OpenMP threads a default-threaded call would use (1 without OpenMP). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
