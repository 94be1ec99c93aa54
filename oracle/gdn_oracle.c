/*
 * gdn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU implementation of the Gated DeltaNet recurrence,
 * run token by token.  It is the oracle that the CUDA path is checked
 * against; nothing in the product path may link or call it.  It shares no
 * code, header or constant with the CUDA library.
 *
 * The recurrence (Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *     alpha_t = exp(g_t)      (the kernel receives g and exponentiates it)
 *
 * S_t is dk x dv, row index = key channel.  alpha_t is either one value per
 * (token, head) ("scalar" gate, original GDN) or one value per key channel
 * (per-channel gate, GDN-2 / KDA; "Gated DeltaNet" entity trail, finding of
 * 2026-07-29: the gate promoted to per-key-channel).
 *
 * The update is carried out in delta-rule form, where the state is corrected
 * by the prediction error of the current key (the same finding describes the
 * rule this way): with S' = Diag(alpha_t) S_{t-1},
 *     e_t = v_t - S'^T k_t,    S_t = S' + beta_t k_t e_t^T,
 * which expands to exactly the formula above:
 *     S' + beta k (v - S'^T k)^T = S' - beta k k^T S' + beta k v^T.
 * The output uses the UPDATED state S_t (o_t = S_t^T q_t).  No 1/sqrt(dk)
 * query scale is applied (the formula has none).
 *
 * Layouts (row-major, contiguous, fp64):
 *   q, k : [B, T, H, dk]      v, out : [B, T, H, dv]
 *   g    : [B, T, H] (scalar gate) or [B, T, H, dk] (per-channel gate)
 *   beta : [B, T, H]
 *   s0, sT : [B, H, dk, dv]   (s0 may be NULL = zero initial state;
 *                              sT may be NULL = final state not returned)
 *
 * Parallelism: independent (b, h) pairs run on separate OpenMP threads; the
 * arithmetic inside one pair is strictly sequential.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void run_pair(const double* q, const double* k, const double* v,
                     const double* g, const double* beta, const double* s0,
                     double* out, double* sT, long b, long h,
                     long B, long T, long H, long dk, long dv, int per_channel,
                     double* S, double* alpha, double* e)
{
    (void)B;
    if (s0) {
        memcpy(S, s0 + ((b * H + h) * dk) * dv, sizeof(double) * dk * dv);
    } else {
        memset(S, 0, sizeof(double) * dk * dv);
    }
    for (long t = 0; t < T; ++t) {
        const long tok = (b * T + t) * H + h;       /* (b, t, h) flat index */
        const double* qt = q + tok * dk;
        const double* kt = k + tok * dk;
        const double* vt = v + tok * dv;
        const double bt = beta[tok];
        double* ot = out + tok * dv;

        /* alpha_t = exp(g_t): one value per key channel (row of S). */
        for (long i = 0; i < dk; ++i) {
            alpha[i] = per_channel ? exp(g[tok * dk + i]) : exp(g[tok]);
        }
        /* S' = Diag(alpha_t) S_{t-1}: decay applied first, row by row. */
        for (long i = 0; i < dk; ++i) {
            for (long j = 0; j < dv; ++j) S[i * dv + j] *= alpha[i];
        }
        /* e = v_t - S'^T k_t */
        for (long j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (long i = 0; i < dk; ++i) acc += S[i * dv + j] * kt[i];
            e[j] = vt[j] - acc;
        }
        /* S_t = S' + beta_t k_t e^T */
        for (long i = 0; i < dk; ++i) {
            const double bk = bt * kt[i];
            for (long j = 0; j < dv; ++j) S[i * dv + j] += bk * e[j];
        }
        /* o_t = S_t^T q_t */
        for (long j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (long i = 0; i < dk; ++i) acc += S[i * dv + j] * qt[i];
            ot[j] = acc;
        }
    }
    if (sT) {
        memcpy(sT + ((b * H + h) * dk) * dv, S, sizeof(double) * dk * dv);
    }
}

/*
 * Runs the recurrence over T tokens for the (b, h) pairs listed in `sel`
 * (flat index b*H + h; NULL = every pair).  Rows of `out` / `sT` that belong
 * to unselected pairs are left untouched.  Returns 0, or -1 on a bad
 * argument or an allocation failure.
 */
int gdn_oracle_run(const double* q, const double* k, const double* v,
                   const double* g, const double* beta, const double* s0,
                   double* out, double* sT,
                   long B, long T, long H, long dk, long dv, int per_channel,
                   const long* sel, long n_sel, int n_threads)
{
    if (!q || !k || !v || !g || !beta || !out) return -1;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    const long n_pairs = sel ? n_sel : B * H;
    int failed = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * dk * dv);
        double* alpha = (double*)malloc(sizeof(double) * dk);
        double* e = (double*)malloc(sizeof(double) * dv);
        const int have_buffers = (S && alpha && e);
        if (!have_buffers) {
#pragma omp atomic write
            failed = 1;
        }
        /* Every thread reaches the work-sharing loop; one without buffers
         * skips its share (the call then reports failure). */
#pragma omp for schedule(dynamic, 1)
        for (long p = 0; p < n_pairs; ++p) {
            const long bh = sel ? sel[p] : p;
            if (!have_buffers || bh < 0 || bh >= B * H) {
#pragma omp atomic write
                failed = 1;
                continue;
            }
            run_pair(q, k, v, g, beta, s0, out, sT, bh / H, bh % H,
                     B, T, H, dk, dv, per_channel, S, alpha, e);
        }
        free(S);
        free(alpha);
        free(e);
    }
    return failed ? -1 : 0;
}
