/*
 * KDA CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64, token-by-token CPU implementation of the Kimi Delta
 * Attention (KDA) sequence mixer.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load it; the CUDA library never links,
 * calls or includes anything from here, and nothing here comes from the CUDA
 * library.  There is no blocking, fusion or reordering: every token applies the
 * state edit exactly in the order the source states it.
 *
 * Source ("Kimi K3: Architecture, Training, and Million-Token Agentic RL",
 * brenchcc research note):
 *   - section 3.1, recurrence equation:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *       o_t = S_t^T q_t
 *     Diag(alpha_t) multiplies from the left, so it scales ROWS of S (one row
 *     per key channel).
 *   - section 3.2, the same step in edit order (the form coded below):
 *       Sbar_t = Diag(alpha_t) S_{t-1}
 *       vhat_t = Sbar_t^T k_t
 *       S_t    = Sbar_t + beta_t k_t (v_t - vhat_t)^T
 *       o_t    = S_t^T q_t            (read after write; no 1/sqrt(dk) scale)
 *   - section 3.3, lower-bounded gate equation (restated in "Kimi K3 Under the
 *     Hood", section "Sequence mixing: three KDA layers per global MLA layer"):
 *       g_t = g_min * sigmoid(exp(A) * z_t),  alpha_t = exp(g_t),  g_min = -5
 *     read per head h and key channel c as
 *       g[t,h,c] = -5 * sigmoid(exp(A[h,c]) * z[t,h,c]).
 *   - the same section and "Kimi K3 Under the Hood" section "Sequence mixing":
 *     the earlier Kimi Linear gate was an unbounded negative Softplus.  Read
 *     with the same pre-activation (gate kind 1):
 *       g[t,h,c] = -softplus(exp(A[h,c]) * z[t,h,c]),  softplus(x) = log(1 + e^x).
 *
 * Layouts (row-major, all fp64 on this side):
 *   q, k, z : [T, H, dk]     v, o : [T, H, dv]     beta : [T, H]
 *   A       : [H, dk]        states : [N or P, H, dk, dv]  (dv contiguous)
 *   cu_seqlens : [N+1] int32, cu_seqlens[0] = 0, non-decreasing.
 *
 * Parallelism: OpenMP over independent (sequence, head) pairs only; the
 * arithmetic of every pair is the sequential recurrence above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_GMIN (-5.0)
#define KDA_ORACLE_GATE_BOUNDED 0   /* g_min * sigmoid(exp(A) z) */
#define KDA_ORACLE_GATE_SOFTPLUS 1  /* -softplus(exp(A) z), unbounded below */

/* sigmoid(x) = 1 / (1 + exp(-x)).  For x -> -inf exp(-x) overflows to +inf and
 * the result is exactly 0; for x -> +inf it is exactly 1. */
static double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* softplus(x) = log(1 + e^x), written as max(x, 0) + log(1 + e^{-|x|}) so that
 * neither branch overflows. */
static double oracle_softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* Gate of one (token, head): g[c] = g_min * sigmoid(exp(A[c]) * z[c])
 * ("Kimi K3: Architecture, Training, and Million-Token Agentic RL", section 3.3
 * gate equation), or -softplus(exp(A[c]) * z[c]) for the unbounded kind. */
static void oracle_gate_row(const double *z, const double *A, int dk, double *g, int kind)
{
    for (int c = 0; c < dk; ++c)
        g[c] = kind == KDA_ORACLE_GATE_SOFTPLUS ? -oracle_softplus(exp(A[c]) * z[c])
                                                : KDA_ORACLE_GMIN * oracle_sigmoid(exp(A[c]) * z[c]);
}

/* One token of the recurrence on a dk x dv state, in the section 3.2 edit order.
 * S is updated in place; o (length dv) receives S_t^T q_t. */
static void oracle_token_step(double *S, const double *q, const double *k,
                              const double *v, const double *g, double beta,
                              int dk, int dv, double *vhat, double *o)
{
    /* Sbar = Diag(alpha) S: row c is scaled by alpha_c = exp(g_c). */
    for (int c = 0; c < dk; ++c) {
        const double alpha = exp(g[c]);
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= alpha;
    }
    /* vhat = Sbar^T k. */
    for (int j = 0; j < dv; ++j) vhat[j] = 0.0;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) vhat[j] += S[(size_t)c * dv + j] * k[c];
    /* S = Sbar + beta k (v - vhat)^T. */
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j)
            S[(size_t)c * dv + j] += beta * k[c] * (v[j] - vhat[j]);
    /* o = S^T q (after the write). */
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) o[j] += S[(size_t)c * dv + j] * q[c];
}

int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Gate for a whole [T, H, dk] tensor, of the given kind. */
void kda_oracle_gate_kind(const double *z, const double *A, int64_t T, int H, int dk,
                          double *g, int kind)
{
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            oracle_gate_row(z + ((size_t)t * H + h) * dk, A + (size_t)h * dk, dk,
                            g + ((size_t)t * H + h) * dk, kind);
}

void kda_oracle_gate(const double *z, const double *A, int64_t T, int H, int dk,
                     double *g)
{
    kda_oracle_gate_kind(z, A, T, H, dk, g, KDA_ORACLE_GATE_BOUNDED);
}

int kda_oracle_prefill_gate(const double *q, const double *k, const double *v,
                            const double *z, const double *A, const double *beta,
                            const int32_t *cu_seqlens, int num_seqs, int H, int dk,
                            int dv, const double *initial_state, double *o,
                            double *final_state, int every, double *checkpoints,
                            int nthreads, int kind);

int kda_oracle_prefill_ckpt(const double *q, const double *k, const double *v,
                            const double *z, const double *A, const double *beta,
                            const int32_t *cu_seqlens, int num_seqs, int H, int dk,
                            int dv, const double *initial_state, double *o,
                            double *final_state, int every, double *checkpoints,
                            int nthreads)
{
    return kda_oracle_prefill_gate(q, k, v, z, A, beta, cu_seqlens, num_seqs, H, dk, dv,
                                   initial_state, o, final_state, every, checkpoints, nthreads,
                                   KDA_ORACLE_GATE_BOUNDED);
}

/*
 * Prefill over packed variable-length sequences: for every sequence n and head
 * h, start from initial_state[n,h] (zeros when initial_state is NULL), run the
 * recurrence over tokens cu_seqlens[n] .. cu_seqlens[n+1]-1, write o for each
 * token and, when final_state is non-NULL, the state after the last token.
 * An empty sequence passes its initial state through unchanged.
 * nthreads <= 0 uses the OpenMP default.  Returns 0, or -1 on allocation failure.
 */
int kda_oracle_prefill(const double *q, const double *k, const double *v,
                       const double *z, const double *A, const double *beta,
                       const int32_t *cu_seqlens, int num_seqs, int H, int dk,
                       int dv, const double *initial_state, double *o,
                       double *final_state, int nthreads)
{
    return kda_oracle_prefill_ckpt(q, k, v, z, A, beta, cu_seqlens, num_seqs, H, dk, dv,
                                   initial_state, o, final_state, 0, NULL, nthreads);
}

/*
 * Prefill that also records state checkpoints for prefix caching ("Kimi K3
 * Under the Hood", section "Serving two incompatible cache types": KDA states
 * are kept at selected prefix-hash boundaries).  With every > 0, checkpoint j
 * (j = 1 .. L_n / every) of sequence n is the state after its first j * every
 * tokens, stored at row (sum_{m<n} L_m / every) + j - 1 of checkpoints
 * [count, H, dk, dv].
 */
int kda_oracle_prefill_gate(const double *q, const double *k, const double *v,
                            const double *z, const double *A, const double *beta,
                            const int32_t *cu_seqlens, int num_seqs, int H, int dk,
                            int dv, const double *initial_state, double *o,
                            double *final_state, int every, double *checkpoints,
                            int nthreads, int kind)
{
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t pairs = (int64_t)num_seqs * H;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *g = (double *)malloc(sizeof(double) * (size_t)dk);
        double *vhat = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!S || !g || !vhat) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t p = 0; p < pairs; ++p) {
                const int n = (int)(p / H), h = (int)(p % H);
                const size_t sidx = ((size_t)n * H + h) * (size_t)dk * dv;
                if (initial_state)
                    memcpy(S, initial_state + sidx, sizeof(double) * (size_t)dk * dv);
                else
                    memset(S, 0, sizeof(double) * (size_t)dk * dv);
                int64_t ck_base = 0;
                if (every > 0)
                    for (int m = 0; m < n; ++m)
                        ck_base += (cu_seqlens[m + 1] - cu_seqlens[m]) / every;
                for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                    const size_t th = (size_t)t * H + h;
                    oracle_gate_row(z + th * dk, A + (size_t)h * dk, dk, g, kind);
                    oracle_token_step(S, q + th * dk, k + th * dk, v + th * dv, g,
                                      beta[th], dk, dv, vhat, o + th * dv);
                    const int64_t done = t + 1 - cu_seqlens[n];
                    if (every > 0 && checkpoints && done % every == 0) {
                        const size_t row = (size_t)(ck_base + done / every - 1);
                        memcpy(checkpoints + (row * H + h) * (size_t)dk * dv, S,
                               sizeof(double) * (size_t)dk * dv);
                    }
                }
                if (final_state)
                    memcpy(final_state + sidx, S, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(S);
        free(g);
        free(vhat);
    }
    return failed ? -1 : 0;
}

/*
 * One decode step for a batch of B sequences, each carrying one new token:
 * state[slot[b], h] is advanced in place by the same token step and o[b,h] is
 * the read after the write.  slots == NULL means slot[b] = b.  Section 3.2 of
 * the same note gives the decode interface (x_t, S_{t-1}) -> (y_t, S_t).
 */
int kda_oracle_decode_gate(const double *q, const double *k, const double *v,
                           const double *z, const double *A, const double *beta,
                           int B, int H, int dk, int dv, double *state,
                           const int32_t *slots, double *o, int nthreads, int kind)
{
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t pairs = (int64_t)B * H;
#pragma omp parallel
    {
        double *g = (double *)malloc(sizeof(double) * (size_t)dk);
        double *vhat = (double *)malloc(sizeof(double) * (size_t)dv);
        if (!g || !vhat) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t p = 0; p < pairs; ++p) {
                const int b = (int)(p / H), h = (int)(p % H);
                const int slot = slots ? slots[b] : b;
                const size_t th = (size_t)b * H + h;
                double *S = state + ((size_t)slot * H + h) * (size_t)dk * dv;
                oracle_gate_row(z + th * dk, A + (size_t)h * dk, dk, g, kind);
                oracle_token_step(S, q + th * dk, k + th * dk, v + th * dv, g,
                                  beta[th], dk, dv, vhat, o + th * dv);
            }
        }
        free(g);
        free(vhat);
    }
    return failed ? -1 : 0;
}

int kda_oracle_decode(const double *q, const double *k, const double *v,
                      const double *z, const double *A, const double *beta,
                      int B, int H, int dk, int dv, double *state,
                      const int32_t *slots, double *o, int nthreads)
{
    return kda_oracle_decode_gate(q, k, v, z, A, beta, B, H, dk, dv, state, slots, o, nthreads,
                                  KDA_ORACLE_GATE_BOUNDED);
}
