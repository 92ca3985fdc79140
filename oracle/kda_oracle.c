/*
 * KDA oracle: plain, slow, fp64 CPU implementation of the Kimi Delta Attention
 * recurrence.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark call this file; the product path never does.
 * It shares no code with the CUDA library.
 *
 * What it computes ("Kimi Delta Attention: la atencion lineal detras de Kimi K2
 * y Qwen3", section "Como funciona Kimi Delta Attention paso a paso", the
 * per-token step function and the flowchart that follows it):
 *
 *   for each token t of a sequence, with alpha_t = exp(log_alpha_t):
 *     S~   = Diag(alpha_t) S            decay every key channel of the state
 *     vhat = S~^T k_t                   what the decayed state recalls for k_t
 *     e    = beta_t (v_t - vhat)        beta-scaled prediction error
 *     S    = S~ + k_t e^T               write the error back along k_t
 *     o_t  = scale * S^T q_t            read with the query after the write
 *
 * The page stores the state as (d_v, d_k) and reads o = S q; here S is
 * (d_k, d_v) with d_v contiguous and o = S^T q, which is the same arithmetic.
 * The key-axis decay follows the page's per-channel gate Diag(alpha_t), which
 * multiplies the key channels of the state.  `scale` is applied once, to q, at
 * the read (the page divides q by sqrt(d_k) there).
 *
 * Layout: q,k [tokens, H, dk]; v [tokens, H, dv]; log_alpha [tokens, H, dk];
 * beta [tokens, H]; state h0/hT [N, H, dk, dv]; out [tokens, H, dv]; all fp64,
 * contiguous.  Sequence n covers tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.
 * A fixed-length batch [B, T, ...] is the packed case with cu_seqlens = {0, T, 2T, ...}.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One (sequence, head) pair, token by token.  S is dk*dv scratch owned by the caller. */
static void kda_pair(const double* q, const double* k, const double* v,
                     const double* log_alpha, const double* beta,
                     double* out, double* S, double* vhat,
                     int64_t t0, int64_t t1, int64_t h, int64_t H,
                     int64_t dk, int64_t dv, double scale)
{
    for (int64_t t = t0; t < t1; ++t) {
        const double* kt = k + (t * H + h) * dk;
        const double* qt = q + (t * H + h) * dk;
        const double* vt = v + (t * H + h) * dv;
        const double* gt = log_alpha + (t * H + h) * dk;
        const double bt = beta[t * H + h];
        /* decay: row i of S (key channel i) scales by alpha_i */
        for (int64_t i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
        /* predict: vhat = S~^T k */
        for (int64_t j = 0; j < dv; ++j) vhat[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) vhat[j] += S[i * dv + j] * kt[i];
        /* error and write: S += k (beta (v - vhat))^T */
        for (int64_t j = 0; j < dv; ++j) vhat[j] = bt * (vt[j] - vhat[j]);
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * vhat[j];
        /* read: o = scale * S^T q */
        double* ot = out + (t * H + h) * dv;
        for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            for (int64_t j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * (scale * qt[i]);
    }
}

/*
 * Full forward over N packed sequences and H heads.  h0 may be NULL (zero
 * initial state); hT may be NULL (final state not returned).  Returns 0, or -1
 * on inconsistent cu_seqlens.
 */
int kda_oracle_fwd(const double* q, const double* k, const double* v,
                   const double* log_alpha, const double* beta,
                   const double* h0, double* out, double* hT,
                   const int64_t* cu_seqlens, int64_t N, int64_t H,
                   int64_t dk, int64_t dv, double scale)
{
    for (int64_t n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    int bad = 0;
    #pragma omp parallel for schedule(dynamic, 1) reduction(|:bad)
    for (int64_t p = 0; p < N * H; ++p) {
        const int64_t n = p / H, h = p % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)(dk * dv + dv));
        if (!S) { bad |= 1; continue; }
        double* vhat = S + dk * dv;
        if (h0) memcpy(S, h0 + p * dk * dv, sizeof(double) * (size_t)(dk * dv));
        else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
        kda_pair(q, k, v, log_alpha, beta, out, S, vhat,
                 cu_seqlens[n], cu_seqlens[n + 1], h, H, dk, dv, scale);
        if (hT) memcpy(hT + p * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
        free(S);
    }
    return bad ? -2 : 0;
}

/*
 * One decode step for N independent sequences: the same per-token update with
 * one token per sequence, state [N, H, dk, dv] updated in place.
 */
int kda_oracle_step(const double* q, const double* k, const double* v,
                    const double* log_alpha, const double* beta,
                    double* state, double* out,
                    int64_t N, int64_t H, int64_t dk, int64_t dv, double scale)
{
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t p = 0; p < N * H; ++p) {
        double* vhat = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!vhat) { bad |= 1; continue; }
        /* token index p in a [N*H] "packed" view with one head per slot */
        kda_pair(q + p * dk, k + p * dk, v + p * dv, log_alpha + p * dk,
                 beta + p, out + p * dv, state + p * dk * dv, vhat,
                 0, 1, 0, 1, dk, dv, scale);
        free(vhat);
    }
    return bad ? -2 : 0;
}

/* Number of OpenMP threads the oracle will use (reported with CPU timings). */
int kda_oracle_threads(void)
{
    int n = 1;
    #pragma omp parallel
    {
        #pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
