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

/*
 * Backward pass (reverse-mode differentiation of the same per-token step).
 *
 * Given the upstream gradients dout [tokens, H, dv] of the outputs and dhT
 * [N, H, dk, dv] of the final states (NULL: zero), it returns the gradients
 * of the loss sum(dout * out) + sum(dhT * hT) with respect to every input:
 * dq, dk [tokens, H, dk], dv [tokens, H, dv], dlog_alpha [tokens, H, dk],
 * dbeta [tokens, H] and dh0 [N, H, dk, dv] (dh0 may be NULL).
 *
 * Walking the tokens backwards with G = dL/dS_t (the state after token t):
 *   dq_t   = scale S_t do_t                  (o_t = scale S_t^T q_t)
 *   G     += scale q_t do_t^T
 *   de     = G^T k_t,   dk_t += G e          (S_t = S~ + k_t e^T)
 *   dbeta  = de . (v_t - vhat),  dv_t = beta de,  dvhat = -beta de
 *   G     += k_t dvhat^T,  dk_t += S~ dvhat  (vhat = S~^T k_t)
 *   dlog_alpha_i = sum_j G_ij S~_ij,  G <- Diag(alpha) G   (S~ = Diag(alpha) S_{t-1})
 * and dh0 is G after the first token.  The states S_{t-1} are recomputed: the
 * forward keeps the state at every 64th token and each 64-token block is
 * replayed (all its states kept) before it is walked backwards.
 */
#define KDA_ORACLE_BLOCK 64

/* One token of the forward step from S_prev into S_next (both dk*dv); also
 * returns S~ (decayed state), vhat and e. */
static void kda_token_fwd(const double* qt, const double* kt, const double* vt,
                          const double* gt, double bt, const double* S_prev, double* S_dec,
                          double* S_next, double* vhat, double* e, int64_t dk, int64_t dv)
{
    (void)qt;
    for (int64_t i = 0; i < dk; ++i) {
        const double a = exp(gt[i]);
        for (int64_t j = 0; j < dv; ++j) S_dec[i * dv + j] = a * S_prev[i * dv + j];
    }
    for (int64_t j = 0; j < dv; ++j) vhat[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) vhat[j] += S_dec[i * dv + j] * kt[i];
    for (int64_t j = 0; j < dv; ++j) e[j] = bt * (vt[j] - vhat[j]);
    for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S_next[i * dv + j] = S_dec[i * dv + j] + kt[i] * e[j];
}

int kda_oracle_bwd(const double* q, const double* k, const double* v,
                   const double* log_alpha, const double* beta, const double* h0,
                   const double* dout, const double* dhT,
                   double* dq, double* dk_out, double* dv_out, double* dlog_alpha,
                   double* dbeta, double* dh0,
                   const int64_t* cu_seqlens, int64_t N, int64_t H,
                   int64_t dk, int64_t dv, double scale)
{
    for (int64_t n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int64_t SS = dk * dv;
    int bad = 0;
    #pragma omp parallel for schedule(dynamic, 1) reduction(|:bad)
    for (int64_t p = 0; p < N * H; ++p) {
        const int64_t n = p / H, h = p % H;
        const int64_t t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1], L = t1 - t0;
        const int64_t nb = (L + KDA_ORACLE_BLOCK - 1) / KDA_ORACLE_BLOCK;
        /* checkpoints [nb], block states [BLOCK + 1], G, S~, scratch vectors */
        double* ck = (double*)malloc(sizeof(double) * (size_t)((nb > 0 ? nb : 1) * SS));
        double* blk = (double*)malloc(sizeof(double) * (size_t)((KDA_ORACLE_BLOCK + 1) * SS));
        double* G = (double*)malloc(sizeof(double) * (size_t)(2 * SS + 4 * dv));
        if (!ck || !blk || !G) { free(ck); free(blk); free(G); bad |= 1; continue; }
        double* Sdec = G + SS;
        double* vhat = Sdec + SS;
        double* e = vhat + dv;
        double* de = e + dv;
        double* dvhat = de + dv;
        double* S = blk;                            /* running state for the checkpoint pass */
        if (h0) memcpy(S, h0 + p * SS, sizeof(double) * (size_t)SS);
        else memset(S, 0, sizeof(double) * (size_t)SS);
        for (int64_t b = 0; b < nb; ++b) {
            memcpy(ck + b * SS, S, sizeof(double) * (size_t)SS);
            const int64_t ta = t0 + b * KDA_ORACLE_BLOCK;
            const int64_t tb = (ta + KDA_ORACLE_BLOCK < t1) ? ta + KDA_ORACLE_BLOCK : t1;
            for (int64_t t = ta; t < tb; ++t) {
                kda_token_fwd(q + (t * H + h) * dk, k + (t * H + h) * dk, v + (t * H + h) * dv,
                              log_alpha + (t * H + h) * dk, beta[t * H + h], S, Sdec,
                              blk + SS, vhat, e, dk, dv);
                memcpy(S, blk + SS, sizeof(double) * (size_t)SS);
            }
        }
        if (dhT) memcpy(G, dhT + p * SS, sizeof(double) * (size_t)SS);
        else memset(G, 0, sizeof(double) * (size_t)SS);
        for (int64_t b = nb - 1; b >= 0; --b) {
            const int64_t ta = t0 + b * KDA_ORACLE_BLOCK;
            const int64_t tb = (ta + KDA_ORACLE_BLOCK < t1) ? ta + KDA_ORACLE_BLOCK : t1;
            memcpy(blk, ck + b * SS, sizeof(double) * (size_t)SS);
            for (int64_t t = ta; t < tb; ++t)         /* blk[i] = state before token ta + i */
                kda_token_fwd(q + (t * H + h) * dk, k + (t * H + h) * dk, v + (t * H + h) * dv,
                              log_alpha + (t * H + h) * dk, beta[t * H + h], blk + (t - ta) * SS,
                              Sdec, blk + (t - ta + 1) * SS, vhat, e, dk, dv);
            for (int64_t t = tb - 1; t >= ta; --t) {
                const double* qt = q + (t * H + h) * dk;
                const double* kt = k + (t * H + h) * dk;
                const double* vt = v + (t * H + h) * dv;
                const double* gt = log_alpha + (t * H + h) * dk;
                const double bt = beta[t * H + h];
                const double* dot = dout + (t * H + h) * dv;
                const double* Sprev = blk + (t - ta) * SS;
                const double* St = blk + (t - ta + 1) * SS;
                double* dqt = dq + (t * H + h) * dk;
                double* dkt = dk_out + (t * H + h) * dk;
                double* dvt = dv_out + (t * H + h) * dv;
                double* dgt = dlog_alpha + (t * H + h) * dk;
                double* Sn = Sdec;                  /* recompute S~, vhat, e of token t */
                for (int64_t i = 0; i < dk; ++i) {
                    const double a = exp(gt[i]);
                    for (int64_t j = 0; j < dv; ++j) Sn[i * dv + j] = a * Sprev[i * dv + j];
                }
                for (int64_t j = 0; j < dv; ++j) vhat[j] = 0.0;
                for (int64_t i = 0; i < dk; ++i)
                    for (int64_t j = 0; j < dv; ++j) vhat[j] += Sn[i * dv + j] * kt[i];
                for (int64_t j = 0; j < dv; ++j) e[j] = bt * (vt[j] - vhat[j]);
                /* read: dq = scale S_t do; G += scale q do^T */
                for (int64_t i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < dv; ++j) acc += St[i * dv + j] * dot[j];
                    dqt[i] = scale * acc;
                    for (int64_t j = 0; j < dv; ++j) G[i * dv + j] += scale * qt[i] * dot[j];
                }
                /* write: de = G^T k, dk = G e */
                for (int64_t j = 0; j < dv; ++j) de[j] = 0.0;
                for (int64_t i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < dv; ++j) {
                        de[j] += G[i * dv + j] * kt[i];
                        acc += G[i * dv + j] * e[j];
                    }
                    dkt[i] = acc;
                }
                /* error: dbeta, dv, dvhat */
                double db = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    db += de[j] * (vt[j] - vhat[j]);
                    dvt[j] = bt * de[j];
                    dvhat[j] = -bt * de[j];
                }
                dbeta[t * H + h] = db;
                /* predict: G += k dvhat^T, dk += S~ dvhat */
                for (int64_t i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < dv; ++j) {
                        G[i * dv + j] += kt[i] * dvhat[j];
                        acc += Sn[i * dv + j] * dvhat[j];
                    }
                    dkt[i] += acc;
                }
                /* decay: dlog_alpha_i = sum_j G_ij S~_ij; G <- Diag(alpha) G */
                for (int64_t i = 0; i < dk; ++i) {
                    const double a = exp(gt[i]);
                    double acc = 0.0;
                    for (int64_t j = 0; j < dv; ++j) {
                        acc += G[i * dv + j] * Sn[i * dv + j];
                        G[i * dv + j] *= a;
                    }
                    dgt[i] = acc;
                }
            }
        }
        if (dh0) memcpy(dh0 + p * SS, G, sizeof(double) * (size_t)SS);
        free(ck);
        free(blk);
        free(G);
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
