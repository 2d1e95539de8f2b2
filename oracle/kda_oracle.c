/*
 * KDA forward oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, token-by-token CPU implementation of the Kimi Delta Attention
 * forward pass in fp64.  Only the tests, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load it.  It shares no code with the CUDA path.
 *
 * What it computes (FlashKDA pages: "refines Gated DeltaNet with finer
 * channel-wise gating", 7minutos.es section "Que es la atencion Kimi Delta";
 * operator inputs and flags from the same page, section "Debajo del capo", and
 * the chunk_kda call on github.zuobiaodaohang.com, section "作为 FLA 后端的用法"):
 *
 *   for each sequence s and head h, with S (K x V) = initial_state[s,h] or 0:
 *     for each token t of s:
 *       qh = q_t / sqrt(sum q_t^2 + eps)            (use_qk_l2norm_in_kernel)
 *       kh = k_t / sqrt(sum k_t^2 + eps)
 *       b  = 1 / (1 + exp(-beta_t))                 (use_beta_sigmoid_in_kernel)
 *       lam[c] = max(lb, -exp(A_log[h]) * softplus(g_t[c] + dt_bias[h,c]))
 *                                                   (use_gate_in_kernel, safe_gate,
 *                                                    lower_bound in [-5, 0])
 *       S[c,:] *= exp(lam[c])                       S' = Diag(alpha_t) S
 *       S += b * kh (v_t - S^T kh)^T                delta rule
 *       out_t = scale * S^T qh
 *     final_state[s,h] = S
 *
 * Readings where the pages are silent: the gate formula above (natural log,
 * softplus(x) = max(x,0) + log1p(exp(-|x|))), eps = 1e-6 inside the L2 norm,
 * dt_bias of shape [H,K], scale applied to the output, token t's own decay
 * applied before its write, bf16 inputs promoted exactly to fp64.
 *
 * Layouts (row-major, contiguous): q,k,g [B,T,H,K]; v,out [B,T,H,V];
 * beta [B,T,H]; A_log [H]; dt_bias [H,K]; states [N,H,K,V] with S[k][v].
 * With cu_seqlens (B must be 1), sequence s spans tokens [cu[s], cu[s+1]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_STATE_NONE 0
#define ORACLE_STATE_F32 1
#define ORACLE_STATE_BF16 2
#define ORACLE_STATE_F64 3 /* test-only: exact chaining of final -> initial */

static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double softplus(double x)
{
    return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

/* One token of the recurrence on S (K x V, row k at S + k*V), given
 * post-activation values.  out_t may be NULL. */
static void recurrence_step(int64_t K, int64_t V, double *S, const double *qh,
                            const double *kh, const double *v, double b,
                            const double *lam, double scale, double *out_t,
                            double *work /* V doubles */)
{
    for (int64_t c = 0; c < K; ++c) {
        double a = exp(lam[c]);
        for (int64_t j = 0; j < V; ++j)
            S[c * V + j] *= a;
    }
    /* work = v - S^T kh (the prediction error of the delta rule) */
    for (int64_t j = 0; j < V; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < K; ++c)
            acc += S[c * V + j] * kh[c];
        work[j] = v[j] - acc;
    }
    for (int64_t c = 0; c < K; ++c) {
        double f = b * kh[c];
        for (int64_t j = 0; j < V; ++j)
            S[c * V + j] += f * work[j];
    }
    if (out_t) {
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < K; ++c)
                acc += S[c * V + j] * qh[c];
            out_t[j] = scale * acc;
        }
    }
}

/*
 * Recurrence core on post-activation inputs for ONE (sequence, head):
 * qh, kh, lam [T][K]; v [T][V]; b [T]; S0 [K][V] or NULL (zeros).
 * Writes out [T][V] (may be NULL) and S_final [K][V] (may be NULL).
 * Used by the tests to feed exact special cases (beta = 0 or 1, alpha = 1).
 */
int kda_oracle_core(int64_t T, int64_t K, int64_t V, const double *qh, const double *kh,
                    const double *v, const double *b, const double *lam, double scale,
                    const double *S0, double *out, double *S_final)
{
    if (T < 0 || K < 1 || V < 1)
        return -1;
    double *S = (double *)calloc((size_t)(K * V), sizeof(double));
    double *work = (double *)malloc((size_t)V * sizeof(double));
    if (!S || !work) {
        free(S);
        free(work);
        return -2;
    }
    if (S0)
        memcpy(S, S0, (size_t)(K * V) * sizeof(double));
    for (int64_t t = 0; t < T; ++t)
        recurrence_step(K, V, S, qh + t * K, kh + t * K, v + t * V, b[t], lam + t * K,
                        scale, out ? out + t * V : NULL, work);
    if (S_final)
        memcpy(S_final, S, (size_t)(K * V) * sizeof(double));
    free(S);
    free(work);
    return 0;
}

/*
 * Full forward pass from the raw operator inputs (bf16 given as uint16 bit
 * patterns, promoted exactly to fp64).  init_dtype: ORACLE_STATE_NONE / F32 /
 * BF16 / F64.  final_state [N,H,K,V] fp64 (may be NULL); out [B,T,H,V] fp64 (may be
 * NULL).  cu_seqlens NULL means B sequences of length T.  eps is the L2-norm
 * epsilon (1e-6 everywhere except the tests that probe it).
 * Only the (sequence, head) pairs with mask[s*H + h] != 0 are computed when
 * mask is not NULL (the others are left untouched); this lets a test or the
 * CPU baseline time a bounded sample.  Returns 0 on success.
 */
int kda_oracle_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *g,
                   const uint16_t *beta, double scale, const float *A_log, const float *dt_bias,
                   double lower_bound, const void *initial_state, int init_dtype,
                   double *final_state, const int64_t *cu_seqlens, int64_t num_seqs,
                   double *out, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                   double eps, const uint8_t *mask)
{
    if (B < 1 || T < 0 || H < 1 || K < 1 || V < 1)
        return -1;
    if (cu_seqlens && (B != 1 || num_seqs < 1))
        return -1;
    const int64_t N = cu_seqlens ? num_seqs : B;
    const int64_t units = N * H;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t s = u / H, h = u % H;
        if (mask && !mask[u])
            continue;
        int64_t tok0, len;
        if (cu_seqlens) {
            tok0 = cu_seqlens[s];
            len = cu_seqlens[s + 1] - cu_seqlens[s];
        } else {
            tok0 = s * T;
            len = T;
        }
        double *S = (double *)calloc((size_t)(K * V), sizeof(double));
        double *qh = (double *)malloc((size_t)K * sizeof(double));
        double *kh = (double *)malloc((size_t)K * sizeof(double));
        double *vv = (double *)malloc((size_t)V * sizeof(double));
        double *lam = (double *)malloc((size_t)K * sizeof(double));
        double *work = (double *)malloc((size_t)V * sizeof(double));
        if (!S || !qh || !kh || !vv || !lam || !work) {
#pragma omp atomic write
            err = -2;
            free(S); free(qh); free(kh); free(vv); free(lam); free(work);
            continue;
        }
        const size_t state_off = (size_t)((s * H + h) * K * V);
        if (initial_state && init_dtype == ORACLE_STATE_F32) {
            const float *src = (const float *)initial_state + state_off;
            for (int64_t i = 0; i < K * V; ++i)
                S[i] = (double)src[i];
        } else if (initial_state && init_dtype == ORACLE_STATE_F64) {
            memcpy(S, (const double *)initial_state + state_off, (size_t)(K * V) * sizeof(double));
        } else if (initial_state && init_dtype == ORACLE_STATE_BF16) {
            const uint16_t *src = (const uint16_t *)initial_state + state_off;
            for (int64_t i = 0; i < K * V; ++i)
                S[i] = bf16_to_f64(src[i]);
        }
        const double decay_scale = exp((double)A_log[h]);
        for (int64_t t = 0; t < len; ++t) {
            const int64_t tok = tok0 + t; /* flat token index b*T + t or packed index */
            const size_t qk_off = (size_t)((tok * H + h) * K);
            const size_t v_off = (size_t)((tok * H + h) * V);
            double sq = 0.0, sk = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                double a = bf16_to_f64(q[qk_off + c]);
                double bb = bf16_to_f64(k[qk_off + c]);
                sq += a * a;
                sk += bb * bb;
            }
            const double rq = 1.0 / sqrt(sq + eps), rk = 1.0 / sqrt(sk + eps);
            for (int64_t c = 0; c < K; ++c) {
                qh[c] = bf16_to_f64(q[qk_off + c]) * rq;
                kh[c] = bf16_to_f64(k[qk_off + c]) * rk;
                const double x = bf16_to_f64(g[qk_off + c]) + (double)dt_bias[h * K + c];
                lam[c] = fmax(lower_bound, -decay_scale * softplus(x));
            }
            for (int64_t j = 0; j < V; ++j)
                vv[j] = bf16_to_f64(v[v_off + j]);
            const double b = 1.0 / (1.0 + exp(-bf16_to_f64(beta[tok * H + h])));
            recurrence_step(K, V, S, qh, kh, vv, b, lam, scale, out ? out + v_off : NULL, work);
        }
        if (final_state)
            memcpy(final_state + state_off, S, (size_t)(K * V) * sizeof(double));
        free(S); free(qh); free(kh); free(vv); free(lam); free(work);
    }
    return err;
}

/* Threads the OpenMP runtime will use (reported as the CPU baseline's cores). */
int kda_oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
