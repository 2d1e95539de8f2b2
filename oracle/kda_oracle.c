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

/* ------------------------------------------------------------------------------
 * Raw fp64 inputs: forward twin and backward (reverse mode) of the same operator.
 *
 * The twin takes q, k, v, g, beta as fp64 values (not bf16 bit patterns) so that
 * the tests can take finite differences of it; on bf16-exact inputs it performs
 * the same operations as kda_oracle_fwd.  The backward differentiates
 *   L = sum_t <dO_t, out_t> + <dS_final, S_final>
 * with respect to q, k, v, g, beta, A_log, dt_bias and the initial state, token
 * by token in reverse, re-running the recurrence forward from checkpoints taken
 * every ORACLE_CKPT tokens to obtain the state before each token.
 *
 * Gradient of the gate clamp lam = max(lb, z), z = -exp(A_log) softplus(x): the
 * gradient flows through z where z >= lb and is zero where z < lb.
 * ---------------------------------------------------------------------------- */

#define ORACLE_CKPT 64

typedef struct {
    int64_t K, V;
    double *qh, *kh, *lam, *vv; /* activations of one token */
    double rq, rk, b;
    double *x, *z;              /* gate pre-activation x = g + dt_bias and z */
} token_act;

static void sequence_span(int64_t s, const int64_t *cu_seqlens, int64_t T, int64_t *tok0,
                          int64_t *len)
{
    if (cu_seqlens) {
        *tok0 = cu_seqlens[s];
        *len = cu_seqlens[s + 1] - cu_seqlens[s];
    } else {
        *tok0 = s * T;
        *len = T;
    }
}

/* Activations of token `tok` of head h from raw fp64 inputs. */
static void activate_f64(token_act *a, const double *q, const double *k, const double *v,
                         const double *g, const double *beta, const double *A_log,
                         const double *dt_bias, double lower_bound, double eps, int64_t tok,
                         int64_t h, int64_t H)
{
    const int64_t K = a->K, V = a->V;
    const double *qt = q + (tok * H + h) * K, *kt = k + (tok * H + h) * K;
    const double *gt = g + (tok * H + h) * K;
    double sq = 0.0, sk = 0.0;
    for (int64_t c = 0; c < K; ++c) {
        sq += qt[c] * qt[c];
        sk += kt[c] * kt[c];
    }
    a->rq = 1.0 / sqrt(sq + eps);
    a->rk = 1.0 / sqrt(sk + eps);
    const double decay_scale = exp(A_log[h]);
    for (int64_t c = 0; c < K; ++c) {
        a->qh[c] = qt[c] * a->rq;
        a->kh[c] = kt[c] * a->rk;
        a->x[c] = gt[c] + dt_bias[h * K + c];
        a->z[c] = -decay_scale * softplus(a->x[c]);
        a->lam[c] = fmax(lower_bound, a->z[c]);
    }
    for (int64_t j = 0; j < V; ++j)
        a->vv[j] = v[(tok * H + h) * V + j];
    a->b = 1.0 / (1.0 + exp(-beta[tok * H + h]));
}

static int act_alloc(token_act *a, int64_t K, int64_t V)
{
    a->K = K;
    a->V = V;
    a->qh = (double *)malloc((size_t)K * sizeof(double));
    a->kh = (double *)malloc((size_t)K * sizeof(double));
    a->lam = (double *)malloc((size_t)K * sizeof(double));
    a->x = (double *)malloc((size_t)K * sizeof(double));
    a->z = (double *)malloc((size_t)K * sizeof(double));
    a->vv = (double *)malloc((size_t)V * sizeof(double));
    return (a->qh && a->kh && a->lam && a->x && a->z && a->vv) ? 0 : -2;
}

static void act_free(token_act *a)
{
    free(a->qh); free(a->kh); free(a->lam); free(a->x); free(a->z); free(a->vv);
}

/* Forward on raw fp64 inputs; S0 [N,H,K,V] fp64 or NULL.  out / final_state may be NULL. */
int kda_oracle_fwd_f64(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, double scale, const double *A_log,
                       const double *dt_bias, double lower_bound, const double *S0,
                       double *final_state, const int64_t *cu_seqlens, int64_t num_seqs,
                       double *out, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                       double eps)
{
    if (B < 1 || T < 0 || H < 1 || K < 1 || V < 1)
        return -1;
    if (cu_seqlens && (B != 1 || num_seqs < 1))
        return -1;
    const int64_t N = cu_seqlens ? num_seqs : B;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < N * H; ++u) {
        const int64_t s = u / H, h = u % H;
        int64_t tok0, len;
        sequence_span(s, cu_seqlens, T, &tok0, &len);
        token_act a;
        double *S = (double *)calloc((size_t)(K * V), sizeof(double));
        double *work = (double *)malloc((size_t)V * sizeof(double));
        if (act_alloc(&a, K, V) || !S || !work) {
#pragma omp atomic write
            err = -2;
            act_free(&a); free(S); free(work);
            continue;
        }
        const size_t state_off = (size_t)(u * K * V);
        if (S0)
            memcpy(S, S0 + state_off, (size_t)(K * V) * sizeof(double));
        for (int64_t t = 0; t < len; ++t) {
            const int64_t tok = tok0 + t;
            activate_f64(&a, q, k, v, g, beta, A_log, dt_bias, lower_bound, eps, tok, h, H);
            recurrence_step(K, V, S, a.qh, a.kh, a.vv, a.b, a.lam, scale,
                            out ? out + (tok * H + h) * V : NULL, work);
        }
        if (final_state)
            memcpy(final_state + state_off, S, (size_t)(K * V) * sizeof(double));
        act_free(&a); free(S); free(work);
    }
    return err;
}

/*
 * Reverse-mode step through token t of one (sequence, head).
 *   Sprev: state before the token (K x V), read only.
 *   dS:    on entry dL/dS_t from everything after the token (later tokens and the
 *          final state); on exit dL/dS_{t-1}.
 *   dO_t:  dL/dout_t [V].
 * Writes dv [V]; returns dqh, dkh, dlam [K] and db (all w.r.t. the activations).
 * work: 3*V + K*V doubles of scratch.
 *
 * Forward relations differentiated (the recurrence of the operator):
 *   Sp = Diag(alpha) Sprev, alpha = exp(lam);  r = v - Sp^T kh;
 *   S_t = Sp + b kh r^T;  out_t = scale S_t^T qh.
 */
static void reverse_step(int64_t K, int64_t V, const double *Sprev, double *dS,
                         const token_act *a, double scale, const double *dO_t, double *dqh,
                         double *dkh, double *dlam, double *db, double *dv, double *work)
{
    double *r = work, *e = work + V, *dr = work + 2 * V, *Sp = work + 3 * V;
    for (int64_t c = 0; c < K; ++c) {
        const double al = exp(a->lam[c]);
        for (int64_t j = 0; j < V; ++j)
            Sp[c * V + j] = al * Sprev[c * V + j];
    }
    for (int64_t j = 0; j < V; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < K; ++c)
            acc += Sp[c * V + j] * a->kh[c];
        r[j] = a->vv[j] - acc;
    }
    /* out_t = scale S_t^T qh: dS_t += scale qh dO^T, dqh = scale S_t dO */
    for (int64_t c = 0; c < K; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < V; ++j) {
            const double St = Sp[c * V + j] + a->b * a->kh[c] * r[j];
            acc += St * dO_t[j];
            dS[c * V + j] += scale * a->qh[c] * dO_t[j];
        }
        dqh[c] = scale * acc;
    }
    /* S_t = Sp + b kh r^T: e = dS^T kh, dr = b e, db = r . e, dkh = b dS r */
    for (int64_t j = 0; j < V; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < K; ++c)
            acc += dS[c * V + j] * a->kh[c];
        e[j] = acc;
        dr[j] = a->b * acc;
    }
    double dbs = 0.0;
    for (int64_t j = 0; j < V; ++j)
        dbs += r[j] * e[j];
    *db = dbs;
    for (int64_t c = 0; c < K; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < V; ++j)
            acc += dS[c * V + j] * r[j];
        dkh[c] = a->b * acc;
    }
    /* r = v - Sp^T kh: dv = dr, dSp = dS - kh dr^T, dkh -= Sp dr */
    for (int64_t j = 0; j < V; ++j)
        dv[j] = dr[j];
    for (int64_t c = 0; c < K; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < V; ++j) {
            acc += Sp[c * V + j] * dr[j];
            dS[c * V + j] -= a->kh[c] * dr[j];
        }
        dkh[c] -= acc;
    }
    /* Sp = Diag(alpha) Sprev: dalpha = rowsum(dSp o Sprev), dSprev = Diag(alpha) dSp;
     * alpha = exp(lam): dlam = dalpha alpha */
    for (int64_t c = 0; c < K; ++c) {
        const double al = exp(a->lam[c]);
        double acc = 0.0;
        for (int64_t j = 0; j < V; ++j) {
            acc += dS[c * V + j] * Sprev[c * V + j];
            dS[c * V + j] *= al;
        }
        dlam[c] = acc * al;
    }
}

/*
 * Backward of kda_oracle_fwd_f64.  Inputs as there, plus dO [B,T,H,V] and
 * dS_final [N,H,K,V] (NULL = zero).  Outputs (fp64, same layouts as the inputs):
 * dq, dk, dg [B,T,H,K], dv [B,T,H,V], dbeta [B,T,H], dA_log [H], ddt_bias [H,K],
 * dS0 [N,H,K,V] (may be NULL), and dlam_out [B,T,H,K] = dL/dlam (may be NULL; lets a
 * test see both sides of the clamp's kink).  Tokens outside every sequence are left
 * untouched.
 */
int kda_oracle_bwd_f64(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, double scale, const double *A_log,
                       const double *dt_bias, double lower_bound, const double *S0,
                       const double *dO, const double *dS_final, const int64_t *cu_seqlens,
                       int64_t num_seqs, double *dq, double *dk, double *dv, double *dg,
                       double *dbeta, double *dA_log, double *ddt_bias, double *dS0,
                       double *dlam_out, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                       double eps)
{
    if (B < 1 || T < 0 || H < 1 || K < 1 || V < 1)
        return -1;
    if (cu_seqlens && (B != 1 || num_seqs < 1))
        return -1;
    const int64_t N = cu_seqlens ? num_seqs : B;
    const int64_t units = N * H;
    /* per-unit partial sums of dA_log and ddt_bias, reduced in order afterwards */
    double *part = (double *)calloc((size_t)(units * (K + 1)), sizeof(double));
    if (!part)
        return -2;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int64_t s = u / H, h = u % H;
        int64_t tok0, len;
        sequence_span(s, cu_seqlens, T, &tok0, &len);
        const int64_t KV = K * V, nck = len / ORACLE_CKPT + 1;
        token_act a;
        double *ck = (double *)calloc((size_t)(nck * KV), sizeof(double));
        double *states = (double *)malloc((size_t)((ORACLE_CKPT + 1) * KV) * sizeof(double));
        double *dS = (double *)calloc((size_t)KV, sizeof(double));
        double *work = (double *)malloc((size_t)(3 * V + KV) * sizeof(double));
        double *dqh = (double *)malloc((size_t)(3 * K) * sizeof(double));
        if (act_alloc(&a, K, V) || !ck || !states || !dS || !work || !dqh) {
#pragma omp atomic write
            err = -2;
            act_free(&a); free(ck); free(states); free(dS); free(work); free(dqh);
            continue;
        }
        double *dkh = dqh + K, *dlam = dqh + 2 * K;
        const size_t state_off = (size_t)(u * KV);

        /* forward sweep: checkpoint the state before tokens 0, CKPT, 2 CKPT, ... */
        if (S0)
            memcpy(ck, S0 + state_off, (size_t)KV * sizeof(double));
        memcpy(states, ck, (size_t)KV * sizeof(double));
        for (int64_t t = 0; t < len; ++t) {
            activate_f64(&a, q, k, v, g, beta, A_log, dt_bias, lower_bound, eps, tok0 + t, h, H);
            recurrence_step(K, V, states, a.qh, a.kh, a.vv, a.b, a.lam, scale, NULL, work);
            if ((t + 1) % ORACLE_CKPT == 0 && (t + 1) / ORACLE_CKPT < nck)
                memcpy(ck + ((t + 1) / ORACLE_CKPT) * KV, states, (size_t)KV * sizeof(double));
        }

        /* reverse sweep, one checkpoint block at a time */
        if (dS_final)
            memcpy(dS, dS_final + state_off, (size_t)KV * sizeof(double));
        double *dAp = part + u * (K + 1);
        for (int64_t blk = (len - 1) / ORACLE_CKPT; len > 0 && blk >= 0; --blk) {
            const int64_t t0 = blk * ORACLE_CKPT;
            const int64_t t1 = t0 + ORACLE_CKPT < len ? t0 + ORACLE_CKPT : len;
            /* states[i] = state before token t0 + i */
            memcpy(states, ck + blk * KV, (size_t)KV * sizeof(double));
            for (int64_t t = t0; t + 1 < t1; ++t) {
                memcpy(states + (t - t0 + 1) * KV, states + (t - t0) * KV,
                       (size_t)KV * sizeof(double));
                activate_f64(&a, q, k, v, g, beta, A_log, dt_bias, lower_bound, eps, tok0 + t, h, H);
                recurrence_step(K, V, states + (t - t0 + 1) * KV, a.qh, a.kh, a.vv, a.b, a.lam,
                                scale, NULL, work);
            }
            for (int64_t t = t1 - 1; t >= t0; --t) {
                const int64_t tok = tok0 + t;
                activate_f64(&a, q, k, v, g, beta, A_log, dt_bias, lower_bound, eps, tok, h, H);
                double db;
                reverse_step(K, V, states + (t - t0) * KV, dS, &a, scale, dO + (tok * H + h) * V,
                             dqh, dkh, dlam, &db, dv + (tok * H + h) * V, work);
                /* q^ = q rq: dq = rq (dqh - q^ (q^ . dqh)); the same for k */
                double pq = 0.0, pk = 0.0;
                for (int64_t c = 0; c < K; ++c) {
                    pq += a.qh[c] * dqh[c];
                    pk += a.kh[c] * dkh[c];
                }
                const double ea = exp(A_log[h]);
                for (int64_t c = 0; c < K; ++c) {
                    dq[(tok * H + h) * K + c] = a.rq * (dqh[c] - a.qh[c] * pq);
                    dk[(tok * H + h) * K + c] = a.rk * (dkh[c] - a.kh[c] * pk);
                    /* lam = max(lb, z), z = -exp(A_log) softplus(x), softplus' = sigmoid */
                    double dx = 0.0;
                    if (a.z[c] >= lower_bound) {
                        dx = -dlam[c] * ea / (1.0 + exp(-a.x[c]));
                        dAp[K] += dlam[c] * a.z[c];
                    }
                    dg[(tok * H + h) * K + c] = dx;
                    if (dlam_out)
                        dlam_out[(tok * H + h) * K + c] = dlam[c];
                    dAp[c] += dx;
                }
                dbeta[tok * H + h] = db * a.b * (1.0 - a.b);
            }
        }
        if (dS0)
            memcpy(dS0 + state_off, dS, (size_t)KV * sizeof(double));
        act_free(&a); free(ck); free(states); free(dS); free(work); free(dqh);
    }
    for (int64_t hh = 0; hh < H; ++hh) {
        double sa = 0.0;
        for (int64_t c = 0; c < K; ++c)
            ddt_bias[hh * K + c] = 0.0;
        for (int64_t s = 0; s < N; ++s) {
            const double *p = part + (s * H + hh) * (K + 1);
            for (int64_t c = 0; c < K; ++c)
                ddt_bias[hh * K + c] += p[c];
            sa += p[K];
        }
        dA_log[hh] = sa;
    }
    free(part);
    return err;
}
