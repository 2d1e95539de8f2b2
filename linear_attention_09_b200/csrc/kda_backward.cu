// KDA backward pass for sm_100a: reverse mode through the token recurrence.
//
// Operator (FlashKDA pages: 7minutos.es "¿Qué es la atención Kimi Delta...?"), per
// (sequence, head) with S (K x V, fp32, S[k][v]):
//   S'_t = Diag(alpha_t) S_{t-1},  r_t = v_t - S'_t^T k^_t,
//   S_t  = S'_t + b_t k^_t r_t^T,  out_t = scale S_t^T q^_t.
// Given dL/dout and dL/dS_final this computes dq, dk, dv, dg, dbeta (fp32, the
// layouts of the inputs), dA_log, ddt_bias and dL/dS_0.  Reverse mode of one token,
// with dS = dL/dS_t:
//   dS += scale q^ dO^T;  dq^ = scale S_t dO;  e = dS^T k^;  dr = b e;  db = r . e;
//   dk^ = b dS r - S'_t dr;  dv = dr;  dS' = dS - k^ dr^T;
//   dalpha = rowsum(dS' o S_{t-1});  dS_{t-1} = Diag(alpha) dS';
// then through the activations: the L2 norms, the sigmoid and the gate
// lam = max(lb, -exp(A_log) softplus(g + dt_bias)) (gradient zero where the clamp
// holds the value at lb, i.e. where -exp(A_log) softplus(x) < lb).
//
// Schedule.  One CTA of 512 threads per (sequence, head), persistent over the
// units.  Thread (v, qr): value column v, rows c = 32 qr + i (i < 32); S and dS live
// in registers.  The columns of S evolve independently (the reductions over k
// stay inside one warp: the four row quarters of a column are adjacent lanes).
//   1. Forward sweep over the sequence; the state before every 64-token chunk is
//      stored in the workspace.
//   2. Reverse over the chunks.  For each chunk: re-run it from its checkpoint and
//      keep the state before each 8-token sub-chunk (workspace, per CTA).  Then,
//      per sub-chunk in reverse, per token in reverse, re-run the sub-chunk from its
//      start state up to the token (at most 7 steps) and take the reverse step.
// Reductions over v (for dq^, dk^, dalpha) run as a reduce-scatter over the 8
// columns of a warp followed by a sum over the 16 warps in shared memory.  The
// norms, gate and sigmoid gradients of a sub-chunk are taken once its 8 tokens are
// done.  Everything is fp32 on the CUDA cores: each step is a matrix-vector
// product on the state, with no contraction large enough for the tensor cores.
#include <cstddef>

#include "kda.h"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int BT = 512;          // threads per CTA
constexpr int NW = BT / 32;      // 16 warps
constexpr int RQ = 32;           // state rows per thread
constexpr int SUB = 8;           // tokens per sub-chunk
constexpr int CH = 64;           // tokens per checkpoint chunk
constexpr int NSUB = CH / SUB;   // sub-chunks per chunk
constexpr int QP = 36;           // padded floats per row quarter (bank-conflict-free float4 reads)
constexpr int ROWP = 4 * QP;     // floats per token in the padded per-channel layout
constexpr int STATE = kHead * kHead;
constexpr unsigned FULL = 0xffffffffu;

struct Smem {
    float4 ssub[RQ / 4][BT];     // start state of the current sub-chunk, thread-private
    alignas(16) float kh[SUB][ROWP];
    alignas(16) float qh[SUB][ROWP];
    alignas(16) float al[SUB][ROWP];
    alignas(16) float xs[SUB][ROWP];
    alignas(16) float zs[SUB][ROWP];
    alignas(16) float vv[SUB][kHead];
    alignas(16) float dO[SUB][kHead];
    alignas(16) float red[2][NW][3][kHead + 32];  // per-warp row sums of one token (double-buffered)
    alignas(16) float res[SUB][3][kHead];    // dq^ / scale, dk^, dalpha per token of the sub-chunk
    float b[SUB], rq[SUB], rk[SUB];
    float redb[2][NW];
    float resb[SUB];             // db per token
    float dtb[kHead];
    float pacc[SUB][kHead + 1];  // per-epilogue-warp partial ddt_bias and dA_log
};

// Padded index of channel c: quarter c / 32 at a 36-float stride.
__device__ __forceinline__ int pidx(int c) { return (c >> 5) * QP + (c & 31); }

__device__ __forceinline__ float bf2f(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ float4 bf4(const __nv_bfloat16 *p, size_t i)
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(p + i);
    __nv_bfloat162 lo, hi;
    memcpy(&lo, &raw.x, 4);
    memcpy(&hi, &raw.y, 4);
    const float2 a = __bfloat1622float2(lo), c = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, c.x, c.y);
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

// Stage tokens [tok, tok + L) of head h (L <= SUB): activations in the padded
// per-channel layout, v (and dO when want_dO) per column.  Warps 0..7 take one
// token's channels each, warps 8..15 its v / dO.
__device__ void stage(Smem &sm, const BwdParams &p, int64_t tok, int L, int64_t h, float ea,
                      bool want_dO)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tt = warp & 7;
    if (tt >= L) return;
    const int64_t row = (tok + tt) * p.H + h;
    const int c0 = 4 * lane;
    if (warp < 8) {
        const float4 q4 = bf4(p.q, row * kHead + c0), k4 = bf4(p.k, row * kHead + c0);
        const float4 g4 = bf4(p.g, row * kHead + c0);
        const float sq = warp_sum(q4.x * q4.x + q4.y * q4.y + q4.z * q4.z + q4.w * q4.w);
        const float sk = warp_sum(k4.x * k4.x + k4.y * k4.y + k4.z * k4.z + k4.w * k4.w);
        const float rq = rsqrtf(sq + 1e-6f), rk = rsqrtf(sk + 1e-6f);
        const float qa[4] = {q4.x, q4.y, q4.z, q4.w}, ka[4] = {k4.x, k4.y, k4.z, k4.w};
        const float ga[4] = {g4.x, g4.y, g4.z, g4.w};
        float4 qo, ko, ao, xo, zo;
        float *qp = &qo.x, *kp = &ko.x, *ap = &ao.x, *xp = &xo.x, *zp = &zo.x;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x = ga[j] + sm.dtb[c0 + j];
            const float sp = fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));  // softplus
            const float z = -ea * sp;
            qp[j] = qa[j] * rq;
            kp[j] = ka[j] * rk;
            xp[j] = x;
            zp[j] = z;
            ap[j] = expf(fmaxf(p.lower_bound, z));
        }
        const int pi = pidx(c0);
        *reinterpret_cast<float4 *>(&sm.qh[tt][pi]) = qo;
        *reinterpret_cast<float4 *>(&sm.kh[tt][pi]) = ko;
        *reinterpret_cast<float4 *>(&sm.al[tt][pi]) = ao;
        *reinterpret_cast<float4 *>(&sm.xs[tt][pi]) = xo;
        *reinterpret_cast<float4 *>(&sm.zs[tt][pi]) = zo;
        if (lane == 0) {
            sm.rq[tt] = rq;
            sm.rk[tt] = rk;
            sm.b[tt] = 1.f / (1.f + expf(-bf2f(p.beta, row)));
        }
    } else {
        *reinterpret_cast<float4 *>(&sm.vv[tt][c0]) = bf4(p.v, row * kHead + c0);
        if (want_dO) *reinterpret_cast<float4 *>(&sm.dO[tt][c0]) = bf4(p.dout, row * kHead + c0);
    }
}

// One token of the recurrence on this thread's 32 rows of column v.
__device__ __forceinline__ void fwd_step(float (&s)[RQ], const Smem &sm, int tt, int qr, int v)
{
    const float *kr = &sm.kh[tt][qr * QP], *ar = &sm.al[tt][qr * QP];
    float pa = 0.f;
#pragma unroll
    for (int i = 0; i < RQ; i += 4) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kr + i);
        const float4 a4 = *reinterpret_cast<const float4 *>(ar + i);
        s[i] *= a4.x;
        s[i + 1] *= a4.y;
        s[i + 2] *= a4.z;
        s[i + 3] *= a4.w;
        pa = fmaf(s[i], k4.x, pa);
        pa = fmaf(s[i + 1], k4.y, pa);
        pa = fmaf(s[i + 2], k4.z, pa);
        pa = fmaf(s[i + 3], k4.w, pa);
    }
    pa += __shfl_xor_sync(FULL, pa, 1);
    pa += __shfl_xor_sync(FULL, pa, 2);
    const float br = sm.b[tt] * (sm.vv[tt][v] - pa);
#pragma unroll
    for (int i = 0; i < RQ; i += 4) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kr + i);
        s[i] = fmaf(k4.x, br, s[i]);
        s[i + 1] = fmaf(k4.y, br, s[i + 1]);
        s[i + 2] = fmaf(k4.z, br, s[i + 2]);
        s[i + 3] = fmaf(k4.w, br, s[i + 3]);
    }
}

// Reduce-scatter of 8 rows over the 8 columns of a warp (lane bits 2..4, m = lane >> 2):
// on entry x[i] is this lane's value for row i of a block of 8; returns the warp's sum
// for row m of the block.
__device__ __forceinline__ float reduce8(const float (&x)[8], int m)
{
    float y[4], z[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = m & 4;
        y[i] = (up ? x[i + 4] : x[i]) + __shfl_xor_sync(FULL, up ? x[i] : x[i + 4], 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = m & 2;
        z[i] = (up ? y[i + 2] : y[i]) + __shfl_xor_sync(FULL, up ? y[i] : y[i + 2], 8);
    }
    const bool up = m & 1;
    return (up ? z[1] : z[0]) + __shfl_xor_sync(FULL, up ? z[0] : z[1], 4);
}

// Position of channel c in the per-warp row sums: 8 floats of padding per quarter, so
// that the 32 lanes' stores of one block (c = 32 qr + 8 bk + m) hit 32 distinct banks.
__device__ __forceinline__ int ridx(int c) { return c + 8 * (c >> 5); }

__global__ void __launch_bounds__(BT, 1) bwd_kernel(const BwdParams p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = lane >> 2, qr = lane & 3;
    const int v = 8 * warp + m;
    const int64_t units = p.N * p.H;

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t sq = u / p.H, h = u % p.H;
        const int64_t bos = p.cu ? p.cu[sq] : sq * p.T;
        const int64_t len = p.cu ? p.cu[sq + 1] - bos : p.T;
        const int64_t nch = (len + CH - 1) / CH;
        const float ea = expf(p.A_log[h]);
        float *ck = p.ckpt + (size_t)((bos / CH + sq) * p.H + h) * STATE;  // chunk n at + n*H*STATE
        const size_t ck_stride = (size_t)p.H * STATE;
        float4 *scr = reinterpret_cast<float4 *>(p.scratch + (size_t)blockIdx.x * NSUB * STATE);
        const size_t st_off = (size_t)u * STATE;
        __syncthreads();  // the previous unit's last readers of dtb / pacc are done
        if (tid < kHead) sm.dtb[tid] = p.dt_bias[h * kHead + tid];

        // ---- 1. forward sweep: checkpoints before every chunk ----
        float s[RQ];
#pragma unroll
        for (int i = 0; i < RQ; ++i) {
            const size_t e = st_off + (size_t)(32 * qr + i) * kHead + v;
            s[i] = !p.init ? 0.f
                 : p.init_dtype == KDA_STATE_BF16 ? bf2f(static_cast<const __nv_bfloat16 *>(p.init), e)
                                                  : static_cast<const float *>(p.init)[e];
        }
        for (int64_t n = 0; n < nch; ++n) {
            float *c = ck + n * ck_stride;
#pragma unroll
            for (int i = 0; i < RQ; ++i) c[(32 * qr + i) * kHead + v] = s[i];
            for (int j = 0; j < NSUB; ++j) {
                const int64_t t0 = n * CH + j * SUB;
                if (t0 >= len) break;
                const int L = (int)(len - t0 < SUB ? len - t0 : SUB);
                __syncthreads();
                stage(sm, p, bos + t0, L, h, ea, false);
                __syncthreads();
                for (int tt = 0; tt < L; ++tt) fwd_step(s, sm, tt, qr, v);
            }
        }

        // ---- 2. reverse sweep ----
        float ds[RQ];
#pragma unroll
        for (int i = 0; i < RQ; ++i)
            ds[i] = p.dfinal ? p.dfinal[st_off + (size_t)(32 * qr + i) * kHead + v] : 0.f;
        for (int i = tid; i < SUB * (kHead + 1); i += BT) (&sm.pacc[0][0])[i] = 0.f;

        for (int64_t n = nch - 1; n >= 0; --n) {
            const int nsub = (int)((len - n * CH + SUB - 1) / SUB < NSUB ? (len - n * CH + SUB - 1) / SUB : NSUB);
            // 2a. start states of the chunk's sub-chunks
            {
                const float *c = ck + n * ck_stride;
#pragma unroll
                for (int i = 0; i < RQ; ++i) s[i] = c[(32 * qr + i) * kHead + v];
            }
            for (int j = 0; j < nsub; ++j) {
#pragma unroll
                for (int i = 0; i < RQ; i += 4)
                    scr[((size_t)j * (RQ / 4) + i / 4) * BT + tid] =
                        make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
                if (j == nsub - 1) break;
                __syncthreads();
                stage(sm, p, bos + n * CH + j * SUB, SUB, h, ea, false);
                __syncthreads();
                for (int tt = 0; tt < SUB; ++tt) fwd_step(s, sm, tt, qr, v);
            }
            // 2b. sub-chunks in reverse
            for (int j = nsub - 1; j >= 0; --j) {
                const int64_t t0 = n * CH + j * SUB;
                const int L = (int)(len - t0 < SUB ? len - t0 : SUB);
                __syncthreads();
                stage(sm, p, bos + t0, L, h, ea, true);
#pragma unroll
                for (int i = 0; i < RQ / 4; ++i) sm.ssub[i][tid] = scr[((size_t)j * (RQ / 4) + i) * BT + tid];
                __syncthreads();
                for (int tt = L - 1; tt >= 0; --tt) {
#pragma unroll
                    for (int i = 0; i < RQ / 4; ++i) {
                        const float4 f = sm.ssub[i][tid];
                        s[4 * i] = f.x;
                        s[4 * i + 1] = f.y;
                        s[4 * i + 2] = f.z;
                        s[4 * i + 3] = f.w;
                    }
                    for (int t2 = 0; t2 < tt; ++t2) fwd_step(s, sm, t2, qr, v);
                    // s = S_{t-1}; ds = dL/dS_t from everything after token t
                    const float *kr = &sm.kh[tt][qr * QP], *ar = &sm.al[tt][qr * QP];
                    const float *qp = &sm.qh[tt][qr * QP];
                    const float bt = sm.b[tt];
                    float pa = 0.f;
#pragma unroll
                    for (int i = 0; i < RQ; ++i) pa = fmaf(ar[i] * s[i], kr[i], pa);
                    pa += __shfl_xor_sync(FULL, pa, 1);
                    pa += __shfl_xor_sync(FULL, pa, 2);
                    const float r = sm.vv[tt][v] - pa, br = bt * r;
                    const float dOv = sm.dO[tt][v], dOs = p.scale * dOv;
                    const int buf = tt & 1;
                    float e = 0.f;
                    // dS_t += scale q^ dO^T; dq^ partial S_t dO; e partial dS^T k^
#pragma unroll
                    for (int bk = 0; bk < 4; ++bk) {
                        float x[8];
#pragma unroll
                        for (int i2 = 0; i2 < 8; ++i2) {
                            const int i = 8 * bk + i2;
                            const float st = fmaf(kr[i], br, ar[i] * s[i]);
                            ds[i] = fmaf(qp[i], dOs, ds[i]);
                            e = fmaf(ds[i], kr[i], e);
                            x[i2] = st * dOv;
                        }
                        sm.red[buf][warp][0][ridx(32 * qr + 8 * bk + m)] = reduce8(x, m);
                    }
                    e += __shfl_xor_sync(FULL, e, 1);
                    e += __shfl_xor_sync(FULL, e, 2);
                    const float dr = bt * e;
                    const float dbw = warp_sum(qr == 0 ? r * e : 0.f);
                    if (lane == 0) sm.redb[buf][warp] = dbw;
                    if (qr == 0) p.dv[(bos + t0 + tt) * p.H * kHead + h * kHead + v] = dr;
                    // dk^ partial: b dS r - S' dr (dS = dL/dS_t)
#pragma unroll
                    for (int bk = 0; bk < 4; ++bk) {
                        float x[8];
#pragma unroll
                        for (int i2 = 0; i2 < 8; ++i2) {
                            const int i = 8 * bk + i2;
                            x[i2] = fmaf(ds[i], br, -(ar[i] * s[i]) * dr);
                        }
                        sm.red[buf][warp][1][ridx(32 * qr + 8 * bk + m)] = reduce8(x, m);
                    }
                    // dS' = dS - k^ dr^T; dalpha partial rowsum(dS' o S_{t-1}); dS_{t-1} = alpha dS'
#pragma unroll
                    for (int bk = 0; bk < 4; ++bk) {
                        float x[8];
#pragma unroll
                        for (int i2 = 0; i2 < 8; ++i2) {
                            const int i = 8 * bk + i2;
                            ds[i] = fmaf(-kr[i], dr, ds[i]);
                            x[i2] = ds[i] * s[i];
                            ds[i] *= ar[i];
                        }
                        sm.red[buf][warp][2][ridx(32 * qr + 8 * bk + m)] = reduce8(x, m);
                    }
                    __syncthreads();
                    if (tid < 3 * kHead) {
                        const int arr = tid >> 7, c = tid & (kHead - 1);
                        float acc = 0.f;
#pragma unroll
                        for (int w = 0; w < NW; ++w) acc += sm.red[buf][w][arr][ridx(c)];
                        sm.res[tt][arr][c] = acc;
                    } else if (tid == 3 * kHead) {
                        float acc = 0.f;
#pragma unroll
                        for (int w = 0; w < NW; ++w) acc += sm.redb[buf][w];
                        sm.resb[tt] = acc;
                    }
                }
                __syncthreads();
                // 2c. gradients through the activations of the sub-chunk's tokens
                if (warp < L) {
                    const int tt = warp, c0 = 4 * lane, pi = pidx(c0);
                    const int64_t row = (bos + t0 + tt) * p.H + h;
                    const float4 q4 = *reinterpret_cast<const float4 *>(&sm.qh[tt][pi]);
                    const float4 k4 = *reinterpret_cast<const float4 *>(&sm.kh[tt][pi]);
                    const float4 a4 = *reinterpret_cast<const float4 *>(&sm.al[tt][pi]);
                    const float4 x4 = *reinterpret_cast<const float4 *>(&sm.xs[tt][pi]);
                    const float4 z4 = *reinterpret_cast<const float4 *>(&sm.zs[tt][pi]);
                    const float4 dqh4 = *reinterpret_cast<const float4 *>(&sm.res[tt][0][c0]);
                    const float4 dkh4 = *reinterpret_cast<const float4 *>(&sm.res[tt][1][c0]);
                    const float4 da4 = *reinterpret_cast<const float4 *>(&sm.res[tt][2][c0]);
                    const float qa[4] = {q4.x, q4.y, q4.z, q4.w}, ka[4] = {k4.x, k4.y, k4.z, k4.w};
                    const float aa[4] = {a4.x, a4.y, a4.z, a4.w}, xa[4] = {x4.x, x4.y, x4.z, x4.w};
                    const float za[4] = {z4.x, z4.y, z4.z, z4.w};
                    float dqh[4] = {dqh4.x, dqh4.y, dqh4.z, dqh4.w}, dkh[4] = {dkh4.x, dkh4.y, dkh4.z, dkh4.w};
                    const float dal[4] = {da4.x, da4.y, da4.z, da4.w};
                    float pq = 0.f, pk = 0.f;
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) {
                        dqh[j2] *= p.scale;
                        pq = fmaf(qa[j2], dqh[j2], pq);
                        pk = fmaf(ka[j2], dkh[j2], pk);
                    }
                    pq = warp_sum(pq);
                    pk = warp_sum(pk);
                    const float rq = sm.rq[tt], rk = sm.rk[tt];
                    float4 dq4, dk4, dg4;
                    float *dqo = &dq4.x, *dko = &dk4.x, *dgo = &dg4.x;
                    float dA = 0.f;
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) {
                        dqo[j2] = rq * (dqh[j2] - qa[j2] * pq);
                        dko[j2] = rk * (dkh[j2] - ka[j2] * pk);
                        const float dlam = dal[j2] * aa[j2];
                        const bool open = za[j2] >= p.lower_bound;  // clamp not holding
                        const float sig = 1.f / (1.f + expf(-xa[j2]));
                        const float dx = open ? -dlam * ea * sig : 0.f;
                        dgo[j2] = dx;
                        sm.pacc[tt][c0 + j2] += dx;  // row tt belongs to this warp alone
                        dA += open ? dlam * za[j2] : 0.f;
                    }
                    dA = warp_sum(dA);
                    if (lane == 0) sm.pacc[tt][kHead] += dA;
                    *reinterpret_cast<float4 *>(p.dq + row * kHead + c0) = dq4;
                    *reinterpret_cast<float4 *>(p.dk + row * kHead + c0) = dk4;
                    *reinterpret_cast<float4 *>(p.dg + row * kHead + c0) = dg4;
                    if (lane == 0) {
                        const float bt = sm.b[tt];
                        p.dbeta[row] = sm.resb[tt] * bt * (1.f - bt);
                    }
                }
            }
        }

        // ---- 3. dL/dS_0 and the per-unit parameter partials ----
        if (p.dinit) {
#pragma unroll
            for (int i = 0; i < RQ; ++i) p.dinit[st_off + (size_t)(32 * qr + i) * kHead + v] = ds[i];
        }
        __syncthreads();
        if (tid <= kHead) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < SUB; ++w) acc += sm.pacc[w][tid];
            p.part[(size_t)u * (kHead + 1) + tid] = acc;
        }
    }
}

// dA_log[h] and ddt_bias[h, :]: sums of the per-(sequence, head) partials, in
// sequence order.
__global__ void __launch_bounds__(kHead + 1) param_reduce_kernel(const float *part, int64_t N,
                                                                 int64_t H, float *dA_log,
                                                                 float *ddt_bias)
{
    const int64_t h = blockIdx.x;
    const int c = threadIdx.x;
    float acc = 0.f;
    for (int64_t s = 0; s < N; ++s) acc += part[(size_t)(s * H + h) * (kHead + 1) + c];
    if (c < kHead)
        ddt_bias[h * kHead + c] = acc;
    else
        dA_log[h] = acc;
}

}  // namespace

size_t bwd_layout(int64_t total_tokens, int64_t N, int64_t H, BwdLayout *out)
{
    const size_t a = 256;
    auto up = [a](size_t x) { return (x + a - 1) / a * a; };
    BwdLayout l{};
    const int64_t units = N * H;
    l.grid = (int)(units < kBwdMaxCtas ? units : kBwdMaxCtas);
    l.ckpt_bytes = up((size_t)(total_tokens / CH + N + 1) * H * STATE * 4);
    l.scratch_bytes = up((size_t)l.grid * NSUB * STATE * 4);
    l.part_bytes = up((size_t)units * (kHead + 1) * 4);
    if (out) *out = l;
    return l.ckpt_bytes + l.scratch_bytes + l.part_bytes;
}

int launch_backward(const BwdParams &p, const BwdLayout &l, cudaStream_t stream)
{
    const int64_t units = p.N * p.H;
    if (units <= 0) return 0;
    static int smem_set = 0;
    const int smem = (int)sizeof(Smem);
    if (!smem_set) {
        if (cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return KDA_ERR_CUDA;
        smem_set = 1;
    }
    bwd_kernel<<<l.grid, BT, smem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    param_reduce_kernel<<<(unsigned)p.H, kHead + 1, 0, stream>>>(p.part, p.N, p.H, p.dA_log,
                                                                 p.ddt_bias);
    return cudaGetLastError() == cudaSuccess ? 2 : KDA_ERR_CUDA;
}

}  // namespace kda
