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
// units.  Thread (r8, cg): rows c = 32 g + 4 r8 + j (g, j < 4; 16 rows) of the two
// value columns 2 cg, 2 cg + 1; S and dS live in registers.  The columns of S evolve
// independently; the reductions over k of one column stay inside a warp (its eight
// row groups are adjacent lanes).  Each row's k^ / alpha / q^ values, read from
// shared memory, serve two columns: a step is bound by the shared-memory-to-register
// path, so the bytes read per step are what this layout halves.
//   1. Forward sweep over the sequence; the state before every 64-token chunk is
//      stored in the workspace.
//   2. Reverse over the chunks.  For each chunk: re-run it from its checkpoint and
//      keep the state before each 4-token sub-chunk (workspace, per CTA).  Then,
//      per sub-chunk in reverse, per token in reverse, re-run the sub-chunk from its
//      start state up to the token (at most 3 steps) and take the reverse step.
// Reductions over v (for dq^, dk^, dalpha) sum the thread's two columns and
// reduce-scatter over the warp's four column groups; each token's per-warp partials
// go to their own shared-memory slot, summed over the 16 warps once the sub-chunk's
// tokens are done (no barrier per token).  The norms, gate and sigmoid gradients of
// the sub-chunk follow.  While a sub-chunk computes, the rows of the next one are
// prefetched into L2.  Everything is fp32 on the CUDA cores: each step is a
// matrix-vector product on the state, with no contraction large enough for the
// tensor cores.
#include <cstddef>

#include "kda.h"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int BT = 512;          // threads per CTA
constexpr int NW = BT / 32;      // 16 warps
constexpr int RR = 16;           // state rows per thread (per column)
constexpr int NS = 2 * RR;       // state entries per thread
constexpr int SUB = 4;           // tokens per sub-chunk
constexpr int CH = 64;           // tokens per checkpoint chunk
constexpr int NSUB = CH / SUB;   // sub-chunks per chunk
constexpr int STATE = kHead * kHead;
constexpr unsigned FULL = 0xffffffffu;

struct Smem {
    float4 ssub[NS / 4][BT];     // start state of the current sub-chunk, thread-private
    alignas(16) float kh[SUB][kHead];
    alignas(16) float qh[SUB][kHead];
    alignas(16) float al[SUB][kHead];
    alignas(16) float xs[SUB][kHead];
    alignas(16) float zs[SUB][kHead];
    alignas(16) float vv[SUB][kHead];
    alignas(16) float dO[SUB][kHead];
    alignas(16) float red[SUB][NW][3][kHead];  // per-warp row sums of each token of the sub-chunk
    alignas(16) float res[SUB][3][kHead];    // dq^ / scale, dk^, dalpha per token of the sub-chunk
    float b[SUB], rq[SUB], rk[SUB];
    float redb[SUB][NW];
    float resb[SUB];             // db per token
    float dtb[kHead];
    float pacc[SUB][kHead + 1];  // per-epilogue-warp partial ddt_bias and dA_log
};

// Thread layout: lane = 8 cgl + r8; column group cg = 4 warp + cgl (columns 2 cg,
// 2 cg + 1); register entry i = 4 g + j holds row 32 g + 4 r8 + j.
struct Lane {
    int r8, cgl, v0;
};

__device__ __forceinline__ int row_of(const Lane &L, int i) { return 32 * (i >> 2) + 4 * L.r8 + (i & 3); }

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float f4(const float4 &a, int j) { return j == 0 ? a.x : j == 1 ? a.y : j == 2 ? a.z : a.w; }

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

// Sum over the eight row groups of a column (lane bits 0..2).
__device__ __forceinline__ float rows_sum(float x)
{
    x += __shfl_xor_sync(FULL, x, 1);
    x += __shfl_xor_sync(FULL, x, 2);
    x += __shfl_xor_sync(FULL, x, 4);
    return x;
}

// Reduce-scatter over the warp's four column groups (lane bits 3, 4) of a 16-row
// partial delivered in pairs: lo = entry i, hi = entry i + 8 (i < 8).  The first
// round (partner lane ^ 16) halves the rows; `half` collects them.
__device__ __forceinline__ float scatter_a(float lo, float hi, int cgl)
{
    const bool up = cgl & 2;
    return (up ? hi : lo) + __shfl_xor_sync(FULL, up ? lo : hi, 16);
}

// Second round (partner lane ^ 8): entries 4 cgl .. 4 cgl + 3 of the column sums.
__device__ __forceinline__ float4 scatter_b(const float (&h)[8], int cgl)
{
    const bool up = cgl & 1;
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = (up ? h[i + 4] : h[i]) + __shfl_xor_sync(FULL, up ? h[i] : h[i + 4], 8);
    return make_float4(o[0], o[1], o[2], o[3]);
}

// Stage tokens [tok, tok + L) of head h (L <= SUB): activations per channel, v (and
// dO when want_dO) per column.  Warps 0..7 take one token's channels each, warps
// 8..15 its v / dO.
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
        float qo[4], ko[4], ao[4], xo[4], zo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x = f4(g4, j) + sm.dtb[c0 + j];
            const float sp = fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));  // softplus
            const float z = -ea * sp;
            qo[j] = f4(q4, j) * rq;
            ko[j] = f4(k4, j) * rk;
            xo[j] = x;
            zo[j] = z;
            ao[j] = expf(fmaxf(p.lower_bound, z));
        }
        *reinterpret_cast<float4 *>(&sm.qh[tt][c0]) = make_float4(qo[0], qo[1], qo[2], qo[3]);
        *reinterpret_cast<float4 *>(&sm.kh[tt][c0]) = make_float4(ko[0], ko[1], ko[2], ko[3]);
        *reinterpret_cast<float4 *>(&sm.al[tt][c0]) = make_float4(ao[0], ao[1], ao[2], ao[3]);
        *reinterpret_cast<float4 *>(&sm.xs[tt][c0]) = make_float4(xo[0], xo[1], xo[2], xo[3]);
        *reinterpret_cast<float4 *>(&sm.zs[tt][c0]) = make_float4(zo[0], zo[1], zo[2], zo[3]);
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

// Hint the rows of tokens [tok, tok + L) of head h towards L2, so that the stage() of
// that sub-chunk waits on L2 rather than DRAM: one 128-byte line per thread (two per
// 256-byte row of q, k, g, v and, with want_dO, dO), beta by threads 448 and up.
__device__ __forceinline__ void prefetch_rows(const BwdParams &p, int64_t tok, int L, int64_t h,
                                              bool want_dO)
{
    const int t = threadIdx.x;
    const int narr = want_dO ? 5 : 4;
    if (t < narr * 2 * L) {
        const int a = t / (2 * L), rem = t - a * 2 * L, tt = rem >> 1, half = rem & 1;
        const __nv_bfloat16 *base = a == 0 ? p.q : a == 1 ? p.k : a == 2 ? p.g : a == 3 ? p.v : p.dout;
        const __nv_bfloat16 *addr = base + ((tok + tt) * p.H + h) * kHead + 64 * half;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(addr));
    } else if (t >= 448 && t < 448 + L) {
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.beta + (tok + (t - 448)) * p.H + h));
    }
}

// One token of the recurrence on this thread's 16 rows of its two columns.
// s[i] is column 2 cg, s[RR + i] column 2 cg + 1.
__device__ __forceinline__ void fwd_step(float (&s)[NS], const Smem &sm, int tt, const Lane &L)
{
    float pa0 = 0.f, pa1 = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 k4 = ld4(&sm.kh[tt][32 * g + 4 * L.r8]), a4 = ld4(&sm.al[tt][32 * g + 4 * L.r8]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 4 * g + j;
            s[i] *= f4(a4, j);
            s[RR + i] *= f4(a4, j);
            pa0 = fmaf(s[i], f4(k4, j), pa0);
            pa1 = fmaf(s[RR + i], f4(k4, j), pa1);
        }
    }
    pa0 = rows_sum(pa0);
    pa1 = rows_sum(pa1);
    const float2 v2 = *reinterpret_cast<const float2 *>(&sm.vv[tt][L.v0]);
    const float bt = sm.b[tt];
    const float br0 = bt * (v2.x - pa0), br1 = bt * (v2.y - pa1);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 k4 = ld4(&sm.kh[tt][32 * g + 4 * L.r8]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 4 * g + j;
            s[i] = fmaf(f4(k4, j), br0, s[i]);
            s[RR + i] = fmaf(f4(k4, j), br1, s[RR + i]);
        }
    }
}

__global__ void __launch_bounds__(BT, 1) bwd_kernel(const BwdParams p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    Lane L;
    L.r8 = lane & 7;
    L.cgl = lane >> 3;
    L.v0 = 2 * (4 * warp + L.cgl);
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
        // entry i of this thread's two columns in a [K][V] state: + row * 128 + v0 (+1)
        auto at = [&](int i) { return (size_t)row_of(L, i) * kHead + L.v0; };
        __syncthreads();  // the previous unit's last readers of dtb / pacc are done
        if (tid < kHead) sm.dtb[tid] = p.dt_bias[h * kHead + tid];

        // ---- 1. forward sweep: checkpoints before every chunk ----
        // (dtype tests outside the unrolled loops: the 16 loads are in flight together)
        float s[NS];
        if (p.init && p.init_dtype == KDA_STATE_BF16) {
            const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(p.init) + st_off;
#pragma unroll
            for (int i = 0; i < RR; ++i) {
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(src + at(i)));
                s[i] = x.x;
                s[RR + i] = x.y;
            }
        } else if (p.init) {
            const float *src = static_cast<const float *>(p.init) + st_off;
#pragma unroll
            for (int i = 0; i < RR; ++i) {
                const float2 x = *reinterpret_cast<const float2 *>(src + at(i));
                s[i] = x.x;
                s[RR + i] = x.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NS; ++i) s[i] = 0.f;
        }
        for (int64_t n = 0; n < nch; ++n) {
            float *c = ck + n * ck_stride;
#pragma unroll
            for (int i = 0; i < RR; ++i) *reinterpret_cast<float2 *>(c + at(i)) = make_float2(s[i], s[RR + i]);
            for (int j = 0; j < NSUB; ++j) {
                const int64_t t0 = n * CH + j * SUB;
                if (t0 >= len) break;
                const int Lj = (int)(len - t0 < SUB ? len - t0 : SUB);
                __syncthreads();
                stage(sm, p, bos + t0, Lj, h, ea, false);
                __syncthreads();
                if (t0 + SUB < len)
                    prefetch_rows(p, bos + t0 + SUB, (int)(len - t0 - SUB < SUB ? len - t0 - SUB : SUB), h, false);
                for (int tt = 0; tt < Lj; ++tt) fwd_step(s, sm, tt, L);
            }
        }

        // ---- 2. reverse sweep ----
        float ds[NS];
        if (p.dfinal) {
#pragma unroll
            for (int i = 0; i < RR; ++i) {
                const float2 x = *reinterpret_cast<const float2 *>(p.dfinal + st_off + at(i));
                ds[i] = x.x;
                ds[RR + i] = x.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NS; ++i) ds[i] = 0.f;
        }
        for (int i = tid; i < SUB * (kHead + 1); i += BT) (&sm.pacc[0][0])[i] = 0.f;

        for (int64_t n = nch - 1; n >= 0; --n) {
            const int64_t left = (len - n * CH + SUB - 1) / SUB;
            const int nsub = (int)(left < NSUB ? left : NSUB);
            // 2a. start states of the chunk's sub-chunks
            {
                const float *c = ck + n * ck_stride;
#pragma unroll
                for (int i = 0; i < RR; ++i) {
                    const float2 x = *reinterpret_cast<const float2 *>(c + at(i));
                    s[i] = x.x;
                    s[RR + i] = x.y;
                }
            }
            for (int j = 0; j < nsub; ++j) {
#pragma unroll
                for (int i = 0; i < NS; i += 4)
                    scr[((size_t)j * (NS / 4) + i / 4) * BT + tid] =
                        make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
                if (j == nsub - 1) break;
                __syncthreads();
                stage(sm, p, bos + n * CH + j * SUB, SUB, h, ea, false);
                __syncthreads();
                {
                    // next: sub-chunk j + 1 here, or (the last one) the first of 2b, with dO
                    const int64_t tn = n * CH + (j + 1) * SUB;
                    prefetch_rows(p, bos + tn, (int)(len - tn < SUB ? len - tn : SUB), h, j + 1 == nsub - 1);
                }
                for (int tt = 0; tt < SUB; ++tt) fwd_step(s, sm, tt, L);
            }
            // 2b. sub-chunks in reverse
            for (int j = nsub - 1; j >= 0; --j) {
                const int64_t t0 = n * CH + j * SUB;
                const int Lj = (int)(len - t0 < SUB ? len - t0 : SUB);
                __syncthreads();
                stage(sm, p, bos + t0, Lj, h, ea, true);
#pragma unroll
                for (int i = 0; i < NS / 4; ++i) sm.ssub[i][tid] = scr[((size_t)j * (NS / 4) + i) * BT + tid];
                __syncthreads();
                // next: sub-chunk j - 1 (with dO), or the first sub-chunk of chunk n - 1 (2a)
                if (j > 0)
                    prefetch_rows(p, bos + t0 - SUB, SUB, h, true);
                else if (n > 0)
                    prefetch_rows(p, bos + (n - 1) * CH, SUB, h, false);
                for (int tt = Lj - 1; tt >= 0; --tt) {
#pragma unroll
                    for (int i = 0; i < NS / 4; ++i) {
                        const float4 f = sm.ssub[i][tid];
                        s[4 * i] = f.x;
                        s[4 * i + 1] = f.y;
                        s[4 * i + 2] = f.z;
                        s[4 * i + 3] = f.w;
                    }
                    for (int t2 = 0; t2 < tt; ++t2) fwd_step(s, sm, t2, L);
                    // s = S_{t-1}; ds = dL/dS_t from everything after token t
                    const float *kr = &sm.kh[tt][4 * L.r8], *ar = &sm.al[tt][4 * L.r8];
                    const float *qp = &sm.qh[tt][4 * L.r8];  // row group g at + 32 g
                    const float bt = sm.b[tt];
                    float pa0 = 0.f, pa1 = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const float4 k4 = ld4(kr + 32 * g), a4 = ld4(ar + 32 * g);
#pragma unroll
                        for (int j2 = 0; j2 < 4; ++j2) {
                            const int i = 4 * g + j2;
                            pa0 = fmaf(f4(a4, j2) * s[i], f4(k4, j2), pa0);
                            pa1 = fmaf(f4(a4, j2) * s[RR + i], f4(k4, j2), pa1);
                        }
                    }
                    pa0 = rows_sum(pa0);
                    pa1 = rows_sum(pa1);
                    const float2 v2 = *reinterpret_cast<const float2 *>(&sm.vv[tt][L.v0]);
                    const float2 o2 = *reinterpret_cast<const float2 *>(&sm.dO[tt][L.v0]);
                    const float r0 = v2.x - pa0, r1 = v2.y - pa1;
                    const float br0 = bt * r0, br1 = bt * r1;
                    const float dOs0 = p.scale * o2.x, dOs1 = p.scale * o2.y;
                    float e0 = 0.f, e1 = 0.f;
                    // dS_t += scale q^ dO^T; dq^ partial S_t dO; e partial dS^T k^
                    {
                        float hf[8];
#pragma unroll
                        for (int g = 0; g < 2; ++g) {
                            const float4 kl = ld4(kr + 32 * g), kh4 = ld4(kr + 32 * (g + 2));
                            const float4 al4 = ld4(ar + 32 * g), ah4 = ld4(ar + 32 * (g + 2));
                            const float4 ql = ld4(qp + 32 * g), qh4 = ld4(qp + 32 * (g + 2));
#pragma unroll
                            for (int j2 = 0; j2 < 4; ++j2) {
                                float x[2];
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int i = 4 * g + j2 + 8 * hh;
                                    const float kk = f4(hh ? kh4 : kl, j2), aa = f4(hh ? ah4 : al4, j2);
                                    const float qq = f4(hh ? qh4 : ql, j2);
                                    const float st0 = fmaf(kk, br0, aa * s[i]);
                                    const float st1 = fmaf(kk, br1, aa * s[RR + i]);
                                    ds[i] = fmaf(qq, dOs0, ds[i]);
                                    ds[RR + i] = fmaf(qq, dOs1, ds[RR + i]);
                                    e0 = fmaf(ds[i], kk, e0);
                                    e1 = fmaf(ds[RR + i], kk, e1);
                                    x[hh] = fmaf(st0, o2.x, st1 * o2.y);
                                }
                                hf[4 * g + j2] = scatter_a(x[0], x[1], L.cgl);
                            }
                        }
                        *reinterpret_cast<float4 *>(&sm.red[tt][warp][0][32 * L.cgl + 4 * L.r8]) =
                            scatter_b(hf, L.cgl);
                    }
                    e0 = rows_sum(e0);
                    e1 = rows_sum(e1);
                    const float dr0 = bt * e0, dr1 = bt * e1;
                    const float dbw = warp_sum(L.r8 == 0 ? fmaf(r0, e0, r1 * e1) : 0.f);
                    if (lane == 0) sm.redb[tt][warp] = dbw;
                    if (L.r8 == 0)
                        *reinterpret_cast<float2 *>(p.dv + (bos + t0 + tt) * p.H * kHead + h * kHead + L.v0) =
                            make_float2(dr0, dr1);
                    // dk^ partial: b dS r - S' dr (dS = dL/dS_t)
                    {
                        float hf[8];
#pragma unroll
                        for (int g = 0; g < 2; ++g) {
                            const float4 al4 = ld4(ar + 32 * g), ah4 = ld4(ar + 32 * (g + 2));
#pragma unroll
                            for (int j2 = 0; j2 < 4; ++j2) {
                                float x[2];
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int i = 4 * g + j2 + 8 * hh;
                                    const float aa = f4(hh ? ah4 : al4, j2);
                                    x[hh] = fmaf(ds[i], br0, -(aa * s[i]) * dr0) +
                                            fmaf(ds[RR + i], br1, -(aa * s[RR + i]) * dr1);
                                }
                                hf[4 * g + j2] = scatter_a(x[0], x[1], L.cgl);
                            }
                        }
                        *reinterpret_cast<float4 *>(&sm.red[tt][warp][1][32 * L.cgl + 4 * L.r8]) =
                            scatter_b(hf, L.cgl);
                    }
                    // dS' = dS - k^ dr^T; dalpha partial rowsum(dS' o S_{t-1}); dS_{t-1} = alpha dS'
                    {
                        float hf[8];
#pragma unroll
                        for (int g = 0; g < 2; ++g) {
                            const float4 kl = ld4(kr + 32 * g), kh4 = ld4(kr + 32 * (g + 2));
                            const float4 al4 = ld4(ar + 32 * g), ah4 = ld4(ar + 32 * (g + 2));
#pragma unroll
                            for (int j2 = 0; j2 < 4; ++j2) {
                                float x[2];
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int i = 4 * g + j2 + 8 * hh;
                                    const float kk = f4(hh ? kh4 : kl, j2), aa = f4(hh ? ah4 : al4, j2);
                                    ds[i] = fmaf(-kk, dr0, ds[i]);
                                    ds[RR + i] = fmaf(-kk, dr1, ds[RR + i]);
                                    x[hh] = fmaf(ds[i], s[i], ds[RR + i] * s[RR + i]);
                                    ds[i] *= aa;
                                    ds[RR + i] *= aa;
                                }
                                hf[4 * g + j2] = scatter_a(x[0], x[1], L.cgl);
                            }
                        }
                        *reinterpret_cast<float4 *>(&sm.red[tt][warp][2][32 * L.cgl + 4 * L.r8]) =
                            scatter_b(hf, L.cgl);
                    }
                }
                // sums over the 16 warps of every token's partials
                __syncthreads();
                for (int it = tid; it < Lj * 3 * kHead; it += BT) {
                    const int tt = it / (3 * kHead), r = it - tt * 3 * kHead, arr = r >> 7, c = r & (kHead - 1);
                    float acc = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) acc += sm.red[tt][w][arr][c];
                    sm.res[tt][arr][c] = acc;
                }
                if (tid < Lj) {
                    float acc = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) acc += sm.redb[tid][w];
                    sm.resb[tid] = acc;
                }
                __syncthreads();
                // 2c. gradients through the activations of the sub-chunk's tokens
                if (warp < Lj) {
                    const int tt = warp, c0 = 4 * lane;
                    const int64_t row = (bos + t0 + tt) * p.H + h;
                    const float4 q4 = ld4(&sm.qh[tt][c0]), k4 = ld4(&sm.kh[tt][c0]);
                    const float4 a4 = ld4(&sm.al[tt][c0]), x4 = ld4(&sm.xs[tt][c0]);
                    const float4 z4 = ld4(&sm.zs[tt][c0]);
                    const float4 dqh4 = ld4(&sm.res[tt][0][c0]), dkh4 = ld4(&sm.res[tt][1][c0]);
                    const float4 da4 = ld4(&sm.res[tt][2][c0]);
                    float pq = 0.f, pk = 0.f;
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) {
                        pq = fmaf(f4(q4, j2), p.scale * f4(dqh4, j2), pq);
                        pk = fmaf(f4(k4, j2), f4(dkh4, j2), pk);
                    }
                    pq = warp_sum(pq);
                    pk = warp_sum(pk);
                    const float rq = sm.rq[tt], rk = sm.rk[tt];
                    float dqo[4], dko[4], dgo[4];
                    float dA = 0.f;
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) {
                        dqo[j2] = rq * (p.scale * f4(dqh4, j2) - f4(q4, j2) * pq);
                        dko[j2] = rk * (f4(dkh4, j2) - f4(k4, j2) * pk);
                        const float dlam = f4(da4, j2) * f4(a4, j2);
                        const float z = f4(z4, j2);
                        const bool open = z >= p.lower_bound;  // clamp not holding
                        const float sig = 1.f / (1.f + expf(-f4(x4, j2)));
                        const float dx = open ? -dlam * ea * sig : 0.f;
                        dgo[j2] = dx;
                        sm.pacc[tt][c0 + j2] += dx;  // row tt belongs to this warp alone
                        dA += open ? dlam * z : 0.f;
                    }
                    dA = warp_sum(dA);
                    if (lane == 0) sm.pacc[tt][kHead] += dA;
                    *reinterpret_cast<float4 *>(p.dq + row * kHead + c0) = make_float4(dqo[0], dqo[1], dqo[2], dqo[3]);
                    *reinterpret_cast<float4 *>(p.dk + row * kHead + c0) = make_float4(dko[0], dko[1], dko[2], dko[3]);
                    *reinterpret_cast<float4 *>(p.dg + row * kHead + c0) = make_float4(dgo[0], dgo[1], dgo[2], dgo[3]);
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
            for (int i = 0; i < RR; ++i)
                *reinterpret_cast<float2 *>(p.dinit + st_off + at(i)) = make_float2(ds[i], ds[RR + i]);
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
    // per CTA: the token schedule's sub-chunk states, or the chunked schedule's tiles
    const size_t per_cta = (size_t)NSUB * STATE * 4 > bwd_chunked_scratch_bytes_per_cta()
                               ? (size_t)NSUB * STATE * 4
                               : bwd_chunked_scratch_bytes_per_cta();
    l.scratch_bytes = up((size_t)l.grid * per_cta);
    l.part_bytes = up((size_t)units * (kHead + 1) * 4);
    if (out) *out = l;
    return l.ckpt_bytes + l.scratch_bytes + l.part_bytes;
}

int launch_param_reduce(const BwdParams &p, cudaStream_t stream)
{
    param_reduce_kernel<<<(unsigned)p.H, kHead + 1, 0, stream>>>(p.part, p.N, p.H, p.dA_log,
                                                                 p.ddt_bias);
    return cudaGetLastError() == cudaSuccess ? 1 : KDA_ERR_CUDA;
}

int launch_backward_token(const BwdParams &p, const BwdLayout &l, cudaStream_t stream)
{
    const int64_t units = p.N * p.H;
    if (units <= 0) return 0;
    static int smem_set[64];
    const int smem = (int)sizeof(Smem);
    if (!set_smem_limit_once(bwd_kernel, smem, smem_set)) return KDA_ERR_CUDA;
    bwd_kernel<<<l.grid, BT, smem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    const int n = launch_param_reduce(p, stream);
    return n < 0 ? n : 1 + n;
}

}  // namespace kda
