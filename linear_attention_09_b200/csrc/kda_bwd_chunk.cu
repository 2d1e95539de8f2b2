// KDA backward pass for sm_100a in the chunked form: the adjoint of the per-chunk
// matrix form of the forward, over 64-token chunks in reverse.
//
// Forward of one chunk of L tokens from state S0 (K x V, S[k][v]), on the activations
// q^, k^, b, lam, with G the in-chunk inclusive cumulative sum of lam, Gam = e^G and
// GL = G[L-1] (the chunked form of the recurrence of the FlashKDA pages, 7minutos.es
// "¿Qué es la atención Kimi Delta...?"):
//   A_ij = sum_c k^_i k^_j e^(G_i - G_j) (j < i),  P_ij = same with q^_i (j <= i)
//   M = I + Diag(b) A,  T = M^-1 Diag(b),  Y = v - (k^ Gam) S0,  U = T Y
//   O = scale [(q^ Gam) S0 + P U],  S_end = Diag(e^GL) S0 + K'^T U,  K' = k^ e^(GL - G).
// Reverse of the chunk, given dO and dS (= dL/dS_end):
//   dU = scale P^T dO + K' dS;  dY = T^T dU = dv;  dT = dU Y^T (lower)
//   dS0 = scale (q^ Gam)^T dO + Diag(e^GL) dS - (k^ Gam)^T dY          (passed to chunk n-1)
//   d(k^ Gam) = -dY S0^T;  d(q^ Gam) = scale dO S0^T;  dP = scale dO U^T (lower)
//   dK' = U dS^T;  d(e^GL) contributes rowsum(dS o S0) e^GL to dG[L-1]
//   dM^-1 = dT Diag(b), db_j = sum_i dT_ij M^-1_ij;  dM = -M^-T dM^-1 M^-T
//   dA = Diag(b) dM (strict lower), db_i += sum_j dM_ij A_ij
// then through the decay-weighted products A and P into dq^, dk^ and dG (the factor
// e^(G_i - G_j) split at reference tokens of 16-token blocks, so that every factor stays
// in the fp32 range), and dlam = the reverse cumulative sum of dG over the chunk,
// followed by the gradients of the L2 norms, the sigmoid and the gate as in the
// token-level backward.
//
// The states before every chunk come from the forward kernel (its checkpoint
// instantiation, one launch before this one).  Schedule: one CTA of 512 threads per
// (sequence, head), persistent over the units, chunks in reverse; everything is fp32
// on the CUDA cores.  The activations (q^, k^, G; channel-major) and the 64 x 64
// matrices live in shared memory; the 64 x 128 tiles of a chunk (dO, dU, dY, the
// transposes of dO, Y, U and dY, k^ Gam, q^ Gam, K', the gradient accumulators) and dS
// live in a per-CTA scratch region of global memory (L2-resident as far as it fits).
// The products stream their operands from there through a two-slab shared-memory ring
// filled by cp.async (the copy of slab s + 1 in flight while slab s is used), so that
// L2 latency is not paid per load; Y and dU stay in the ring for the product right
// after theirs.  Every product is a register-blocked loop whose second operand is read
// along its rows by consecutive lanes, so each operand that appears in both
// orientations is stored in both.
#include <atomic>
#include <cstddef>

#include "kda.h"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int CC = 64;             // tokens per chunk
constexpr int CT = 512;            // threads per CTA
constexpr int CW = CT / 32;        // warps
constexpr int LDT = 65;            // row stride of the channel-major tiles and 64 x 64 matrices
constexpr int LDE = 129;           // row stride of the token-major epilogue tiles
constexpr int ST = kHead * kHead;  // floats of one state
constexpr int TILE = CC * kHead;   // floats of one 64 x 128 tile
constexpr unsigned FULL = 0xffffffffu;
constexpr float kL2e = 1.4426950408889634f;

constexpr int STG = 4096;  // floats of one slot of the operand ring
constexpr int NSLOT = 2;   // slots: slab s + 1 in flight while slab s is used

struct CSmem {
    float stg[NSLOT][STG];  // operand ring (first: 16-byte aligned for cp.async)
    float QT[kHead][LDT];  // q^   [channel][token]
    float KT[kHead][LDT];  // k^
    float GT[kHead][LDT];  // G log2(e): in-chunk inclusive cumulative sum of the log-decay
    union {
        struct {
            float A[CC][LDT];   // A (strict lower part; the rest 0)
            float PT[CC][LDT];  // P^T: PT[t][i] = P[i][t]; later W = dM^-1 M^-T
            float Mi[CC][LDT];  // M^-1 (unit lower)
            float X[CC][LDT];   // dT (lower), then dA (strict lower)
            float dP[CC][LDT];  // dP (lower)
        } m;
        struct {
            float o0[CC][LDE], o1[CC][LDE];  // [token][channel] staging of the outputs
            float red[2][CW][CC];            // per-warp partial sums of the norm gradients
        } e;
    } u;
    float b[CC], rq[CC], rk[CC], db[CC];
    float eGL[kHead], G2L[kHead], dGL[kHead], extra[kHead], dtb[kHead];
};

// Per-CTA scratch (floats): the tiles in the order of these offsets.  Two gradient
// accumulators reuse the tiles of operands that are dead by the time they are first
// written (phase 11): dq^ that of K' (last read in phase 8), dG that of dU (10).  Y
// itself never leaves the SM (phase 7 reads it from the operand ring).  A smaller
// footprint keeps more of the scratch in L2.
enum : int {
    S_DO = 0, S_DOT = TILE, S_KGT = 2 * TILE, S_QGT = 3 * TILE, S_KPT = 4 * TILE, S_DKT = 5 * TILE,
    S_YT = 6 * TILE, S_UT = 7 * TILE, S_DU = 8 * TILE, S_DY = 9 * TILE, S_DYT = 10 * TILE,
    S_DS = 11 * TILE, S_DQT = S_KPT, S_DGT = S_DU,
    S_PACC = 11 * TILE + ST,  // per-warp partial ddt_bias (0..127) and dA_log (128)
    S_FLOATS = S_PACC + CW * (kHead + 1)
};

__device__ __forceinline__ float ex2f(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2f(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(x) = max(x, 0) + ln(1 + e^-|x|) in the base-2 hardware functions (relative
// error ~1e-6, far inside the gradients' bars; where e^-|x| < 2^-24 the second term,
// then below 6e-8, rounds away against max(x, 0) > 16)
__device__ __forceinline__ float softplus_f(float x)
{
    return fmaxf(x, 0.f) + 0.6931471805599453f * lg2f(1.f + ex2f(-fabsf(x) * kL2e));
}

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + ex2f(-x * kL2e)); }

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// L2 policy for inputs read once per chunk: evicted before the scratch tiles.
__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ float bf_once(const __nv_bfloat16 *p, size_t i, uint64_t pol)
{
    unsigned short x;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(x) : "l"(p + i), "l"(pol));
    return __bfloat162float(__ushort_as_bfloat16(x));
}

__device__ __forceinline__ float wsum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

__device__ __forceinline__ void cp16(float *dst, const float *src)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// This thread's share of copying n contiguous floats (n % 4 == 0, 16-byte aligned).
__device__ __forceinline__ void stage_rows(float *dst, const float *src, int n)
{
    for (int i = threadIdx.x; i < n / 4; i += CT) cp16(dst + 4 * i, src + 4 * i);
}

// This thread's share of copying columns [c, c + w) of `rows` rows of a row-major matrix
// with leading dimension ld into a dense [rows][w] block (w % 4 == 0).
__device__ __forceinline__ void stage_cols(float *dst, const float *src, int rows, int ld, int c, int w)
{
    const int per = w / 4;
    for (int i = threadIdx.x; i < rows * per; i += CT) {
        const int r = i / per, q = i - r * per;
        cp16(dst + r * w + 4 * q, src + (size_t)r * ld + c + 4 * q);
    }
}

// Slabs 0..nslab-1 of a product: issue(s, buf) starts the copies of slab s into ring
// slot s % 2, body(buf, s) uses it once it has landed (every thread's copies); the
// copy of slab s + 1 is in flight during body(., s).  Called by all threads; ends
// with a barrier, after which the ring is free.  (Measured: slabs of 16 rows in two
// slots beat slabs of 8 in four slots with two in flight; the cost per slab does not
// shrink with its size.)
template <class Issue, class Body>
__device__ __forceinline__ void staged(float (*stg)[STG], int nslab, Issue issue, Body body)
{
    issue(0, stg[0]);
    cp_commit();
    for (int s = 0; s < nslab; ++s) {
        if (s + 1 < nslab) issue(s + 1, stg[(s + 1) & 1]);
        cp_commit();
        cp_wait1();
        __syncthreads();
        body(static_cast<const float *>(stg[s & 1]), s);
        __syncthreads();
    }
}

__device__ __forceinline__ float comp(const float4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// acc[r][j] += sum_k A[k][r0 + r] B[k][lane + 32 j] over a slab: A is [ks][64] (rows
// r0..r0 + 3 of row k in one 16-byte load), B is [ks][32 J].
template <int J>
__device__ __forceinline__ void mm_k4(float (&acc)[4][J], const float *A, int r0, const float *B, int ks)
{
    const int lane = threadIdx.x & 31;
#pragma unroll 4
    for (int k = 0; k < ks; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(A + k * CC + r0);
        float b[J];
#pragma unroll
        for (int j = 0; j < J; ++j) b[j] = B[k * 32 * J + lane + 32 * j];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) acc[r][j] = fmaf(comp(a, r), b[j], acc[r][j]);
    }
}

// acc[r][j] += sum_k A[row0 + r][k] B[k][lane + 32 j] over a slab: A is [rows][ks]
// (four k of a row in one 16-byte load), B is [ks][32 J]; ks % 4 == 0.
template <int R, int J>
__device__ __forceinline__ void mm_r4(float (&acc)[R][J], const float *A, int row0, const float *B, int ks)
{
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int k = 0; k < ks; k += 4) {
        float4 a[R];
#pragma unroll
        for (int r = 0; r < R; ++r) a[r] = *reinterpret_cast<const float4 *>(A + (row0 + r) * ks + k);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            float b[J];
#pragma unroll
            for (int j = 0; j < J; ++j) b[j] = B[(k + kk) * 32 * J + lane + 32 * j];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < J; ++j) acc[r][j] = fmaf(comp(a[r], kk), b[j], acc[r][j]);
        }
    }
}

// acc[r][j] += sum_{k in [k0, k1)} fa(r, k) fb(k, j): fa is the same for every lane of
// the warp (a broadcast), fb(k, j) reads column lane + 32 j of row k.
template <int R, int J, class FA, class FB>
__device__ __forceinline__ void mm(float (&acc)[R][J], int k0, int k1, FA fa, FB fb)
{
#pragma unroll 4
    for (int k = k0; k < k1; ++k) {
        float a[R], b[J];
#pragma unroll
        for (int r = 0; r < R; ++r) a[r] = fa(r, k);
#pragma unroll
        for (int j = 0; j < J; ++j) b[j] = fb(k, j);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < J; ++j) acc[r][j] = fmaf(a[r], b[j], acc[r][j]);
    }
}

__global__ void __launch_bounds__(CT, 1) bwdc_kernel(const BwdParams p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CSmem &sm = *reinterpret_cast<CSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *scr = p.scratch + (size_t)blockIdx.x * S_FLOATS;
    float *DO = scr + S_DO, *DOT = scr + S_DOT, *KGT = scr + S_KGT, *QGT = scr + S_QGT;
    float *KPT = scr + S_KPT, *YT = scr + S_YT, *UT = scr + S_UT;
    float *ring = &sm.stg[0][0];  // the operand ring as one [64][128] tile between products
    float *DU = scr + S_DU, *DY = scr + S_DY, *DYT = scr + S_DYT, *DKT = scr + S_DKT;
    float *DQT = scr + S_DQT, *DGT = scr + S_DGT, *DS = scr + S_DS, *PACC = scr + S_PACC;
    const int r0 = 4 * warp;  // rows of this warp in the 64-row products
    const int c0 = 8 * warp;  // rows (channels) of this warp in the 128-row products
    const int64_t units = p.N * p.H;
    const size_t rs = (size_t)p.H * kHead;  // row stride of the [tokens, H, 128] tensors
    const uint64_t once = evict_first_policy();

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t sq = u / p.H, h = u % p.H;
        const int64_t bos = p.cu ? p.cu[sq] : sq * p.T;
        int64_t len = p.cu ? p.cu[sq + 1] - bos : p.T;
        if (len < 0) len = 0;
        const int64_t nch = (len + CC - 1) / CC;
        const float ea = expf(p.A_log[h]);
        const float *ckb = p.ckpt + (size_t)((bos / CC + sq) * p.H + h) * ST;
        const size_t ckstride = (size_t)p.H * ST;
        const size_t st_off = (size_t)u * ST;
        const size_t hb = (size_t)h * kHead;

        __syncthreads();  // the previous unit's readers of dtb, the partials and DS are done
        if (tid < kHead) sm.dtb[tid] = p.dt_bias[h * kHead + tid];
        for (int i = tid; i < CW * (kHead + 1); i += CT) PACC[i] = 0.f;
        for (int i = tid; i < ST; i += CT) DS[i] = p.dfinal ? p.dfinal[st_off + i] : 0.f;
        __syncthreads();

        for (int64_t n = nch - 1; n >= 0; --n) {
            const int64_t tok = bos + n * CC;
            const int L = (int)(len - n * CC < CC ? len - n * CC : CC);
            const float *S0 = ckb + n * ckstride;

            // ---- 1. activations of the chunk's tokens (zero past L), dO ----
#pragma unroll 2
            for (int i = 0; i < CC / CW; ++i) {
                const int t = warp + CW * i;
                const bool in = t < L;
                const size_t row = (size_t)(tok + t) * rs + hb;
                // every load of the token first, so that they share one round trip
                float qv[4], kv[4], gv[4], dv[4], s2q = 0.f, s2k = 0.f;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int c = lane + 32 * m;
                    qv[m] = in ? bf_once(p.q, row + c, once) : 0.f;
                    kv[m] = in ? bf_once(p.k, row + c, once) : 0.f;
                    gv[m] = in ? bf(p.g, row + c) : 0.f;
                    dv[m] = in ? bf_once(p.dout, row + c, once) : 0.f;
                }
                const float braw = (in && lane == 0) ? bf_once(p.beta, (size_t)(tok + t) * p.H + h, once) : 0.f;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    s2q = fmaf(qv[m], qv[m], s2q);
                    s2k = fmaf(kv[m], kv[m], s2k);
                }
                const float rq = rsqrtf(wsum(s2q) + 1e-6f), rk = rsqrtf(wsum(s2k) + 1e-6f);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int c = lane + 32 * m;
                    float lam2 = 0.f;
                    if (in) {
                        const float x = gv[m] + sm.dtb[c];
                        const float sp = softplus_f(x);
                        lam2 = fmaxf(p.lower_bound, -ea * sp) * kL2e;
                    }
                    sm.QT[c][t] = qv[m] * rq;
                    sm.KT[c][t] = kv[m] * rk;
                    sm.GT[c][t] = lam2;
                    DO[t * kHead + c] = dv[m];
                    DOT[c * CC + t] = dv[m];
                }
                if (lane == 0) {
                    sm.b[t] = in ? sigmoid_f(braw) : 0.f;
                    sm.rq[t] = rq;
                    sm.rk[t] = rk;
                }
            }
            for (int i = tid; i < CC * LDT; i += CT) {
                (&sm.u.m.A[0][0])[i] = 0.f;
                (&sm.u.m.PT[0][0])[i] = 0.f;
            }
            if (n > 0) {
                // the next chunk's state towards L2 while this one computes (512 lines); the
                // input rows are read once, with the evict-first policy, and not prefetched
                // (prefetching them displaced scratch tiles: measured slower)
                const float *Sn = S0 - ckstride;  // 16384 floats: line tid of 512
                asm volatile("prefetch.global.L2 [%0];" ::"l"(Sn + 32 * tid));
            }
            __syncthreads();

            // ---- 2. G: inclusive cumulative sum over the chunk (log2 units) ----
            if (tid < kHead) {
                float run = 0.f;
                for (int t = 0; t < CC; ++t) {
                    run += sm.GT[tid][t];
                    sm.GT[tid][t] = run;
                }
                sm.G2L[tid] = sm.GT[tid][L - 1];
                sm.eGL[tid] = ex2f(sm.G2L[tid]);
            }
            __syncthreads();

            // ---- 3. (k^ Gam)^T, (q^ Gam)^T, K'^T; KS[c][j] = k^_j e^(G_e - G_j), e the last
            //      token of j's 16-token block (in the ring, for phase 4) ----
            {
                float *KS = ring;
                for (int e = tid; e < TILE; e += CT) {
                    const int c = e >> 6, t = e & (CC - 1);
                    const float g2 = sm.GT[c][t], gam = ex2f(g2), kh = sm.KT[c][t];
                    KGT[e] = kh * gam;
                    QGT[e] = sm.QT[c][t] * gam;
                    KPT[e] = kh * ex2f(sm.G2L[c] - g2);
                    KS[e] = kh * ex2f(sm.GT[c][t | 15] - g2);
                }
            }
            __syncthreads();

            // ---- 4. A and P: A_ij = sum_c (k^_i e^(G_i - G_e)) KS[c][j] with e the last token of
            //      j's block J (the first factor <= 1 past the block, <= e^75 inside it; KS in
            //      [e^-75, 1]).  Warp (J, rows i0..i0 + 31, half jq of the block): lane = row i,
            //      8 columns j each; 12 warps cover every (row, block J <= row's block) ----
            if (warp < 12) {
                const int jq = warp & 1, slot = warp >> 1;
                const int J = slot < 2 ? 0 : slot < 4 ? 1 : slot == 4 ? 2 : 3;
                const int i0 = slot == 0 ? 0 : slot == 1 ? 32 : slot == 2 ? 16 : slot == 3 ? 48 : slot == 4 ? 32 : 48;
                const int i = i0 + lane, jb = 16 * J + 8 * jq, eJ = 16 * J + 15;
                if (i < CC) {  // lanes past row 63 idle; no shuffles below
                    const float *KS = ring;
                    float a[8], pp[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) a[x] = pp[x] = 0.f;
#pragma unroll 4
                    for (int c = 0; c < kHead; ++c) {
                        const float rho = ex2f(sm.GT[c][i] - sm.GT[c][eJ]);
                        const float kr = sm.KT[c][i] * rho, qr = sm.QT[c][i] * rho;
#pragma unroll
                        for (int x = 0; x < 8; ++x) {
                            const float ks = KS[c * CC + jb + x];
                            a[x] = fmaf(kr, ks, a[x]);
                            pp[x] = fmaf(qr, ks, pp[x]);
                        }
                    }
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const int j = jb + x;
                        if (j < i) sm.u.m.A[i][j] = a[x];
                        if (j <= i) sm.u.m.PT[j][i] = pp[x];
                    }
                }
            }
            __syncthreads();

            // ---- 5. M^-1 = (I + Diag(b) A)^-1 by forward substitution: column 4 warp +
            //      lane / 8, rows j = s + 8 m held by lane s = lane % 8 ----
            {
                const int col = 4 * warp + (lane >> 3), s = lane & 7;
                float xr[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) xr[m] = 0.f;
#pragma unroll
                for (int i = 0; i < CC; ++i) {
                    float part = 0.f;
#pragma unroll
                    for (int m = 0; m < (i + 7) / 8; ++m) part = fmaf(sm.u.m.A[i][s + 8 * m], xr[m], part);
                    part += __shfl_xor_sync(FULL, part, 1);
                    part += __shfl_xor_sync(FULL, part, 2);
                    part += __shfl_xor_sync(FULL, part, 4);
                    const float xi = (i == col) ? 1.f : -sm.b[i] * part;
                    if (s == (i & 7)) xr[i >> 3] = xi;
                }
#pragma unroll
                for (int m = 0; m < 8; ++m) sm.u.m.Mi[s + 8 * m][col] = xr[m];
            }
            __syncthreads();

            // ---- 6. Y = v - (k^ Gam) S0 ----
            {
                float acc[4][4] = {};
                staged(sm.stg, kHead / 16,
                       [&](int s, float *buf) {
                           stage_rows(buf, KGT + s * 16 * CC, 16 * CC);                         // [16][64]
                           stage_rows(buf + 16 * CC, S0 + (size_t)s * 16 * kHead, 16 * kHead);  // [16][128]
                       },
                       [&](const float *buf, int) { mm_k4(acc, buf, r0, buf + 16 * CC, 16); });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int t = r0 + r, vc = lane + 32 * j;
                        const float vin = t < L ? bf_once(p.v, (size_t)(tok + t) * rs + hb + vc, once) : 0.f;
                        const float y = vin - acc[r][j];
                        ring[t * kHead + vc] = y;  // Y stays in the (now free) ring for phase 7
                        YT[vc * CC + t] = y;
                    }
            }
            __syncthreads();

            // ---- 7. U = M^-1 Diag(b) Y ----
            {
                float acc[4][4] = {};
                mm(acc, 0, r0 + 4, [&](int r, int j) { return sm.u.m.Mi[r0 + r][j] * sm.b[j]; },
                   [&](int j, int jj) { return ring[j * kHead + lane + 32 * jj]; });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int t = r0 + r, vc = lane + 32 * j;
                        UT[vc * CC + t] = acc[r][j];
                    }
            }
            __syncthreads();

            // ---- 8. dU = scale P^T dO + K' dS ----
            {
                float acc[4][4] = {};
                staged(sm.stg, CC / 16, [&](int s, float *buf) { stage_rows(buf, DO + s * 16 * kHead, 16 * kHead); },
                       [&](const float *buf, int s) {
                           const int k0 = 16 * s, lo = max(r0 - k0, 0);
                           mm(acc, lo, 16, [&](int r, int k) { return sm.u.m.PT[r0 + r][k0 + k]; },
                              [&](int k, int j) { return buf[k * kHead + lane + 32 * j]; });
                       });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[r][j] *= p.scale;
                staged(sm.stg, kHead / 16,
                       [&](int s, float *buf) {
                           stage_rows(buf, KPT + s * 16 * CC, 16 * CC);                 // [16][64]
                           stage_rows(buf + 16 * CC, DS + s * 16 * kHead, 16 * kHead);  // [16][128]
                       },
                       [&](const float *buf, int) { mm_k4(acc, buf, r0, buf + 16 * CC, 16); });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        DU[(r0 + r) * kHead + lane + 32 * j] = acc[r][j];  // for phase 10
                        ring[(r0 + r) * kHead + lane + 32 * j] = acc[r][j];  // for phase 9
                    }
            }
            __syncthreads();

            // ---- 9. dY = Diag(b) M^-T dU (= dv) ----
            {
                float acc[4][4] = {};
                mm(acc, r0, CC, [&](int r, int i) { return sm.u.m.Mi[i][r0 + r]; },
                   [&](int i, int j) { return ring[i * kHead + lane + 32 * j]; });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int t = r0 + r, vc = lane + 32 * j;
                        const float dy = sm.b[t] * acc[r][j];
                        DY[t * kHead + vc] = dy;
                        DYT[vc * CC + t] = dy;
                        if (t < L) p.dv[(size_t)(tok + t) * rs + hb + vc] = dy;
                    }
            }
            __syncthreads();

            // ---- 10. dT = dU Y^T, dP = scale dO U^T (lower parts); rowsum(dS o S0) e^GL ----
            {
                float aT[4][2] = {}, aP[4][2] = {};
                staged(sm.stg, kHead / 16,
                       [&](int s, float *buf) {
                           stage_cols(buf, DU, CC, kHead, 16 * s, 16);  // [64][16]
                           stage_cols(buf + 1024, DO, CC, kHead, 16 * s, 16);
                           stage_rows(buf + 2048, YT + s * 16 * CC, 16 * CC);  // [16][64]
                           stage_rows(buf + 3072, UT + s * 16 * CC, 16 * CC);
                       },
                       [&](const float *buf, int) {
                           mm_r4(aT, buf, r0, buf + 2048, 16);
                           mm_r4(aP, buf + 1024, r0, buf + 3072, 16);
                       });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int i = r0 + r, j = lane + 32 * jj;
                        sm.u.m.X[i][j] = j <= i ? aT[r][jj] : 0.f;
                        sm.u.m.dP[i][j] = j <= i ? p.scale * aP[r][jj] : 0.f;
                    }
#pragma unroll 4
                for (int rr = 0; rr < 8; ++rr) {
                    const int k = c0 + rr;
                    float s = 0.f;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int vc = lane + 32 * m;
                        s = fmaf(DS[k * kHead + vc], S0[(size_t)k * kHead + vc], s);
                    }
                    s = wsum(s);
                    if (lane == 0) sm.dGL[k] = sm.eGL[k] * s;
                }
            }

            // ---- 11. dK' = U dS^T, d(k^ Gam) = -dY S0^T, d(q^ Gam) = scale dO S0^T, as
            //      [channel][token] (rows c0.., columns lane + 32 jj) into dk^, dq^, dG ----
            {
                float acc[8][2] = {};
                staged(sm.stg, kHead / 16,
                       [&](int s, float *buf) {
                           stage_cols(buf, DS, kHead, kHead, 16 * s, 16);  // [128][16]
                           stage_rows(buf + 2048, UT + s * 16 * CC, 16 * CC);  // [16][64]
                       },
                       [&](const float *buf, int) { mm_r4(acc, buf, c0, buf + 2048, 16); });
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int c = c0 + r;
                    float cs = 0.f;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int t = lane + 32 * jj;
                        const float f = ex2f(sm.G2L[c] - sm.GT[c][t]);
                        const float kp = sm.KT[c][t] * f, d = acc[r][jj];
                        DKT[c * CC + t] = d * f;
                        DGT[c * CC + t] = -d * kp;
                        cs = fmaf(d, kp, cs);
                    }
                    cs = wsum(cs);
                    if (lane == 0) sm.extra[c] = cs;
                }
            }
            {
                float ak[8][2] = {}, aq[8][2] = {};
                staged(sm.stg, kHead / 16,
                       [&](int s, float *buf) {
                           stage_cols(buf, S0, kHead, kHead, 16 * s, 16);  // [128][16]
                           stage_rows(buf + 2048, DYT + s * 16 * CC, 16 * CC);  // [16][64]
                           stage_rows(buf + 3072, DOT + s * 16 * CC, 16 * CC);
                       },
                       [&](const float *buf, int) {
                           mm_r4(ak, buf, c0, buf + 2048, 16);
                           mm_r4(aq, buf, c0, buf + 3072, 16);
                       });
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int c = c0 + r, t = lane + 32 * jj, e = c * CC + t;
                        const float gam = ex2f(sm.GT[c][t]);
                        const float dkg = -ak[r][jj], dqg = p.scale * aq[r][jj];
                        DKT[e] += dkg * gam;
                        DQT[e] = dqg * gam;
                        DGT[e] += (dkg * sm.KT[c][t] + dqg * sm.QT[c][t]) * gam;
                    }
            }
            __syncthreads();

            // ---- 12. dS <- Diag(e^GL) dS + scale (q^ Gam)^T dO - (k^ Gam)^T dY ----
            {
                float acc[8][4] = {};
                float acc2[8][4] = {};  // (k^ Gam)^T dY, subtracted below
                staged(sm.stg, CC / 8,
                       [&](int s, float *buf) {
                           stage_cols(buf, QGT, kHead, CC, 8 * s, 8);  // [128][8]
                           stage_cols(buf + 1024, KGT, kHead, CC, 8 * s, 8);
                           stage_rows(buf + 2048, DO + s * 8 * kHead, 8 * kHead);  // [8][128]
                           stage_rows(buf + 3072, DY + s * 8 * kHead, 8 * kHead);
                       },
                       [&](const float *buf, int) {
                           mm_r4(acc, buf, c0, buf + 2048, 8);
                           mm_r4(acc2, buf + 1024, c0, buf + 3072, 8);
                       });
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int e = (c0 + r) * kHead + lane + 32 * j;
                        DS[e] = fmaf(sm.eGL[c0 + r], DS[e], fmaf(p.scale, acc[r][j], -acc2[r][j]));
                    }
            }

            // ---- 13. the solve's adjoint: db_j = sum_i dT_ij M^-1_ij; W = dM^-1 M^-T
            //      (into PT); dM = -M^-T W; dA = Diag(b) dM (strict lower, into X) ----
            if (tid < CC) {
                float s = 0.f;
                for (int i = tid; i < CC; ++i) s = fmaf(sm.u.m.X[i][tid], sm.u.m.Mi[i][tid], s);
                sm.db[tid] = s;
            }
            {
                float acc[4][2] = {};
                mm(acc, 0, r0 + 4, [&](int r, int k) { return sm.u.m.X[r0 + r][k] * sm.b[k]; },
                   [&](int k, int jj) { return sm.u.m.Mi[lane + 32 * jj][k]; });
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) sm.u.m.PT[r0 + r][lane + 32 * jj] = acc[r][jj];
            }
            __syncthreads();
            {
                float acc[4][2] = {};
                mm(acc, r0, CC, [&](int r, int k) { return sm.u.m.Mi[k][r0 + r]; },
                   [&](int k, int jj) { return sm.u.m.PT[k][lane + 32 * jj]; });
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int i = r0 + r;
                    float d2 = 0.f;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = lane + 32 * jj;
                        const float dm = -acc[r][jj];
                        const bool lo = j < i;
                        d2 += lo ? dm * sm.u.m.A[i][j] : 0.f;
                        sm.u.m.X[i][j] = lo ? sm.b[i] * dm : 0.f;
                    }
                    d2 = wsum(d2);
                    if (lane == 0) sm.db[i] += d2;
                }
            }
            __syncthreads();

            // ---- 14. adjoints of the decay-weighted products, per (channel, token), with the
            //      factor e^(G_i - G_j) split at a reference token of a 16-token block so
            //      that the exponentials are per (channel, token) instead of per pair.
            //      Row side (sums over j <= i), reference e = the last token of j's block:
            //        e^(G_i - G_j) = e^(G_i - G_e) e^(G_e - G_j), the second factor in
            //        [e^-75, 1], the first <= e^75 (it underflows only where the product is
            //        below e^-87).  KS[c][j] = k^_j e^(G_e - G_j) sits in the operand ring.
            {
                float *KS = &sm.stg[0][0];
                for (int e = tid; e < TILE; e += CT) {
                    const int c = e >> 6, j = e & (CC - 1);
                    KS[e] = sm.KT[c][j] * ex2f(sm.GT[c][j | 15] - sm.GT[c][j]);
                }
                __syncthreads();
#pragma unroll 1
                for (int rg = 0; rg < 2; ++rg) {
                    const int cr = c0 + 4 * rg;
                    float ta[4][2] = {}, tp[4][2] = {};
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        // tokens i = lane + 32 jj: blocks J >= 2 hold only j > i for jj = 0
                        float pa[4][2] = {}, pp[4][2] = {};
#pragma unroll 4
                        for (int j = 16 * J; j < 16 * J + 16; ++j) {
                            float dA_[2], dP_[2];
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                dA_[jj] = (J < 2 || jj == 1) ? sm.u.m.X[lane + 32 * jj][j] : 0.f;
                                dP_[jj] = (J < 2 || jj == 1) ? sm.u.m.dP[lane + 32 * jj][j] : 0.f;
                            }
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const float ks = KS[(cr + r) * CC + j];
#pragma unroll
                                for (int jj = 0; jj < 2; ++jj) {
                                    if (J >= 2 && jj == 0) continue;
                                    pa[r][jj] = fmaf(dA_[jj], ks, pa[r][jj]);
                                    pp[r][jj] = fmaf(dP_[jj], ks, pp[r][jj]);
                                }
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r)
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                if (J >= 2 && jj == 0) continue;
                                const int c = cr + r, i = lane + 32 * jj;
                                // blocks past i contribute 0; the clamp keeps their factor finite
                                const float rho = ex2f(fminf(sm.GT[c][i] - sm.GT[c][16 * J + 15], 120.f));
                                ta[r][jj] = fmaf(rho, pa[r][jj], ta[r][jj]);
                                tp[r][jj] = fmaf(rho, pp[r][jj], tp[r][jj]);
                            }
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int c = cr + r, t = lane + 32 * jj, e = c * CC + t;
                            DKT[e] += ta[r][jj];
                            DQT[e] += tp[r][jj];
                            DGT[e] += sm.KT[c][t] * ta[r][jj] + sm.QT[c][t] * tp[r][jj];
                        }
                }
            }
            __syncthreads();
            {
                //      Column side (sums over i >= j), reference s = the first token of i's
                //      block: e^(G_i - G_j) = e^(G_i - G_s) e^(G_s - G_j), the first factor
                //      in [e^-75, 1], the second <= e^75 (it underflows only where the
                //      product is below e^-87).  R[c][i] = e^(G_i - G_s) in the ring.
                float *R = &sm.stg[0][0];
                for (int e = tid; e < TILE; e += CT) {
                    const int c = e >> 6, i = e & (CC - 1);
                    R[e] = ex2f(sm.GT[c][i] - sm.GT[c][i & ~15]);
                }
                __syncthreads();
#pragma unroll 1
                for (int rg = 0; rg < 2; ++rg) {
                    const int cr = c0 + 4 * rg;
                    float ta[4][2] = {};
#pragma unroll
                    for (int I = 0; I < 4; ++I) {
                        // tokens j = lane + 32 jj: blocks I < 2 hold only i < j for jj = 1
                        float pa[4][2] = {};
#pragma unroll 4
                        for (int i = 16 * I; i < 16 * I + 16; ++i) {
                            float dA_[2], dP_[2];
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                dA_[jj] = (I >= 2 || jj == 0) ? sm.u.m.X[i][lane + 32 * jj] : 0.f;
                                dP_[jj] = (I >= 2 || jj == 0) ? sm.u.m.dP[i][lane + 32 * jj] : 0.f;
                            }
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const int c = cr + r;
                                const float kq = sm.KT[c][i], qq = sm.QT[c][i], rr = R[c * CC + i];
#pragma unroll
                                for (int jj = 0; jj < 2; ++jj) {
                                    if (I < 2 && jj == 1) continue;
                                    pa[r][jj] = fmaf(fmaf(dA_[jj], kq, dP_[jj] * qq), rr, pa[r][jj]);
                                }
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r)
#pragma unroll
                            for (int jj = 0; jj < 2; ++jj) {
                                if (I < 2 && jj == 1) continue;
                                const int c = cr + r, j = lane + 32 * jj;
                                // blocks before j contribute 0; the clamp keeps their factor finite
                                const float sig = ex2f(fminf(sm.GT[c][16 * I] - sm.GT[c][j], 120.f));
                                ta[r][jj] = fmaf(sig, pa[r][jj], ta[r][jj]);
                            }
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int c = cr + r, t = lane + 32 * jj, e = c * CC + t;
                            DKT[e] += ta[r][jj];
                            DGT[e] -= sm.KT[c][t] * ta[r][jj];
                        }
                }
            }
            __syncthreads();

            // ---- 15. epilogue: dG[L-1] terms, dlam, norms, sigmoid and gate ----
            if (tid < kHead) DGT[tid * CC + L - 1] += sm.extra[tid] + sm.dGL[tid];
            __syncthreads();
            {
                float pq[2] = {0.f, 0.f}, pk[2] = {0.f, 0.f};
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int c = c0 + r;
                    // reverse cumulative sum over the chunk's tokens: lane holds t = lane, lane + 32
                    float s0 = DGT[c * CC + lane], s1 = DGT[c * CC + lane + 32];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float y0 = __shfl_down_sync(FULL, s0, o), y1 = __shfl_down_sync(FULL, s1, o);
                        if (lane + o < 32) {
                            s0 += y0;
                            s1 += y1;
                        }
                    }
                    s0 += __shfl_sync(FULL, s1, 0);
                    sm.u.e.o0[lane][c] = s0;
                    sm.u.e.o0[lane + 32][c] = s1;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int t = lane + 32 * jj;
                        pq[jj] = fmaf(sm.QT[c][t], DQT[c * CC + t], pq[jj]);
                        pk[jj] = fmaf(sm.KT[c][t], DKT[c * CC + t], pk[jj]);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    sm.u.e.red[0][warp][lane + 32 * jj] = pq[jj];
                    sm.u.e.red[1][warp][lane + 32 * jj] = pk[jj];
                }
            }
            __syncthreads();
            if (tid < 2 * CC) {
                const int a = tid >> 6, t = tid & (CC - 1);
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < CW; ++w) s += sm.u.e.red[a][w][t];
                sm.u.e.red[a][0][t] = s;
            }
            __syncthreads();
#pragma unroll 1
            for (int a = 0; a < 2; ++a) {  // a = 0: dq, a = 1: dk
                const float *DXT = a ? DKT : DQT;
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int c = c0 + r, t = lane + 32 * jj;
                        const float xh = a ? sm.KT[c][t] : sm.QT[c][t];
                        const float rn = a ? sm.rk[t] : sm.rq[t];
                        sm.u.e.o1[t][c] = rn * (DXT[c * CC + t] - xh * sm.u.e.red[a][0][t]);
                    }
                __syncthreads();
                float *dst = a ? p.dk : p.dq;
#pragma unroll 1
                for (int i = 0; i < CC / CW; ++i) {
                    const int t = warp + CW * i;
                    if (t < L) {
                        const size_t row = (size_t)(tok + t) * rs + hb;
#pragma unroll
                        for (int m = 0; m < 4; ++m) dst[row + lane + 32 * m] = sm.u.e.o1[t][lane + 32 * m];
                    }
                }
                __syncthreads();
            }
            {
                float da = 0.f, dxs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < CC / CW; ++i) {
                    const int t = warp + CW * i;
                    if (t >= L) continue;
                    const size_t row = (size_t)(tok + t) * rs + hb;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int c = lane + 32 * m;
                        const float x = bf_once(p.g, row + c, once) + sm.dtb[c];
                        const float z = -ea * softplus_f(x);
                        const bool open = z >= p.lower_bound;  // the clamp is not holding
                        const float dl = sm.u.e.o0[t][c];
                        const float dx = open ? -dl * ea * sigmoid_f(x) : 0.f;
                        p.dg[row + c] = dx;
                        dxs[m] += dx;
                        da += open ? dl * z : 0.f;
                    }
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) PACC[warp * (kHead + 1) + lane + 32 * m] += dxs[m];
                da = wsum(da);
                if (lane == 0) PACC[warp * (kHead + 1) + kHead] += da;
                if (tid < L) {
                    const float bt = sm.b[tid];
                    p.dbeta[(size_t)(tok + tid) * p.H + h] = sm.db[tid] * bt * (1.f - bt);
                }
            }
            __syncthreads();
        }

        // ---- dL/dS_0 and the unit's parameter partials ----
        if (p.dinit)
            for (int i = tid; i < ST; i += CT) p.dinit[st_off + i] = DS[i];
        __syncthreads();
        if (tid <= kHead) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < CW; ++w) acc += PACC[w * (kHead + 1) + tid];
            p.part[(size_t)u * (kHead + 1) + tid] = acc;
        }
    }
}

std::atomic<int> g_bwd_mode{KDA_BWD_CHUNKED};

}  // namespace

size_t bwd_chunked_scratch_bytes_per_cta() { return (size_t)S_FLOATS * sizeof(float); }

int bwd_set_schedule(int mode)
{
    if (mode != KDA_BWD_CHUNKED && mode != KDA_BWD_TOKEN) return KDA_ERR_ARG;
    return g_bwd_mode.exchange(mode);
}

int launch_backward(const BwdParams &p, const BwdLayout &l, cudaStream_t stream)
{
    if (g_bwd_mode.load() == KDA_BWD_TOKEN) return launch_backward_token(p, l, stream);
    const int64_t units = p.N * p.H;
    if (units <= 0) return 0;
    int launches = 0;
    if (p.B * p.T > 0) {  // the states before every chunk (no chunks: nothing to store)
        FwdParams f{};
        f.q = p.q;
        f.k = p.k;
        f.v = p.v;
        f.g = p.g;
        f.beta = p.beta;
        f.A_log = p.A_log;
        f.dt_bias = p.dt_bias;
        f.init = p.init;
        f.init_dtype = p.init_dtype;
        f.final_state = nullptr;
        f.final_dtype = KDA_STATE_F32;
        f.state_layout = KDA_LAYOUT_KV;
        f.cu = p.cu;
        f.out = nullptr;
        f.scale = p.scale;
        f.lower_bound = p.lower_bound;
        f.B = p.B;
        f.T = p.T;
        f.H = p.H;
        f.N = p.N;
        f.ckpt = p.ckpt;
        const int n = launch_chunked(f, stream);
        if (n < 0) return n;
        launches += n;
    }
    static int smem_set[64];
    const int smem = (int)sizeof(CSmem);
    if (!set_smem_limit_once(bwdc_kernel, smem, smem_set)) return KDA_ERR_CUDA;
    bwdc_kernel<<<l.grid, CT, smem, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    const int n = launch_param_reduce(p, stream);
    return n < 0 ? n : launches + 1 + n;
}

}  // namespace kda
