// Chunked KDA forward kernel for sm_100a (B200): tcgen05 tensor cores, TMEM, TMA.
//
// Operator: Kimi Delta Attention, the gated delta rule with channel-wise decay
// described on the FlashKDA pages (7minutos.es, "¿Qué es la atención Kimi
// Delta...?"; chunk_kda flags on github.zuobiaodaohang.com "FlashKDA：用CUTLASS
// fused kernel 给 Kimi Delta Attention 提速 3-5 倍", section "作为 FLA 后端的用法").
//
// One CTA per (sequence, head), two warp roles working one chunk apart: warps
// 0..7 prepare chunk n+1 (activations, intra-chunk products, triangular solve)
// while warps 8..11 run the sequential state pass over chunk n.  Tokens are
// processed in chunks of C = 64.  For a
// chunk starting from state S0 (K x V), with q^, k^ L2-normalised, b = sigmoid(beta),
// lam = clamped log-decay and G the inclusive in-chunk cumulative sum of lam:
//   A_ij = sum_c k^_i k^_j e^{G_i - G_j}   (j <  i)      decay-weighted k k^T
//   P_ij = sum_c q^_i k^_j e^{G_i - G_j}   (j <= i)      masked q k^T
//   T    = (I + Diag(b) A)^-1 Diag(b)                   unit-triangular solve (WY/UT form)
//   w    = T (k^ e^G),  u = T v
//   U    = u - w S0
//   O    = scale [(q^ e^G) S0 + P U]
//   S    = Diag(e^{G_last}) S0 + (k^ e^{G_last - G})^T U
// (derivation: unrolling S_t = Diag(a_t) S_{t-1} + k^_t u_t^T with
//  u_t = b_t (v_t - S'_t^T k^_t) inside the chunk).
//
// Decay factors: with lam >= -5, e^{G_i - G_j} over 64 tokens spans e^{-320}, so
// A and P are formed in two 32-token blocks, each with a reference token r at its
// middle: k^_i e^{G_i - G_r} and k^_j e^{G_r - G_j} stay within e^{+-80} (fp32
// range), and the cross-block part uses the second block's reference for the
// first block's columns.  These products run in tf32; the rest in fp16 (bounded
// operands) or bf16 (the raw v tile with T split into a bf16 hi + lo pair).  The
// state operand S and U are scaled by a power of two per value column before
// the fp16 cast; the state itself stays fp32 in TMEM, stored divided by the
// current power-of-two scale of U so that the state update accumulates in place.
//
// Orientation: the inter-chunk products are computed transposed (M = value
// column v on the 128 TMEM lanes), so S^T and U^T are tensor-core A operands
// read straight from TMEM, and thread v owns value column v.
//
// Launches of long units (>= 1024 tokens on average) run an instantiation in which the
// state warps, idle part of each chunk, also compute the round-1 gate of the chunk
// after next and hand it to the in-chunk warps through TMEM.
//
// Split schedule (few units, many idle SMs): a cluster of 4 CTAs per (sequence,
// head).  CTAs 1..3 each run the in-chunk work for every third chunk and send its
// results ([w ; q^ e^G], k', P, gamma by a bulk copy, u^T by stores) into one of two
// slots in CTA 0's shared memory; CTA 0 runs only the state pass, consuming the
// chunks in order and handing each slot back to the CTA that fills it next.
#include <atomic>
#include <cuda.h>

#include <type_traits>

#include "kda.h"
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {

// Error word: (launch epoch << 8) | code of the first bounded wait that gave up (0 = none).
// A CTA that starts after another CTA of its launch gave up sees its own epoch there and
// returns at once, so a failure that hits every CTA ends after one wave of them; a stale
// word of an earlier launch carries another epoch and is ignored.
__device__ int g_chunk_error;
__shared__ uint32_t s_epoch;  // this launch's epoch (the high bits of its error word)
__shared__ int s_abort;       // set by thread 0: this launch has already failed

namespace {

using namespace sm100;

constexpr int C = 64;        // chunk length
constexpr int NT_IN = 256;   // in-chunk warpgroups: warps 0..7
constexpr int NT_ST = 128;   // state warpgroup: warps 8..11 (thread v <-> TMEM lane v)
constexpr int NT_MMA = 32;   // tensor-core issue warp for the in-chunk products: warp 12
constexpr int NT = NT_IN + NT_ST + NT_MMA;
constexpr uint32_t BAR_IN = 1, BAR_ST = 2;  // named barriers of the two roles
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kLptMax = 128;  // varlen batches up to this many sequences run longest first

// ---- shared memory (byte offsets from a 1024-byte aligned base) ----
// q, k, g, v tiles arrive by TMA as 2 boxes of [64 tokens][64 channels] bf16 with
// the 128-byte swizzle (box b holds channels 64b..64b+63).
constexpr uint32_t SM_Q = 0;                // 16 KB
constexpr uint32_t SM_K = 16 * 1024;        // 16 KB
constexpr uint32_t SM_G = 32 * 1024;        // 16 KB
constexpr uint32_t SM_V = 48 * 1024;        // 16 KB
// A/P operands for one half of the channels (the product runs in two K rounds):
constexpr uint32_t SM_APA = 64 * 1024;      // 32 KB  [k^ rho ; q^ rho] tf32, K-major [128][64]
constexpr uint32_t SM_APB = 96 * 1024;      // 32 KB  [k^ sig ; k^ e^{G_47-G}] tf32, K-major [96(+32 pad)][64]
//   reused once the A/P product has completed (solve):
constexpr uint32_t SM_X = SM_APA;                 // fp32 [64][LST] X = (I + Diag(b) A)^-1
constexpr uint32_t SM_L = SM_APA + 17 * 1024;     // fp32 [64][LST] Diag(b) A (strict lower)
constexpr uint32_t SM_Y = SM_APA + 34 * 1024;     // fp32 3 x [16][16] block products
constexpr uint32_t SM_T16 = SM_APA + 17 * 1024;   // 8 KB fp16 T, K-major [64 i][64 j] (over L)
constexpr uint32_t SM_THI = SM_APA + 25 * 1024;   // 8 KB bf16 high part of T
constexpr uint32_t SM_TLO = SM_APA + 33 * 1024;   // 8 KB bf16 low part of T
constexpr uint32_t SM_KG = 128 * 1024;      // 16 KB  k^ e^G fp16, MN-major (M = channel, K = token)
// handed to the state warpgroup:
constexpr uint32_t SM_WQ = 144 * 1024;      // 32 KB  [w ; q^ e^G] fp16, K-major [128][128]
constexpr uint32_t SM_KP0 = 176 * 1024;     // 16 KB  k' = k^ e^{G_last - G} fp16, MN-major (K = token),
constexpr uint32_t SM_KP1 = 200 * 1024;     // 16 KB    two buffers by chunk parity
constexpr uint32_t SM_P = 192 * 1024;       // 8 KB   P fp16, K-major [64 i][64 j]
constexpr uint32_t SM_MISC = 216 * 1024;    // norms, beta, gamma x2, octant sums, barriers
constexpr uint32_t SM_BYTES = 224 * 1024;
constexpr uint32_t SMEM_ALLOC = SM_BYTES + 1024;  // + alignment slack
constexpr int LST = 68;                     // row stride (floats) of the solve matrices

// ---- tensor memory columns (512 allocated) ----
constexpr uint32_t TM_AP = 0;    // A/P product, lanes = rows, 96 cols        (in-chunk role)
constexpr uint32_t TM_W = 0;     // w^T: lanes = channel, cols = token (64)   (aliases AP)
constexpr uint32_t TM_G = 96;    // round-1 gate G of the in-chunk threads (32) (state -> in-chunk)
constexpr int64_t kGateHandoffTokens = 1024;  // mean tokens per unit from which it is used
constexpr uint32_t TM_S = 128;   // state S / tau, lane v, column k  (128)    (state role)
constexpr uint32_t TM_D1 = 256;  // [w S~^T | (q^ e^G) S~^T] per lane v (128); cols 0..31
                                 //   then hold U~^T (fp16 pairs)
constexpr uint32_t TM_D3 = 384;  // (P U~)^T per lane v (64)
constexpr uint32_t TM_SS = 384;  // S~^T fp16 pairs (A operand), 64 cols      (aliases D3)
constexpr uint32_t TM_U = 448;   // u^T: lanes = v, cols = token (64)         (in-chunk -> state)

// ---- schedules: every role runs in the fused kernel (one CTA per unit) or on one side
//      of the split kernel (in-chunk work on CTAs 1..3, the state pass on CTA 0) ----
enum Mode { kFused = 0, kProducer = 1, kConsumer = 2 };
constexpr int kSplitCta = 4;       // CTAs per unit in the split kernel
constexpr int kProducers = kSplitCta - 1;
// CTA 0's two slots (byte offsets within a slot of SLOT_BYTES, 1024-aligned parts first)
constexpr uint32_t SL_WQ = 0;              // 32 KB [w ; q^ e^G] fp16, as SM_WQ
constexpr uint32_t SL_KP = 32 * 1024;      // 16 KB k' fp16, as SM_KP0
constexpr uint32_t SL_P = 48 * 1024;       // 8 KB  P fp16, as SM_P
constexpr uint32_t SL_U = 56 * 1024;       // u^T fp32, row v at SL_U + v * SL_UROW
constexpr uint32_t SL_UROW = 272;          // 64 floats + 16 bytes: rows start in rotating banks
constexpr uint32_t SL_GAM = SL_U + 128 * SL_UROW;  // 512 B gamma
constexpr uint32_t SLOT_BYTES = ((SL_GAM + 512 + 1023) / 1024) * 1024;
constexpr uint32_t SL_BARS = 2 * SLOT_BYTES;       // consumer barriers
constexpr uint32_t kSendBytes = 32768 + 16384 + 8192 + 512;  // bulk bytes per chunk
static_assert(SL_BARS + 256 <= 224 * 1024, "two slots fit the shared memory");

__device__ __forceinline__ uint32_t sw(uint32_t row, uint32_t colbyte) { return sw128_offset(row, colbyte); }

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float2 bf2x2(uint32_t w)
{
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
}

// 2^x and log2(x) on the special-function unit; results below 2^-126 flush to zero
// (every such factor here scales terms that are negligible at fp32 precision).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp32 -> tf32 with round-half-away-from-zero: the tensor core reads the upper
// 19 bits of each 32-bit operand, so adding half a tf32 ulp first rounds.
__device__ __forceinline__ uint32_t tf32b(float x) { return __float_as_uint(x) + 0x1000u; }

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void st_u32(uint8_t *base, uint32_t off, uint32_t x)
{
    *reinterpret_cast<uint32_t *>(base + off) = x;
}

__device__ __forceinline__ void st_u64(uint8_t *base, uint32_t off, uint32_t lo, uint32_t hi)
{
    *reinterpret_cast<uint2 *>(base + off) = make_uint2(lo, hi);
}

// Power of two s >= max|x| (1 for zero): the fp16 operand x / s lies in [-1, 1].
__device__ __forceinline__ float pow2_ceil(float m)
{
    if (!(m > 0.f)) return 1.f;
    const uint32_t e = (__float_as_uint(m) >> 23) & 0xFF;  // m in [2^(e-127), 2^(e-126))
    return __uint_as_float(min(e + 1u, 254u) << 23);
}

struct Bars {
    uint64_t qkg[2];   // TMA q, k, g 64-channel box b         (tx bytes)
    uint64_t v;        // TMA v tile                           (tx bytes)
    uint64_t mma_in;   // in-chunk role's tensor-core work     (commit)
    uint64_t mma_st;   // state role's tensor-core work        (commit)
    uint64_t full;     // chunk operands ready for the state role (1 arrival)
    uint64_t wq_free;  // [w ; q^ e^G] consumed                (commit)
    uint64_t kp_free[2];  // k' buffer b, gamma slot b and P consumed (commit after the
                          // state role's second product of a chunk of parity b)
    uint64_t u_free;   // u^T read out of TMEM                 (128 arrivals)
    uint64_t ops;      // operands of the next in-chunk product written (one arrival per
                       // in-chunk warp); the issue warp waits on it
    uint64_t gate_rdy;  // fused: chunk n's round-1 gate (n >= 2) is in TM_G   (1 arrival)
    uint64_t gate_free; // fused: TM_G and the round-1 octant sums read   (one arrival per in-chunk warp)
    // split kernel, CTAs 1..3:
    uint64_t u_rdy;     // u^T of the chunk complete in TMEM              (commit)
    uint64_t slot_free; // CTA 0 released the slot this CTA fills next    (1 remote arrival)
};

// Split kernel, CTA 0: slot s holds a chunk once its bulk bytes, its 128 u^T rows and
// CTA 0's own re-arming arrival (which sets the expected bytes) are all in.
struct SlotBars {
    uint64_t full[2];
    uint64_t mma_st;
};

struct TMaps {
    CUtensorMap q, k, g, v;  // 2-D [tokens][H*128] bf16, box [64][64], 128-byte swizzle
};

struct Ctx {
    uint8_t *sm;
    float *rkq_s /* [2][64][2] */, *b_s /* [2][64] */, *gam_s /* [2][128] */, *osum /* [8][128] */,
        *dtb_s /* [128] */;  // [2] = by chunk parity
    Bars *bars;
    uint32_t tb;  // TMEM base
    int64_t h, H, tok0, len, rstride;
    int64_t unit;  // (sequence, head) unit = sequence * H + head
    int nchunks;
    // split kernel: this CTA's chunks are first, first + kProducers, ... (CTAs 1..3);
    // CTA 0's slot base and slot barriers as shared::cluster addresses
    int first;
    uint32_t c_slots, c_full;
};

// The same for a barrier completed by other CTAs of the cluster (acquire at cluster scope).
__device__ __forceinline__ bool wait_or_flag_cluster(uint64_t *bar, uint32_t parity, int code);

// Bounded wait (about 1 s at 1965 MHz); one that gives up records (epoch << 8) | code
// unless an earlier failure of the launch is already recorded.  The spin itself stays
// minimal: extra work in this inlined loop, which sits at every hand-off, measurably
// slowed the kernel.
__device__ __forceinline__ bool wait_or_flag(uint64_t *bar, uint32_t parity, int code)
{
    if (mbar_wait(bar, parity, 2000000000LL)) return true;
    atomicCAS(&g_chunk_error, 0, (int)(s_epoch << 8) | code);
    return false;
}

__device__ __forceinline__ bool wait_or_flag_cluster(uint64_t *bar, uint32_t parity, int code)
{
    if (mbar_wait_cluster(bar, parity, 2000000000LL)) return true;
    atomicCAS(&g_chunk_error, 0, (int)(s_epoch << 8) | code);
    return false;
}

// q, k and g box b (channels 64b..64b+63) of the chunk starting at token tok
__device__ __forceinline__ void load_qkg_box(uint8_t *sm, const TMaps &tm, uint64_t *bar, int64_t h,
                                             int64_t tok, int b)
{
    mbar_arrive_expect_tx(bar, 3 * 8192);
    const int32_t x = (int32_t)(h * kHead + 64 * b), y = (int32_t)tok;
    tma_load_2d(sm + SM_Q + 8192 * b, &tm.q, bar, x, y);
    tma_load_2d(sm + SM_K + 8192 * b, &tm.k, bar, x, y);
    tma_load_2d(sm + SM_G + 8192 * b, &tm.g, bar, x, y);
}

__device__ __forceinline__ void load_tile(uint8_t *dst, const CUtensorMap *tm, uint64_t *bar,
                                          int64_t h, int64_t tok)
{
    tma_load_2d(dst, tm, bar, (int32_t)(h * kHead), (int32_t)tok);
    tma_load_2d(dst + 8192, tm, bar, (int32_t)(h * kHead + 64), (int32_t)tok);
}

// =====================================================================================
// In-chunk role (warps 0..7): for every chunk, the per-token activations, the
// decay-weighted products A and P (tf32), the triangular solve for T, and the
// products w = T (k^ e^G), u = T v; hands [w ; q^ e^G], k', P, u^T and gamma over.
// =====================================================================================
template <Mode M, bool GH = false>
__device__ void in_chunk_role(const FwdParams &p, const TMaps &tm, const Ctx &cx)
{
    uint8_t *sm = cx.sm;
    Bars *bars = cx.bars;
    const uint32_t tb = cx.tb;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ln = tid & 127, hf = tid >> 7;
    const uint32_t lq = (uint32_t)((warp & 3) * 32) << 16;
    float *Lm = reinterpret_cast<float *>(sm + SM_L);
    float *Xm = reinterpret_cast<float *>(sm + SM_X);
    const int64_t H = cx.H, h = cx.h;
    // log-decay in log2 units: lam2 = max(lb log2e, -A log2e max(x,0) - A lg2(1 + 2^(-|x| log2e)))
    const float aexp = (cx.len > 0) ? ex2(p.A_log[h] * kLog2e) : 0.f;
    const float a2 = aexp * kLog2e, lb2 = p.lower_bound * kLog2e;
    uint32_t mma_cnt = 0;  // completed phases of bars->mma_in waited on so far
    bool ok = true;
    // The role's own chunks: all of the unit's (fused), or every kProducers-th from
    // cx.first (split kernel); n counts own chunks (the phases of the local barriers),
    // uc(n) is the chunk of the unit.
    constexpr int S = (M == kProducer) ? kProducers : 1;
    const int f = (M == kProducer) ? cx.first : 0;
    auto uc = [&](int n) { return f + S * n; };
    const int nown = cx.nchunks > f ? (cx.nchunks - f + S - 1) / S : 0;
    bool sent_ok = true;  // split kernel, thread 0: the last hand-off's slot wait

    // Channel-pass thread mapping: channel pair 2cp, 2cp+1 (of each 64-channel round),
    // token octant oc (tokens 8oc..8oc+7; their rows have row % 8 == j).  Swizzled byte
    // offsets of the pair in row 8oc + j, precomputed once:
    //   o16[j]: 16-bit tiles and fp16 operands (column byte 4cp within a 128-byte row)
    //   o32[j]: tf32 operands (column byte 8 (cp % 16) within the atom (cp / 16))
    const int cp = lane, oc = warp, t0 = oc * 8, blk = oc >> 2;
    uint32_t o16[8], o32[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        o16[j] = sw((uint32_t)(t0 + j), (uint32_t)cp * 4u);
        o32[j] = (uint32_t)(cp >> 4) * 16384u + sw((uint32_t)(t0 + j), (uint32_t)(cp & 15) * 8u);
    }

    // beta logits are read one chunk ahead as raw bf16 bits (thread t < 64 holds token t
    // of the chunk after the one being prepared); converting them only when that chunk
    // starts keeps the global load off the critical path
    const uint16_t *beta_g = reinterpret_cast<const uint16_t *>(p.beta);
    uint16_t beta_bits = 0;
    auto chunk_len = [&](int m) {
        const int64_t rem = cx.len - (int64_t)m * C;
        return (int)(rem < C ? rem : C);
    };
    auto load_beta = [&](int m) {  // raw beta of chunk m (zero past the sequence end)
        beta_bits = 0;
        if (tid < C && m < cx.nchunks && (int64_t)m * C + tid < cx.len)
            beta_bits = beta_g[(cx.tok0 + (int64_t)m * C + tid) * H + h];
    };

    // ---- norms (thread: token tid/4, 16-byte chunks 2 (tid%4), 2 (tid%4) + 1 of both
    //      64-channel boxes; each 8-lane phase then reads 8 distinct bank groups) and beta
    //      of the chunk whose tiles are in shared memory, of length Lc, into buffer buf.
    //      A partial chunk's tiles also hold the rows after the sequence (the next
    //      sequence's tokens, or whatever follows the batch); those tokens must add
    //      exactly zero whatever their bits (0 * NaN is NaN), so the threads that own
    //      their q and k chunks here overwrite them with zeros before any other read. ----
    auto norms = [&](int Lc, int buf) {
        const float beta_c = __uint_as_float((uint32_t)beta_bits << 16);
        const int t = tid >> 2, qq = tid & 3;
        if (t >= Lc) {  // a row after the sequence end: cleared, whatever its bits
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const uint32_t off = (uint32_t)(ch >> 1) * 8192u + sw(t, (2 * qq + (ch & 1)) * 16);
                *reinterpret_cast<uint4 *>(sm + SM_Q + off) = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(sm + SM_K + off) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            const uint32_t off = (uint32_t)(ch >> 1) * 8192u + sw(t, (2 * qq + (ch & 1)) * 16);
            const uint4 qr = *reinterpret_cast<const uint4 *>(sm + SM_Q + off);
            const uint4 kr = *reinterpret_cast<const uint4 *>(sm + SM_K + off);
            const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w}, kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 qf = bf2x2(qw[e]), kf = bf2x2(kw[e]);
                sq += qf.x * qf.x + qf.y * qf.y;
                sk += kf.x * kf.x + kf.y * kf.y;
            }
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sk += __shfl_xor_sync(0xffffffffu, sk, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        sk += __shfl_xor_sync(0xffffffffu, sk, 2);
        if (qq == 0)  // (1/|k|, 1/|q|) per token, zero past the chunk end
            *reinterpret_cast<float2 *>(cx.rkq_s + buf * 128 + 2 * t) =
                (t < Lc) ? make_float2(rsqrtf(sk + 1e-6f), rsqrtf(sq + 1e-6f)) : make_float2(0.f, 0.f);
        if (tid < C) cx.b_s[buf * 64 + tid] = (tid < Lc) ? __fdividef(1.f, 1.f + ex2(-beta_c * kLog2e)) : 0.f;
    };

    // ---- gate of one 64-channel round: in-octant cumulative log2-decay of the pair
    //      (tokens t0 .. t0+7) and the octant sums for the prefix ----
    auto gate_round = [&](int round, int Lc, float2 (&Gq)[8]) {
        const int c0 = 64 * round + 2 * cp;
        const uint32_t rb = (uint32_t)round * 8192u;
        const float2 dtb = *reinterpret_cast<const float2 *>(cx.dtb_s + c0);
        float2 run = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // branch-free: tokens past the chunk end read finite tile data and get lam = 0
            const float2 g2 = bf2x2(*reinterpret_cast<const uint32_t *>(sm + SM_G + rb + o16[j]));
            const float x0 = g2.x + dtb.x, x1 = g2.y + dtb.y;
            const float e0 = lg2(1.f + ex2(-fabsf(x0) * kLog2e));
            const float e1 = lg2(1.f + ex2(-fabsf(x1) * kLog2e));
            const bool valid = t0 + j < Lc;
            run.x += valid ? fmaxf(lb2, -a2 * fmaxf(x0, 0.f) - aexp * e0) : 0.f;
            run.y += valid ? fmaxf(lb2, -a2 * fmaxf(x1, 0.f) - aexp * e1) : 0.f;
            Gq[j] = run;
        }
        *reinterpret_cast<float2 *>(cx.osum + oc * 128 + c0) = run;
    };

    // Chunk 0's norms and round-0 gate run here.  For chunk n+1, the round-0 gate runs
    // while chunk n's second A/P product is on the tensor cores and the norms while its
    // w/u products are (the octant-sum barrier at the top of the round publishes them).
    // Norms and beta are double-buffered by chunk parity.
    float2 G0[8];  // round-0 gate of the chunk about to be processed
    if (nown > 0) {
        load_beta(uc(0));
        ok = named_bar_and(BAR_IN, NT_IN, wait_or_flag(&bars->qkg[0], 0, 6) && wait_or_flag(&bars->qkg[1], 0, 13));
        if (ok) {
            norms(chunk_len(uc(0)), 0);
            gate_round(0, chunk_len(uc(0)), G0);
            load_beta(uc(1));
        }
    }

    for (int n = 0; n < nown && ok; ++n) {
        const int64_t ctok = cx.tok0 + (int64_t)uc(n) * C;
        const int L = chunk_len(uc(n));
        const bool has_next = n + 1 < nown;
        const uint32_t par = (uint32_t)n & 1u, ppar = (uint32_t)(n - 1) & 1u;
        const uint32_t skp = par ? SM_KP1 : SM_KP0;  // this chunk's k' buffer
        const float *rkq_c = cx.rkq_s + par * 128, *b_c = cx.b_s + par * 64;  // norms, beta

        // ---- channel pass in two rounds of 64 channels.  Block 0 = tokens 0..31
        //      (reference token 15), block 1 = tokens 32..63 (reference token 47). ----
        for (int round = 0; round < 2; ++round) {
            const int c0 = 64 * round + 2 * cp;  // first channel of the pair
            const uint32_t rb = (uint32_t)round * 8192u;
            float2 G[8];  // in-chunk cumulative log2-decay of the pair, tokens t0 .. t0+7
            bool gaok = true;
            if (round == 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) G[j] = G0[j];
            } else if (GH && n >= 2) {
                // the state warps computed this round's gate during the previous chunk
                gaok = wait_or_flag(&bars->gate_rdy, par, 23);
                tc_fence_after();
                uint32_t gr[16];
                tmem_ld16(tb + lq + TM_G + 16 * (warp >> 2), gr);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) G[j] = make_float2(__uint_as_float(gr[2 * j]), __uint_as_float(gr[2 * j + 1]));
            } else {
                gate_round(1, L, G);
            }
            // Round 0 first waits until chunk n-2, the previous user of this chunk's k'
            // buffer and gamma slot (both indexed by chunk parity), is fully consumed.
            bool kok = true;
            if constexpr (M == kFused) {
                if (round == 0 && n >= 2) kok = wait_or_flag(&bars->kp_free[par], (uint32_t)((n >> 1) - 1) & 1u, 8);
            } else {
                // the previous hand-off's bulk copies have read [w ; q^ e^G], P, k' and gamma
                if (round == 0 && n >= 1 && tid == 0) {
                    bulk_wait_read_all();
                    kok = sent_ok;
                }
            }

            // octant sums -> chunk prefix sums and the reference values G15, G31, G47, G63
            ok = named_bar_and(BAR_IN, NT_IN, kok && gaok);
            if (!ok) break;
            float2 os[8];
#pragma unroll
            for (int o = 0; o < 8; ++o) os[o] = *reinterpret_cast<const float2 *>(cx.osum + o * 128 + c0);
            if (GH && round == 1 && n >= 2) {  // TM_G and the round-1 octant sums are read
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->gate_free);
            }
            float2 pre = make_float2(0.f, 0.f);
#pragma unroll
            for (int o = 0; o < 8; ++o)
                if (o < oc) { pre.x += os[o].x; pre.y += os[o].y; }
            float2 ref[4];  // G15, G31, G47, G63 (log2 units)
            ref[0] = make_float2(os[0].x + os[1].x, os[0].y + os[1].y);
#pragma unroll
            for (int r2 = 1; r2 < 4; ++r2)
                ref[r2] = make_float2(ref[r2 - 1].x + os[2 * r2].x + os[2 * r2 + 1].x,
                                      ref[r2 - 1].y + os[2 * r2].y + os[2 * r2 + 1].y);
#pragma unroll
            for (int j = 0; j < 8; ++j) { G[j].x += pre.x; G[j].y += pre.y; }
            if (oc == 7)  // gamma = e^{G63} of this chunk (double-buffered by chunk parity)
                *reinterpret_cast<float2 *>(cx.gam_s + par * 128 + c0) = make_float2(ex2(ref[3].x), ex2(ref[3].y));
            // per-channel factors (each a decay over at most 32 tokens, so >= e^-160):
            //   block 0: e^{G_t} = rho e^{G15};  e^{G31-G_t} = sig e^{G31-G15} (=: s1 <= 1)
            //            e^{G63-G_t} = s1 e^{G63-G31};  e^{G47-G_t} = s1 e^{G47-G31}
            //   block 1: e^{G_t} = rho e^{G47};  e^{G63-G_t} = sig e^{G63-G47}
            // (e^{G15}, e^{G47} may underflow only where every factor they scale is below
            //  e^-12 of the unit-size terms it is added to)
            const float2 Gr = blk ? ref[2] : ref[0];
            const float2 fo = make_float2(ex2(ref[2].x - ref[1].x), ex2(ref[2].y - ref[1].y));
            const float2 fa = make_float2(ex2(Gr.x), ex2(Gr.y));
            float2 fb = make_float2(1.f, 1.f), fc;
            if (blk == 0) {
                fb = make_float2(ex2(ref[1].x - ref[0].x), ex2(ref[1].y - ref[0].y));
                fc = make_float2(ex2(ref[3].x - ref[1].x), ex2(ref[3].y - ref[1].y));
            } else {
                fc = make_float2(ex2(ref[3].x - ref[2].x), ex2(ref[3].y - ref[2].y));
            }
            // every thread waits for the buffers it is about to overwrite; a wait that
            // gives up is combined into the barrier after the operand rows
            bool wok = true;
            if (round == 1)  // A/P operands of round 0 must be consumed first
                wok = wait_or_flag(&bars->mma_in, (mma_cnt++) & 1u, 1);
            else if (M == kFused && n > 0)  // q^ e^G of the previous chunk must be consumed
                wok = wait_or_flag(&bars->wq_free, ppar, 7);
            // operand rows of this octant; the block (uniform per warp) is a compile-time
            // branch of the loop body, and tokens past the chunk end have zero norms.
            auto operand_rows = [&](auto blk0_tag) {
                constexpr bool kBlk0 = decltype(blk0_tag)::value;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float2 rkq = *reinterpret_cast<const float2 *>(rkq_c + 2 * (t0 + j));
                    const float2 kk = mul2(bf2x2(*reinterpret_cast<const uint32_t *>(sm + SM_K + rb + o16[j])),
                                           make_float2(rkq.x, rkq.x));
                    const float2 qv = mul2(bf2x2(*reinterpret_cast<const uint32_t *>(sm + SM_Q + rb + o16[j])),
                                           make_float2(rkq.y, rkq.y));
                    const float d0 = G[j].x - Gr.x, d1 = G[j].y - Gr.y;
                    const float2 rho = make_float2(ex2(d0), ex2(d1));
                    const float2 sig = make_float2(ex2(-d0), ex2(-d1));
                    const float2 kr = mul2(kk, rho), qr = mul2(qv, rho), ks = mul2(kk, sig);
                    st_u64(sm, SM_APA + o32[j], tf32b(kr.x), tf32b(kr.y));
                    st_u64(sm, SM_APA + 8192 + o32[j], tf32b(qr.x), tf32b(qr.y));
                    st_u64(sm, SM_APB + o32[j], tf32b(ks.x), tf32b(ks.y));
                    float2 kp;
                    if (kBlk0) {
                        const float2 s1 = mul2(sig, fb);  // e^{G31 - G_t} <= 1
                        kp = mul2(s1, fc);
                        const float2 ko = mul2(kk, mul2(s1, fo));
                        st_u64(sm, SM_APB + 8192 + o32[j], tf32b(ko.x), tf32b(ko.y));
                    } else {
                        kp = mul2(sig, fc);
                    }
                    const float2 kg = mul2(kr, fa), qg = mul2(qr, fa), kpp = mul2(kk, kp);
                    st_u32(sm, SM_KG + rb + o16[j], pack_f16(kg.x, kg.y));
                    st_u32(sm, SM_WQ + 2 * rb + 8192 + o16[j], pack_f16(qg.x, qg.y));
                    st_u32(sm, skp + rb + o16[j], pack_f16(kpp.x, kpp.y));
                }
            };
            if (blk == 0) operand_rows(std::true_type{});
            else operand_rows(std::false_type{});
            // hand this round's operands to the issue warp (A/P += [k^ rho ; q^ rho]
            // [k^ sig ; k^ e^{G47-G}]^T over the round's 64 channels)
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ops);
            ok = named_bar_and(BAR_IN, NT_IN, wok);
            if (!ok) break;
        }
        if (!ok) break;
        // ---- while the round-1 A/P product runs: the next chunk's round-0 gate (its
        //      first box was requested after this chunk's round 0) ----
        bool gok = true;
        if (has_next) {
            gok = wait_or_flag(&bars->qkg[0], par ^ 1u, 6);
            gate_round(0, chunk_len(uc(n + 1)), G0);
        }
        {
            // the A/P product is complete, and chunk n-1's second state product (the last
            // reader of the single P tile) is done before P is overwritten
            const bool aok = wait_or_flag(&bars->mma_in, (mma_cnt++) & 1u, 1);
            const bool pok = M != kFused || n < 1 || wait_or_flag(&bars->kp_free[ppar], (uint32_t)((n - 1) >> 1) & 1u, 11);
            ok = named_bar_and(BAR_IN, NT_IN, aok && pok && gok);
        }
        tc_fence_after();
        if (!ok) break;

        // ---- select the valid blocks of the A/P product.  Thread = (row ln, column
        //      half hf).  Rows 0..63: Diag(b) A -> fp32 (solve); rows 64..127: P -> fp16.
        {
            const int i = ln & 63;
            const bool ib1 = i >= 32;
            // columns j in [32 hf, 32 hf + 32): block-0 columns of a block-1 row sit at 64 + j
            const uint32_t cbase = hf ? 32u : (ib1 ? 64u : 0u);
            float d[32];
            {
                uint32_t u[32];
                tmem_ld32(tb + lq + TM_AP + cbase, u);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) d[j] = __uint_as_float(u[j]);
            }
            const int jb = 32 * hf;
            if (ln < 64) {
                const float bi = b_c[i];
#pragma unroll
                for (int j0 = 0; j0 < 32; j0 += 4) {
                    float e4[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) e4[jj] = (jb + j0 + jj < i) ? bi * d[j0 + jj] : 0.f;
                    *reinterpret_cast<float4 *>(Lm + i * LST + jb + j0) = make_float4(e4[0], e4[1], e4[2], e4[3]);
                }
            } else {
#pragma unroll
                for (int j0 = 0; j0 < 32; j0 += 8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int jj = 0; jj < 8; jj += 2)
                        pk[jj / 2] = pack_f16((jb + j0 + jj <= i) ? d[j0 + jj] : 0.f,
                                              (jb + j0 + jj + 1 <= i) ? d[j0 + jj + 1] : 0.f);
                    *reinterpret_cast<uint4 *>(sm + SM_P + sw(i, (jb + j0) * 2)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
        tc_fence_before();
        named_bar(BAR_IN, NT_IN);
        tc_fence_after();

        // ---- X = (I + Diag(b) A)^-1 by blocked forward substitution on 16 x 16 blocks.
        //      Diagonal blocks: warp I (one per scheduler) solves block I, lane = column j
        //      (lanes 16..31 idle), row sums split four ways.
        if (warp < 4 && lane < 16) {
            const int I = warp, j = lane, base = 16 * I;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const float *Li = Lm + (base + i) * LST + base;
#pragma unroll
                for (int m0 = 0; m0 < i; m0 += 4) {
                    const float4 l4 = *reinterpret_cast<const float4 *>(Li + m0);
                    acc[0] += l4.x * x[m0];
                    if (m0 + 1 < i) acc[1] += l4.y * x[m0 + 1];
                    if (m0 + 2 < i) acc[2] += l4.z * x[m0 + 2];
                    if (m0 + 3 < i) acc[3] += l4.w * x[m0 + 3];
                }
                x[i] = ((i == j) ? 1.f : 0.f) - ((acc[0] + acc[1]) + (acc[2] + acc[3]));
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) Xm[(base + i) * LST + base + j] = x[i];
        } else if (warp >= 4) {
            // zero the blocks above the block diagonal
            for (int e = tid - 128; e < 6 * 256; e += NT_IN - 128) {
                const int blkid = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int I = blkid < 3 ? 0 : (blkid < 5 ? 1 : 2);
                const int J = blkid < 3 ? blkid + 1 : (blkid < 5 ? blkid - 1 : 3);
                Xm[(16 * I + r) * LST + 16 * J + cc] = 0.f;
            }
        }
        named_bar(BAR_IN, NT_IN);
        //      Blocks below the diagonal by recursive doubling in fp32, all 256 threads:
        //        X_(2B+1)(2B) = -X_(2B+1)(2B+1) L_(2B+1)(2B) X_(2B)(2B)   (16 x 16, B = 0, 1)
        //        X_hl         = -X_hh L_hl X_ll                          (32 x 32 halves)
        //      where h, l are the token halves 32..63 and 0..31.  Every X_II is lower
        //      triangular and the blocks above the diagonal are zero, which bounds the
        //      inner loops below.
        {
            float *Zs = reinterpret_cast<float *>(sm + SM_Y);  // 2 x [16][16]: L_(2B+1)(2B) X_(2B)(2B)
            float *Zb = Zs + 512;                              // [32][ZST]:   L_hl X_ll
            constexpr int ZST = 36;
            {
                // thread = (B, row r, columns c, c + 1)
                const int B = tid >> 7, r = (tid >> 3) & 15, c = (tid & 7) * 2, o = 32 * B;
                const float *Ar = Lm + (o + 16 + r) * LST + o;
                const float *Bc = Xm + o * LST + o + c;
                float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; m += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(Ar + m);
                    const float2 b0 = *reinterpret_cast<const float2 *>(Bc + (m + 0) * LST);
                    const float2 b1 = *reinterpret_cast<const float2 *>(Bc + (m + 1) * LST);
                    const float2 b2 = *reinterpret_cast<const float2 *>(Bc + (m + 2) * LST);
                    const float2 b3 = *reinterpret_cast<const float2 *>(Bc + (m + 3) * LST);
                    a0.x += a.x * b0.x; a0.y += a.x * b0.y;
                    a1.x += a.y * b1.x; a1.y += a.y * b1.y;
                    a0.x += a.z * b2.x; a0.y += a.z * b2.y;
                    a1.x += a.w * b3.x; a1.y += a.w * b3.y;
                }
                *reinterpret_cast<float2 *>(Zs + B * 256 + r * 16 + c) = make_float2(a0.x + a1.x, a0.y + a1.y);
                named_bar(BAR_IN, NT_IN);
                const float *Xr = Xm + (o + 16 + r) * LST + o + 16;
                const float *Zc = Zs + B * 256 + c;
                a0 = make_float2(0.f, 0.f);
                a1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; m += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(Xr + m);
                    const float2 b0 = *reinterpret_cast<const float2 *>(Zc + (m + 0) * 16);
                    const float2 b1 = *reinterpret_cast<const float2 *>(Zc + (m + 1) * 16);
                    const float2 b2 = *reinterpret_cast<const float2 *>(Zc + (m + 2) * 16);
                    const float2 b3 = *reinterpret_cast<const float2 *>(Zc + (m + 3) * 16);
                    a0.x += a.x * b0.x; a0.y += a.x * b0.y;
                    a1.x += a.y * b1.x; a1.y += a.y * b1.y;
                    a0.x += a.z * b2.x; a0.y += a.z * b2.y;
                    a1.x += a.w * b3.x; a1.y += a.w * b3.y;
                }
                *reinterpret_cast<float2 *>(Xm + (o + 16 + r) * LST + o + c) =
                    make_float2(-(a0.x + a1.x), -(a0.y + a1.y));
            }
            named_bar(BAR_IN, NT_IN);
            {
                // Zb = L_hl X_ll: thread = (row r = lane, columns c4 ..+3); rows m < c4 of
                // X_ll are zero in these columns.  Column groups 0,1,2,3,7,6,5,4 for warps
                // 0..7, so that the two warps of each scheduler (w, w+4) share 9 quads.
                const int r = lane, c4 = 4 * (warp < 4 ? warp : 11 - warp);
                const float *Ar = Lm + (32 + r) * LST;
                float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
                for (int m = c4; m < 32; m += 4) {
                    const float4 a = *reinterpret_cast<const float4 *>(Ar + m);
                    const float4 b0 = *reinterpret_cast<const float4 *>(Xm + (m + 0) * LST + c4);
                    const float4 b1 = *reinterpret_cast<const float4 *>(Xm + (m + 1) * LST + c4);
                    const float4 b2 = *reinterpret_cast<const float4 *>(Xm + (m + 2) * LST + c4);
                    const float4 b3 = *reinterpret_cast<const float4 *>(Xm + (m + 3) * LST + c4);
                    a0.x += a.x * b0.x; a0.y += a.x * b0.y; a0.z += a.x * b0.z; a0.w += a.x * b0.w;
                    a1.x += a.y * b1.x; a1.y += a.y * b1.y; a1.z += a.y * b1.z; a1.w += a.y * b1.w;
                    a0.x += a.z * b2.x; a0.y += a.z * b2.y; a0.z += a.z * b2.z; a0.w += a.z * b2.w;
                    a1.x += a.w * b3.x; a1.y += a.w * b3.y; a1.z += a.w * b3.z; a1.w += a.w * b3.w;
                }
                *reinterpret_cast<float4 *>(Zb + r * ZST + c4) =
                    make_float4(a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, a0.w + a1.w);
            }
            named_bar(BAR_IN, NT_IN);
            {
                // X_hl = -X_hh Zb: thread = (rows r4 ..+3 of the half, column c = lane);
                // X_hh is lower triangular, so row r needs m <= r only (row groups
                // permuted as the column groups above)
                const int r4 = 4 * (warp < 4 ? warp : 11 - warp), c = lane;
                float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
                for (int m = 0; m < r4 + 4; m += 4) {
                    const float z0 = Zb[(m + 0) * ZST + c], z1 = Zb[(m + 1) * ZST + c];
                    const float z2 = Zb[(m + 2) * ZST + c], z3 = Zb[(m + 3) * ZST + c];
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const float4 x = *reinterpret_cast<const float4 *>(Xm + (32 + r4 + rr) * LST + 32 + m);
                        a[rr] += x.x * z0;
                        b[rr] += x.y * z1;
                        a[rr] += x.z * z2;
                        b[rr] += x.w * z3;
                    }
                }
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) Xm[(32 + r4 + rr) * LST + c] = -(a[rr] + b[rr]);
            }
            named_bar(BAR_IN, NT_IN);
        }
        // T = X Diag(b): fp16 copy (for w) and bf16 hi + lo pair (for u = T v).
        // Thread = (row i = tid % 64, columns 16 (tid / 64) ..+15): the lanes of a warp
        // take consecutive rows, so the float4 reads of X (row stride 68 floats) and the
        // swizzled 16-byte stores are free of bank conflicts.
        {
            const int i = tid & 63, jq = (tid >> 6) * 16;
            const float *Xr = Xm + i * LST + jq;
#pragma unroll
            for (int j0 = 0; j0 < 16; j0 += 8) {
                const float4 x0 = *reinterpret_cast<const float4 *>(Xr + j0);
                const float4 x1 = *reinterpret_cast<const float4 *>(Xr + j0 + 4);
                const float4 b0 = *reinterpret_cast<const float4 *>(b_c + jq + j0);
                const float4 b1 = *reinterpret_cast<const float4 *>(b_c + jq + j0 + 4);
                const float tv[8] = {x0.x * b0.x, x0.y * b0.y, x0.z * b0.z, x0.w * b0.w,
                                     x1.x * b1.x, x1.y * b1.y, x1.z * b1.z, x1.w * b1.w};
                uint32_t p16[4], phi[4], plo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    p16[e] = pack_f16(tv[2 * e], tv[2 * e + 1]);
                    const __nv_bfloat162 hh = __floats2bfloat162_rn(tv[2 * e], tv[2 * e + 1]);
                    const float2 hf = __bfloat1622float2(hh);
                    const __nv_bfloat162 ll = __floats2bfloat162_rn(tv[2 * e] - hf.x, tv[2 * e + 1] - hf.y);
                    phi[e] = *reinterpret_cast<const uint32_t *>(&hh);
                    plo[e] = *reinterpret_cast<const uint32_t *>(&ll);
                }
                const uint32_t off = sw(i, (jq + j0) * 2);
                *reinterpret_cast<uint4 *>(sm + SM_T16 + off) = make_uint4(p16[0], p16[1], p16[2], p16[3]);
                *reinterpret_cast<uint4 *>(sm + SM_THI + off) = make_uint4(phi[0], phi[1], phi[2], phi[3]);
                *reinterpret_cast<uint4 *>(sm + SM_TLO + off) = make_uint4(plo[0], plo[1], plo[2], plo[3]);
            }
        }
        // a partial chunk's v rows after the sequence are cleared before u = T v reads
        // them (16-byte chunks, every in-chunk thread; the v tile arrived long before)
        bool vok = true;
        if (L < C) {
            vok = wait_or_flag(&bars->v, par, 15);
            if (vok) {
                for (int e = tid; e < (C - L) * 16; e += NT_IN) {
                    const int r = L + (e >> 4);
                    *reinterpret_cast<uint4 *>(sm + SM_V + (uint32_t)(e & 8) * 1024u + (uint32_t)(r * 128 + (e & 7) * 16)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        // hand T to the issue warp (w^T = (k^ e^G)^T T^T, u^T = v^T (T_hi + T_lo)^T)
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ops);

        // ---- w^T = (k^ e^G)^T T^T (fp16), u^T = v^T (T_hi + T_lo)^T (bf16) run on the issue warp ----
        // ---- while the w/u products run: the next chunk's norms (its second box was
        //      requested after this chunk's round 1; they go to the other buffer, since
        //      this chunk's b may still be read by a warp finishing T) ----
        bool sok = true;
        if (has_next) {
            sok = wait_or_flag(&bars->qkg[1], par ^ 1u, 13);
            norms(chunk_len(uc(n + 1)), (int)(par ^ 1u));
            load_beta(uc(n + 2));
        }
        {
            // (if the issue warp gave up, this bounded wait runs out)
            const bool mok = wait_or_flag(&bars->mma_in, (mma_cnt++) & 1u, 3);
            ok = named_bar_and(BAR_IN, NT_IN, sok && mok && vok);
        }
        tc_fence_after();
        if (!ok) break;

        // ---- w (lanes = channel) -> fp16 rows of [w ; q^ e^G]; thread = (channel ln,
        //      tokens 32 hf .. 32 hf + 31) ----
        {
            const int c = ln;
            const uint32_t w64 = (uint32_t)(c >> 6) * 16384u, cb64 = (uint32_t)(c & 63) * 2u;
            uint32_t u[32];
            tmem_ld32(tb + lq + TM_W + 32 * hf, u);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
                *reinterpret_cast<__half *>(sm + SM_WQ + w64 + sw(32 * hf + j, cb64)) = __float2half_rn(__uint_as_float(u[j]));
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(BAR_IN, NT_IN);
        if constexpr (M == kFused) {
            if (tid == 0) mbar_arrive(&bars->full);  // chunk n handed to the state role
        } else if (tid == 0) {
            // chunk uc(n) into CTA 0's slot uc(n) & 1, once CTA 0 has released it (its
            // previous content, chunk uc(n) - 2, consumed); the bulk bytes complete the
            // slot's barrier together with the u^T rows of the sending warps
            const int c = uc(n);
            sent_ok = c < 2 || wait_or_flag(&bars->slot_free, (uint32_t)(n - (f >= 2 ? 0 : 1)) & 1u, 16);
            if (sent_ok) {
                const uint32_t slot = cx.c_slots + (uint32_t)(c & 1) * SLOT_BYTES;
                const uint32_t fb = cx.c_full + (uint32_t)(c & 1) * 8u;
                bulk_s2cluster(slot + SL_WQ, sm + SM_WQ, 32768, fb);
                bulk_s2cluster(slot + SL_KP, sm + skp, 16384, fb);
                bulk_s2cluster(slot + SL_P, sm + SM_P, 8192, fb);
                bulk_s2cluster(slot + SL_GAM, cx.gam_s + par * 128, 512, fb);
                bulk_commit();
            }
        }
    }
    if constexpr (M == kProducer) {
        if (tid == 0) bulk_wait_read_all();  // no copy still reads this CTA's shared memory
    }
}

// =====================================================================================
// Issue role (warp 12, one thread): the in-chunk role's tensor-core products.  For each
// chunk it waits for the operands of A/P round 0, A/P round 1 and the w/u products
// (the `ops` barrier, one arrival per in-chunk warp) and commits each group to
// `mma_in`.  The in-chunk warps never stall on issuing.
// =====================================================================================
template <Mode M>
__device__ void mma_role(const TMaps &tm, const Ctx &cx)
{
    if ((threadIdx.x & 31) != 0) return;
    uint8_t *sm = cx.sm;
    Bars *bars = cx.bars;
    const uint32_t tb = cx.tb;
    const uint32_t sa = smem_u32(sm + SM_APA), sb = smem_u32(sm + SM_APB);
    const uint32_t skg = smem_u32(sm + SM_KG), st16 = smem_u32(sm + SM_T16);
    const uint32_t sv = smem_u32(sm + SM_V), shi = smem_u32(sm + SM_THI), slo = smem_u32(sm + SM_TLO);
    const uint32_t idap = idesc(128, 96, kTF32, kTF32, false, false);
    const uint32_t idw = idesc(128, 64, kF16, kF16, true, false);
    const uint32_t idu = idesc(128, 64, kBF16, kBF16, true, false);
    uint32_t ops_cnt = 0;
    constexpr int S = (M == kProducer) ? kProducers : 1;
    const int f = (M == kProducer) ? cx.first : 0;
    const int nown = cx.nchunks > f ? (cx.nchunks - f + S - 1) / S : 0;
    for (int n = 0; n < nown; ++n) {
        const uint32_t par = (uint32_t)n & 1u, ppar = (uint32_t)(n - 1) & 1u;
        for (int round = 0; round < 2; ++round) {
            if (!wait_or_flag(&bars->ops, (ops_cnt++) & 1u, 12)) return;
            tc_fence_after();
#pragma unroll
            for (int st = 0; st < 8; ++st) {
                const uint64_t da = desc_sw128(sa + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024);
                const uint64_t db = desc_sw128(sb + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024);
                mma_tf32_ss(tb + TM_AP, da, db, idap, (round > 0 || st > 0) ? 1u : 0u);
            }
            mma_commit(&bars->mma_in);
            // The round's operands are written, so every in-chunk thread is done with this
            // round's box of q, k and g: the next own chunk's box goes in (off the in-chunk
            // threads' path, while the product runs).  At round 0 the previous chunk's u
            // product has completed (the in-chunk threads waited for it before handing the
            // chunk over), so this chunk's v tile may replace the last one.
            if (n + 1 < nown)
                load_qkg_box(sm, tm, &bars->qkg[round], cx.h, cx.tok0 + (int64_t)(f + S * (n + 1)) * C, round);
            if (round == 0 && n >= 1) {
                mbar_arrive_expect_tx(&bars->v, 16384);
                load_tile(sm + SM_V, &tm.v, &bars->v, cx.h, cx.tok0 + (int64_t)(f + S * n) * C);
            }
        }
        if (!wait_or_flag(&bars->ops, (ops_cnt++) & 1u, 12)) return;
        if (!wait_or_flag(&bars->v, par, 2)) return;
        if (n > 0 && !wait_or_flag(&bars->u_free, ppar, 9)) return;  // u^T of chunk n-1 read
        tc_fence_after();
#pragma unroll
        for (int st = 0; st < 4; ++st)
            mma_f16_ss(tb + TM_W, desc_sw128(skg + st * 2048, 8192, 1024),
                       desc_sw128(st16 + st * 32, 16, 1024), idw, st > 0);
#pragma unroll
        for (int st = 0; st < 4; ++st)
            mma_f16_ss(tb + TM_U, desc_sw128(sv + st * 2048, 8192, 1024),
                       desc_sw128(shi + st * 32, 16, 1024), idu, st > 0);
#pragma unroll
        for (int st = 0; st < 4; ++st)
            mma_f16_ss(tb + TM_U, desc_sw128(sv + st * 2048, 8192, 1024),
                       desc_sw128(slo + st * 32, 16, 1024), idu, 1);
        mma_commit(&bars->mma_in);  // w and u: T, v and k^ e^G are consumed once it completes
        if constexpr (M == kProducer) mma_commit(&bars->u_rdy);
    }
}

// =====================================================================================
// Split kernel, CTAs 1..3, warps 8..11 (thread v <-> TMEM lane v): each chunk's u^T
// row v, read out of TMEM once the w/u products complete, stored into row v of CTA
// 0's slot for the chunk; then one arrival each on the slot's barrier.
// =====================================================================================
__device__ void u_send_role(const Ctx &cx)
{
    Bars *bars = cx.bars;
    const uint32_t tb = cx.tb;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int v = tid - NT_IN;
    const uint32_t lq = (uint32_t)((warp & 3) * 32) << 16;
    const int f = cx.first;
    const int nown = cx.nchunks > f ? (cx.nchunks - f + kProducers - 1) / kProducers : 0;
    for (int n = 0; n < nown; ++n) {
        const int c = f + kProducers * n;
        if (!wait_or_flag(&bars->u_rdy, (uint32_t)n & 1u, 17)) return;
        tc_fence_after();
        uint32_t a[32], b[32];
        tmem_ld32(tb + lq + TM_U, a);
        tmem_ld32(tb + lq + TM_U + 32, b);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->u_free);  // the next chunk's u product may overwrite TM_U
        if (c >= 2 && !wait_or_flag(&bars->slot_free, (uint32_t)(n - (f >= 2 ? 0 : 1)) & 1u, 18)) return;
        const uint32_t row = cx.c_slots + (uint32_t)(c & 1) * SLOT_BYTES + SL_U + (uint32_t)v * SL_UROW;
#pragma unroll
        for (int j = 0; j < 8; ++j) st_cluster_v4(row + 16u * j, make_uint4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]));
#pragma unroll
        for (int j = 0; j < 8; ++j)
            st_cluster_v4(row + 128u + 16u * j, make_uint4(b[4 * j], b[4 * j + 1], b[4 * j + 2], b[4 * j + 3]));
        mbar_arrive_remote(cx.c_full + (uint32_t)(c & 1) * 8u);
    }
}

// =====================================================================================
// State role (warps 8..11, thread v <-> TMEM lane v): the sequential pass over the
// chunks.  TMEM column block TM_S holds S / tau (tau = the scale of the current U~).
// Per chunk:  S~ = S / sigma -> MMA1: D1 = S~^T [w ; q^ e^G]^T -> U = u - sigma D1[:,0:64]
//   -> U~ = U / tau' -> TM_S <- (gamma * TM_S) tau / tau' -> MMA2: TM_S += U~^T k',
//   D3 = U~^T P^T -> out = scale (sigma D1[:,64:128] + tau' D3).
// =====================================================================================
template <Mode M, bool GH = false, bool CK = false>
__device__ void state_role(const FwdParams &p, const Ctx &cx)
{
    uint8_t *sm = cx.sm;
    Bars *bars = cx.bars;
    const uint32_t tb = cx.tb;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int v = tid - NT_IN;  // value column = TMEM lane
    const uint32_t lq = (uint32_t)((warp & 3) * 32) << 16;
    const bool leader = (v == 0);
    const int64_t H = cx.H, h = cx.h, rstride = cx.rstride;
    const size_t state_off = (size_t)cx.unit * kHead * kHead;
    uint32_t mma_cnt = 0;
    bool ok = true;
    // split kernel, CTA 0: the chunks arrive in two slots of this CTA's shared memory
    SlotBars *sb = reinterpret_cast<SlotBars *>(sm + SL_BARS);
    uint64_t *bar_mma = (M == kConsumer) ? &sb->mma_st : &bars->mma_st;

    // element (k, v) of a state in either layout: S[k][v] (rows of the KV layout are
    // read and written coalesced across threads v) or S[v][k] (thread v owns a row)
    const bool vk = p.state_layout == KDA_LAYOUT_VK;
    auto st_idx = [&](int kk) -> size_t {
        return state_off + (vk ? (size_t)v * kHead + kk : (size_t)kk * kHead + v);
    };

    // initial state (column v) -> TM_S with tau = 1.  The dtype test sits outside the
    // load loops, so that each group's 32 independent loads are in flight together
    // (four memory round trips per thread instead of one per element).
    float tau = 1.f;
    {
        const float *i32 = p.init && p.init_dtype == KDA_STATE_F32 ? reinterpret_cast<const float *>(p.init) : nullptr;
        const __nv_bfloat16 *i16 =
            p.init && p.init_dtype == KDA_STATE_BF16 ? reinterpret_cast<const __nv_bfloat16 *>(p.init) : nullptr;
        for (int k0 = 0; k0 < kHead; k0 += 32) {
            uint32_t r[2][16];
            if (i32) {
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j >> 4][j & 15] = __float_as_uint(__ldg(i32 + st_idx(k0 + j)));
            } else if (i16) {
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j >> 4][j & 15] = __float_as_uint(bf2f(i16[st_idx(k0 + j)]));
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j >> 4][j & 15] = 0u;
            }
            tmem_st16(tb + lq + TM_S + k0, r[0]);
            tmem_st16(tb + lq + TM_S + k0 + 16, r[1]);
        }
    }
    tmem_wait_st();

    // Fused kernel: the round-1 gate of chunk m >= 2 for the in-chunk threads that share
    // this thread's TMEM lane (in-chunk warps q and q + 4, lane l: octants q and q + 4 of
    // the channel pair 64 + 2 l, 65 + 2 l), the same arithmetic as theirs, into TM_G (warp
    // q reads columns 0..15, warp q + 4 columns 16..31) and the round-1 octant sums,
    // computed after this role's work on chunk m - 2, in its idle time, once the in-chunk
    // warps have read chunk m - 1's (gate_free) and chunk m's g box 1 is in.  The gates
    // of chunks 0 and 1 stay with the in-chunk warps: this role is still loading the
    // initial state then, and a unit's first chunks would wait for it.
    auto gate_r1 = [&](int m) -> bool {
        bool w = m < 3 || wait_or_flag(&bars->gate_free, (uint32_t)(m - 3) & 1u, 24);
        w = w && wait_or_flag(&bars->qkg[1], (uint32_t)m & 1u, 25);
        if (!named_bar_and(BAR_ST, NT_ST, w)) return false;
        tc_fence_after();
        const int q = warp & 3, l = tid & 31, c0 = 64 + 2 * l;
        const int64_t rem = cx.len - (int64_t)m * C;
        const int Lc = (int)(rem < C ? rem : C);
        const float aexp = ex2(p.A_log[h] * kLog2e), a2 = aexp * kLog2e, lb2 = p.lower_bound * kLog2e;
        const float2 dtb = *reinterpret_cast<const float2 *>(cx.dtb_s + c0);
        uint32_t r[2][16];
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
            const int oc = q + 4 * hl, t0 = 8 * oc;
            float2 run = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 g2 = bf2x2(*reinterpret_cast<const uint32_t *>(
                    sm + SM_G + 8192u + sw((uint32_t)(t0 + j), (uint32_t)l * 4u)));
                const float x0 = g2.x + dtb.x, x1 = g2.y + dtb.y;
                const float e0 = lg2(1.f + ex2(-fabsf(x0) * kLog2e));
                const float e1 = lg2(1.f + ex2(-fabsf(x1) * kLog2e));
                const bool valid = t0 + j < Lc;
                run.x += valid ? fmaxf(lb2, -a2 * fmaxf(x0, 0.f) - aexp * e0) : 0.f;
                run.y += valid ? fmaxf(lb2, -a2 * fmaxf(x1, 0.f) - aexp * e1) : 0.f;
                r[hl][2 * j] = __float_as_uint(run.x);
                r[hl][2 * j + 1] = __float_as_uint(run.y);
            }
            *reinterpret_cast<float2 *>(cx.osum + oc * 128 + c0) = run;
        }
        tmem_st16(tb + lq + TM_G, r[0]);
        tmem_st16(tb + lq + TM_G + 16, r[1]);
        tmem_wait_st();
        tc_fence_before();
        named_bar(BAR_ST, NT_ST);
        if (leader) mbar_arrive(&bars->gate_rdy);
        return true;
    };

    for (int n = 0; n < cx.nchunks && ok; ++n) {
        const int64_t ctok = cx.tok0 + (int64_t)n * C;
        const int64_t rem = cx.len - (int64_t)n * C;
        const int L = (int)(rem < C ? rem : C);
        const uint32_t par = (uint32_t)n & 1u;
        const uint32_t slot = par * SLOT_BYTES;  // split kernel: this chunk's slot

        // ---- S~^T = (tau TM_S) / sigma as fp16 pairs into TM_SS ----
        float sigma;
        {
            float mx = 0.f;
            // checkpoint instantiation: the state before this chunk, fp32 S[k][v], to
            // slot (tok0 / 64 + sequence + n) * H + h of p.ckpt
            float *ck = nullptr;
            if constexpr (CK)
                ck = p.ckpt + ((size_t)(cx.tok0 / C + cx.unit / H + n) * H + h) * (kHead * kHead) + v;
#pragma unroll
            for (int k0 = 0; k0 < kHead; k0 += 32) {
                uint32_t a[32];
                tmem_ld32(tb + lq + TM_S + k0, a);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fabsf(__uint_as_float(a[j])));
                if constexpr (CK) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) ck[(k0 + j) * kHead] = tau * __uint_as_float(a[j]);
                }
            }
            sigma = pow2_ceil(mx * tau);
            const float f = tau / sigma;
#pragma unroll
            for (int k0 = 0; k0 < kHead; k0 += 32) {
                uint32_t a[32], r[16];
                tmem_ld32(tb + lq + TM_S + k0, a);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    r[j] = pack_f16(__uint_as_float(a[2 * j]) * f, __uint_as_float(a[2 * j + 1]) * f);
                tmem_st16(tb + lq + TM_SS + k0 / 2, r);
            }
            tmem_wait_st();
        }

        // ---- wait for the chunk's operands; MMA1: D1 = S~^T [w ; q^ e^G]^T ----
        tc_fence_before();  // the S~ stores above precede MMA1
        if constexpr (M == kConsumer)
            ok = named_bar_and(BAR_ST, NT_ST, wait_or_flag_cluster(&sb->full[par], ((uint32_t)n >> 1) & 1u, 10));
        else
            ok = named_bar_and(BAR_ST, NT_ST, wait_or_flag(&bars->full, par, 10));
        tc_fence_after();
        if (!ok) break;
        if (leader) {
            const uint32_t swq = smem_u32(sm + (M == kConsumer ? slot + SL_WQ : SM_WQ));
            const uint32_t id = idesc(128, 128, kF16, kF16, false, false);
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_f16_ts(tb + TM_D1, tb + TM_SS + st * 8,
                           desc_sw128(swq + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024), id, st > 0);
            mma_commit(bar_mma);
            if constexpr (M == kFused) mma_commit(&bars->wq_free);
        }
        ok = named_bar_and(BAR_ST, NT_ST, wait_or_flag(bar_mma, (mma_cnt++) & 1u, 4));
        tc_fence_after();
        if (!ok) break;

        // ---- U = u - sigma D1[:, 0:64]; tau' = pow2 >= max|U|; U~^T -> D1 cols 0..31 ----
        float tau_n;
        {
            float U[C];
#pragma unroll
            for (int t0 = 0; t0 < C; t0 += 32) {
                uint32_t a[32], b[32];
                tmem_ld32(tb + lq + TM_D1 + t0, a);
                if constexpr (M == kConsumer) {  // u^T row v from the slot
                    const uint4 *ur = reinterpret_cast<const uint4 *>(sm + slot + SL_U + (uint32_t)v * SL_UROW + t0 * 4);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 x = ur[j];
                        b[4 * j] = x.x;
                        b[4 * j + 1] = x.y;
                        b[4 * j + 2] = x.z;
                        b[4 * j + 3] = x.w;
                    }
                } else {
                    tmem_ld32(tb + lq + TM_U + t0, b);
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) U[t0 + j] = __uint_as_float(b[j]) - sigma * __uint_as_float(a[j]);
            }
            tc_fence_before();
            if constexpr (M == kFused) mbar_arrive(&bars->u_free);  // u^T of this chunk is out of TMEM
            float mx = 0.f;
#pragma unroll
            for (int t = 0; t < C; ++t) mx = fmaxf(mx, fabsf(U[t]));
            tau_n = pow2_ceil(mx);
            const float inv = 1.f / tau_n;
#pragma unroll
            for (int t0 = 0; t0 < C; t0 += 32) {
                uint32_t r[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) r[j] = pack_f16(U[t0 + 2 * j] * inv, U[t0 + 2 * j + 1] * inv);
                tmem_st16(tb + lq + TM_D1 + t0 / 2, r);
            }
        }
        // ---- TM_S <- gamma * TM_S * (tau / tau'), so that MMA2 can accumulate U~^T k' ----
        {
            const float f = tau / tau_n;
            const float *gam = (M == kConsumer) ? reinterpret_cast<const float *>(sm + slot + SL_GAM) : cx.gam_s + par * 128;
#pragma unroll
            for (int k0 = 0; k0 < kHead; k0 += 32) {
                uint32_t a[32];
                tmem_ld32(tb + lq + TM_S + k0, a);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(gam + k0 + j);
                    a[j] = __float_as_uint(__uint_as_float(a[j]) * (g4.x * f));
                    a[j + 1] = __float_as_uint(__uint_as_float(a[j + 1]) * (g4.y * f));
                    a[j + 2] = __float_as_uint(__uint_as_float(a[j + 2]) * (g4.z * f));
                    a[j + 3] = __float_as_uint(__uint_as_float(a[j + 3]) * (g4.w * f));
                }
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) { lo[j] = a[j]; hi[j] = a[16 + j]; }
                tmem_st16(tb + lq + TM_S + k0, lo);
                tmem_st16(tb + lq + TM_S + k0 + 16, hi);
            }
            tmem_wait_st();
        }
        tau = tau_n;
        tc_fence_before();
        named_bar(BAR_ST, NT_ST);
        tc_fence_after();

        // ---- MMA2: TM_S += U~^T k' (N = 128), D3 = U~^T P^T (N = 64) ----
        if (leader) {
            const uint32_t skp = smem_u32(sm + (M == kConsumer ? slot + SL_KP : (par ? SM_KP1 : SM_KP0)));
            const uint32_t sp = smem_u32(sm + (M == kConsumer ? slot + SL_P : SM_P));
            const uint32_t id2 = idesc(128, 128, kF16, kF16, false, true);
            const uint32_t id3 = idesc(128, 64, kF16, kF16, false, false);
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_f16_ts(tb + TM_S, tb + TM_D1 + st * 8, desc_sw128(skp + st * 2048, 8192, 1024), id2, 1u);
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_f16_ts(tb + TM_D3, tb + TM_D1 + st * 8, desc_sw128(sp + st * 32, 16, 1024), id3, st > 0);
            mma_commit(bar_mma);
            if constexpr (M == kFused) mma_commit(&bars->kp_free[par]);
        }
        ok = named_bar_and(BAR_ST, NT_ST, wait_or_flag(bar_mma, (mma_cnt++) & 1u, 5));
        tc_fence_after();
        if (!ok) break;
        if constexpr (M == kConsumer) {
            // the slot is consumed (MMA1, MMA2 complete; u and gamma read before the
            // barrier above): re-arm it for chunk n + 2 (expected bytes), and tell the CTA
            // that sends chunk n + 2 that it may
            if (leader && n + 2 < cx.nchunks) {
                mbar_arrive_expect_tx(&sb->full[par], kSendBytes);
                const uint32_t dst = 1u + (uint32_t)((n + 2) % kProducers);
                mbar_arrive_remote(mapa_shared(smem_u32(&bars->slot_free), dst));
            }
        }

        // ---- out = scale (sigma D1[:, 64:128] + tau D3): thread v stores column v of each
        //      token; a warp's 32 columns are 64 contiguous bytes of the token's row
        //      (not in the checkpoint instantiation, which writes no output) ----
        if constexpr (!CK) {
            __nv_bfloat16 *op = p.out + (ctok * H + h) * kHead + v;
            const float fs = p.scale * sigma, ft = p.scale * tau;
#pragma unroll 1
            for (int t0 = 0; t0 < C; t0 += 16) {
                uint32_t a[16], b[16];
                tmem_ld16(tb + lq + TM_D1 + 64 + t0, a);
                tmem_ld16(tb + lq + TM_D3 + t0, b);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (t0 + j < L) *op = __float2bfloat16_rn(fs * __uint_as_float(a[j]) + ft * __uint_as_float(b[j]));
                    op += rstride;
                }
            }
        }
        if constexpr (GH) {  // the round-1 gate of the chunk after next
            if (n + 2 < cx.nchunks && !(ok = gate_r1(n + 2))) break;
        }
    }

    // ---- final state = tau TM_S (column v), fp32 or bf16 (round to nearest even) ----
    if (ok && p.final_state) {
        const bool bf = p.final_dtype == KDA_STATE_BF16;
        for (int k0 = 0; k0 < kHead; k0 += 32) {
            uint32_t a[32];
            tmem_ld32(tb + lq + TM_S + k0, a);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float x = tau * __uint_as_float(a[j]);
                if (bf) reinterpret_cast<__nv_bfloat16 *>(p.final_state)[st_idx(k0 + j)] = __float2bfloat16_rn(x);
                else reinterpret_cast<float *>(p.final_state)[st_idx(k0 + j)] = x;
            }
        }
    }
}

// Shared-memory context of a CTA (the same offsets in every CTA of either kernel).
__device__ __forceinline__ void init_ctx(Ctx &cx, uint8_t *sm)
{
    cx.sm = sm;
    cx.rkq_s = reinterpret_cast<float *>(sm + SM_MISC);
    cx.b_s = cx.rkq_s + 256;    // [2][64]
    cx.gam_s = cx.b_s + 128;    // [2][128]
    cx.osum = cx.gam_s + 256;   // [8][128]
    cx.bars = reinterpret_cast<Bars *>(cx.osum + 1024);
    cx.dtb_s = reinterpret_cast<float *>(sm + SM_MISC + 7168);
    cx.first = 0;
    cx.c_slots = cx.c_full = 0;
}

// The launch's (sequence, head) unit u into cx: sequence-major, with the sequences of a
// varlen batch of up to kLptMax in decreasing length.  Every thread of the CTA calls it.
__device__ void locate_unit(const FwdParams &p, Ctx &cx, int64_t u)
{
    uint8_t *sm = cx.sm;
    const int tid = threadIdx.x;
    cx.H = p.H;
    int64_t s = u / p.H;
    cx.h = u % p.H;
    if (p.cu && p.N > 1 && p.N <= kLptMax) {
        // Longest sequences first: unit group r takes the sequence of rank r in decreasing
        // length (ties by index; the ranks are a permutation), so that the end of the grid
        // holds short sequences rather than a long one started last.  The A/P region is
        // free until the first chunk.
        int64_t *lens = reinterpret_cast<int64_t *>(sm + SM_APA);
        int *pick = reinterpret_cast<int *>(sm + SM_APA + 8 * kLptMax);
        for (int i = tid; i < p.N; i += NT) lens[i] = p.cu[i + 1] - p.cu[i];
        __syncthreads();
        for (int c = tid; c < p.N; c += NT) {
            const int64_t lc = lens[c];
            int64_t rank = 0;
            for (int v = 0; v < p.N; ++v) rank += (lens[v] > lc) || (lens[v] == lc && v < c);
            if (rank == s) *pick = c;
        }
        __syncthreads();
        s = *pick;
        __syncthreads();  // every thread has read pick before the region is reused
    }
    cx.unit = s * p.H + cx.h;
    if (p.cu) {
        cx.tok0 = p.cu[s];
        cx.len = p.cu[s + 1] - cx.tok0;
        if (cx.len < 0) cx.len = 0;
    } else {
        cx.tok0 = s * p.T;
        cx.len = p.T;
    }
    cx.rstride = p.H * kHead;
    cx.nchunks = (int)((cx.len + C - 1) / C);
}

// Barriers of a CTA that runs the in-chunk role (fused kernel, or CTAs 1..3 of the split
// kernel); thread 0.
__device__ __forceinline__ void init_bars(Bars *b)
{
    mbar_init(&b->qkg[0], 1);
    mbar_init(&b->qkg[1], 1);
    mbar_init(&b->v, 1);
    mbar_init(&b->mma_in, 1);
    mbar_init(&b->mma_st, 1);
    mbar_init(&b->full, 1);
    mbar_init(&b->wq_free, 1);
    mbar_init(&b->kp_free[0], 1);
    mbar_init(&b->kp_free[1], 1);
    mbar_init(&b->u_free, NT_ST);
    mbar_init(&b->ops, NT_IN / 32);
    mbar_init(&b->gate_rdy, 1);
    mbar_init(&b->gate_free, NT_IN / 32);
    mbar_init(&b->u_rdy, 1);
    mbar_init(&b->slot_free, 1);
}

// Thread 0: has another CTA of this launch already given up?
__device__ __forceinline__ void read_abort(const FwdParams &p)
{
    s_epoch = p.epoch;
    const int e = *reinterpret_cast<volatile int *>(&g_chunk_error);
    s_abort = e != 0 && ((uint32_t)e >> 8) == p.epoch;
}

// GH: the state role computes the round-1 gates of chunks 2.. (launches of long units)
template <bool GH, bool CK = false>
__global__ void __launch_bounds__(NT, 1)
chunk_kernel(const FwdParams p, const __grid_constant__ TMaps tm)
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment by pointer arithmetic on the shared array itself, so that the
    // compiler keeps every access through sm in the shared space (32-bit addresses,
    // shared loads/stores) instead of falling back to generic ones
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    init_ctx(cx, sm);
    uint32_t *tbase_s = reinterpret_cast<uint32_t *>(cx.bars + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    locate_unit(p, cx, blockIdx.x);

    if (tid == 0) {
        read_abort(p);
        init_bars(cx.bars);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase_s, 512);
        tmem_relinquish();
    }
    if (tid < kHead && cx.nchunks > 0) cx.dtb_s[tid] = p.dt_bias[cx.h * kHead + tid];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cx.tb = *tbase_s;
    if (s_abort) {  // another CTA of this launch gave up before this one started
        if (warp == 0) tmem_dealloc(cx.tb, 512);
        return;
    }
    if (tid == 0 && cx.nchunks > 0) {  // first chunk's tiles
        load_qkg_box(sm, tm, &cx.bars->qkg[0], cx.h, cx.tok0, 0);
        load_qkg_box(sm, tm, &cx.bars->qkg[1], cx.h, cx.tok0, 1);
        mbar_arrive_expect_tx(&cx.bars->v, 16384);
        load_tile(sm + SM_V, &tm.v, &cx.bars->v, cx.h, cx.tok0);
    }

    if (warp < NT_IN / 32) in_chunk_role<kFused, GH>(p, tm, cx);
    else if (warp < (NT_IN + NT_ST) / 32) state_role<kFused, GH, CK>(p, cx);
    else mma_role<kFused>(tm, cx);

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(cx.tb, 512);
}

// Split kernel: a cluster of kSplitCta CTAs per unit (cluster index = unit).  CTA 0 runs
// the state pass on chunks that CTAs 1..3 prepare (chunk c on CTA 1 + c % 3).
__global__ void __launch_bounds__(NT, 1)
chunk_kernel_split(const FwdParams p, const __grid_constant__ TMaps tm)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    init_ctx(cx, sm);
    uint32_t *tbase_s = reinterpret_cast<uint32_t *>(cx.bars + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t rank = cluster_ctarank();
    locate_unit(p, cx, blockIdx.x / kSplitCta);
    cx.first = (int)rank - 1;
    cx.c_slots = mapa_shared(smem_u32(sm), 0);  // the same offsets in every CTA
    cx.c_full = mapa_shared(smem_u32(sm + SL_BARS), 0);
    SlotBars *sb = reinterpret_cast<SlotBars *>(sm + SL_BARS);

    if (tid == 0) {
        read_abort(p);
        if (rank == 0) {
            mbar_init(&sb->full[0], 1 + NT_ST);
            mbar_init(&sb->full[1], 1 + NT_ST);
            mbar_init(&sb->mma_st, 1);
        } else {
            init_bars(cx.bars);
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase_s, 512);
        tmem_relinquish();
    }
    if (rank != 0 && tid < kHead && cx.nchunks > cx.first) cx.dtb_s[tid] = p.dt_bias[cx.h * kHead + tid];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cx.tb = *tbase_s;
    if (rank == 0 && tid == 0) {  // slots 0 and 1 expect their first chunks' bulk bytes
        if (cx.nchunks > 0) mbar_arrive_expect_tx(&sb->full[0], kSendBytes);
        if (cx.nchunks > 1) mbar_arrive_expect_tx(&sb->full[1], kSendBytes);
    }
    cluster_sync();  // every CTA's barriers are initialised before any remote access

    if (!s_abort) {
        if (rank == 0) {
            if (warp >= NT_IN / 32 && warp < (NT_IN + NT_ST) / 32) state_role<kConsumer>(p, cx);
        } else {
            if (tid == 0 && cx.first < cx.nchunks) {  // first own chunk's tiles
                const int64_t tok = cx.tok0 + (int64_t)cx.first * C;
                load_qkg_box(sm, tm, &cx.bars->qkg[0], cx.h, tok, 0);
                load_qkg_box(sm, tm, &cx.bars->qkg[1], cx.h, tok, 1);
                mbar_arrive_expect_tx(&cx.bars->v, 16384);
                load_tile(sm + SM_V, &tm.v, &cx.bars->v, cx.h, tok);
            }
            if (warp < NT_IN / 32) in_chunk_role<kProducer>(p, tm, cx);
            else if (warp < (NT_IN + NT_ST) / 32) u_send_role(cx);
            else mma_role<kProducer>(tm, cx);
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while a copy or an arrival may still target it
    if (warp == 0) tmem_dealloc(cx.tb, 512);
}

// Error code the next launch starts with (0 = none); see chunked_inject_error.
std::atomic<int> g_inject{0};

// Driver entry point for cuTensorMapEncodeTiled, resolved once through the runtime.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

}  // namespace

// Launch configuration of the split kernel for `units` units (clusters of kSplitCta).
static void split_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute (&at)[1], int64_t units,
                         cudaStream_t stream)
{
    cfg.gridDim = dim3((unsigned)(units * kSplitCta));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = stream;
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kSplitCta;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
}

// The split kernel serves launches whose units all fit the device at once as clusters
// (so a unit's chunks spread over 4 SMs instead of 1), with at least kSplitMinChunks
// chunks per unit on average; larger launches already fill the SMs with one CTA per unit.
constexpr int64_t kSplitMinChunks = 4;
std::atomic<int> g_schedule{KDA_SCHEDULE_AUTO};
int g_split_clusters[64];  // per device: clusters of the split kernel resident at once, + 1 (0 = unknown)
thread_local int g_last_schedule = KDA_SCHEDULE_FUSED;  // of this thread's last launch

static bool use_split(const FwdParams &p, int64_t units)
{
    const int mode = g_schedule.load();
    if (mode == KDA_SCHEDULE_FUSED || units <= 0) return false;
    const int64_t tokens = p.B * p.T;
    if (mode == KDA_SCHEDULE_AUTO && tokens < kSplitMinChunks * C * (p.cu ? p.N : p.B)) return false;
    int *clusters = g_split_clusters;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (clusters[dev] == 0) {
        static int attr_split[64];
        int n = 0;
        if (set_smem_limit_once(chunk_kernel_split, SMEM_ALLOC, attr_split)) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            split_config(cfg, at, 1, 0);
            if (cudaOccupancyMaxActiveClusters(&n, chunk_kernel_split, &cfg) != cudaSuccess) {
                n = 0;
                cudaGetLastError();
            }
        }
        clusters[dev] = n + 1;
    }
    return units <= clusters[dev] - 1;
}

int launch_chunked(const FwdParams &p, cudaStream_t stream)
{
    const int64_t ctas = p.N * p.H;
    if (ctas <= 0) return 0;
    if (ctas > (int64_t)INT32_MAX) return KDA_ERR_SHAPE;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return KDA_ERR_CUDA;
    // q, k, g, v viewed as 2-D bf16 tensors [tokens][H * 128]; box [64 tokens][64
    // channels] with the 128-byte swizzle; rows past the end read as zeros.
    TMaps tm;
    const int64_t rows = p.B * p.T;
    cuuint64_t dims[2] = {(cuuint64_t)(p.H * kHead), (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)(p.H * kHead * 2)};
    cuuint32_t box[2] = {64, (cuuint32_t)C};
    cuuint32_t estr[2] = {1, 1};
    const __nv_bfloat16 *src[4] = {p.q, p.k, p.g, p.v};
    CUtensorMap *dst[4] = {&tm.q, &tm.k, &tm.g, &tm.v};
    for (int i = 0; i < 4; ++i) {
        if (enc(dst[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(src[i]),
                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return KDA_ERR_CUDA;
    }
    static int attr_plain[64], attr_gh[64], attr_ck[64];
    if (!set_smem_limit_once(chunk_kernel<false>, SMEM_ALLOC, attr_plain) ||
        !set_smem_limit_once(chunk_kernel<true>, SMEM_ALLOC, attr_gh) ||
        (p.ckpt && !set_smem_limit_once(chunk_kernel<true, true>, SMEM_ALLOC, attr_ck)))
        return KDA_ERR_CUDA;
    // the launch's epoch: 24 bits, never 0 (an error word of 0 means no error)
    static std::atomic<uint32_t> epochs{0};
    FwdParams pe = p;
    pe.epoch = (epochs.fetch_add(1u) % 0xFFFFFFu) + 1u;
    const int inject = g_inject.exchange(0);
    if (inject) {  // the launch starts as if one of its CTAs had given up with this code
        const int word = (int)(pe.epoch << 8) | inject;
        if (cudaMemcpyToSymbolAsync(g_chunk_error, &word, sizeof(int), 0, cudaMemcpyHostToDevice,
                                    stream) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    g_last_schedule = KDA_SCHEDULE_FUSED;
    if (p.ckpt) {  // the backward pass's checkpoints: fused schedule, no output
        chunk_kernel<true, true><<<(unsigned)ctas, NT, SMEM_ALLOC, stream>>>(pe, tm);
        return cudaGetLastError() == cudaSuccess ? 1 : KDA_ERR_CUDA;
    }
    if (use_split(p, ctas)) {
        g_last_schedule = KDA_SCHEDULE_SPLIT;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        split_config(cfg, at, ctas, stream);
        if (cudaLaunchKernelEx(&cfg, chunk_kernel_split, pe, tm) == cudaSuccess) return 1;
        // the device refused the cluster launch (a configuration error, which does not
        // stick): the fused kernel computes the same bits; no split launches here again
        cudaGetLastError();
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) g_split_clusters[dev] = 1;
        g_last_schedule = KDA_SCHEDULE_FUSED;
    }
    // units averaging kGateHandoffTokens tokens or more: the state role takes the
    // round-1 gates (measured faster there, and slower for units of a few chunks)
    const int64_t avg_tokens = p.cu ? (p.B * p.T) / (p.N > 0 ? p.N : 1) : p.T;
    if (avg_tokens >= kGateHandoffTokens)
        chunk_kernel<true><<<(unsigned)ctas, NT, SMEM_ALLOC, stream>>>(pe, tm);
    else
        chunk_kernel<false><<<(unsigned)ctas, NT, SMEM_ALLOC, stream>>>(pe, tm);
    return cudaGetLastError() == cudaSuccess ? 1 : KDA_ERR_CUDA;
}

int chunked_last_schedule() { return g_last_schedule; }

int chunked_set_schedule(int mode)
{
    if (mode != KDA_SCHEDULE_AUTO && mode != KDA_SCHEDULE_FUSED && mode != KDA_SCHEDULE_SPLIT)
        return KDA_ERR_ARG;
    return g_schedule.exchange(mode);
}

int chunked_inject_error(int code)
{
    if (code < 0 || code > 255) return KDA_ERR_ARG;  // 0 cancels a pending injection
    g_inject.store(code);
    return KDA_OK;
}

int chunked_device_error(bool reset)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_chunk_error, sizeof(int)) != cudaSuccess) return -1;
    if (reset && v) {
        const int z = 0;
        cudaMemcpyToSymbol(g_chunk_error, &z, sizeof(int));
    }
    return v & 0xFF;  // the code of the wait that gave up
}

}  // namespace kda
