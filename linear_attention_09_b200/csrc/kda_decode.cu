// KDA decode step for sm_100a: one new token per sequence, state read-modify-write.
//
// The operator is the one of kda_chunk.cu (Kimi Delta Attention, FlashKDA pages:
// 7minutos.es "¿Qué es la atención Kimi Delta...?"), applied to a single token with
// the state S (K x V) kept in HBM between calls (fp32 or bf16, S[k][v] or S[v][k], the
// state variants the prefill entry point kda_fwd_ex reads and writes):
//   S' = Diag(alpha) S,  r = v - S'^T k^,  S <- S' + b k^ r^T,
//   o  = scale S^T q^ = scale (S'^T q^ + b r (k^ . q^)).
// One pass reads S (the two contractions S'^T k^ and S'^T q^), one pass writes it:
// every thread keeps its 64 entries of S' in registers in between.  The step is
// bound by HBM traffic (128 KB of state per token-head), so it runs on the CUDA
// cores with coalesced row accesses (streaming cache hints: the state is touched
// once per step); there is no contraction worth a tensor core.
#include "kda.h"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int DT = 256;  // thread = (value column v = tid % 128, row half tid / 128)
constexpr int RH = 64;   // state rows per thread

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// VK: state layout S[v][k] (else S[k][v]); IN_BF16 / OUT_BF16: state element types.
template <bool VK, bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(DT) decode_kernel(const DecodeParams p)
{
    __shared__ float qh_s[kHead], kh_s[kHead], al_s[kHead];  // q^, k^, alpha per channel
    __shared__ float2 part[2][kHead];                         // per half: (S'^T k^, S'^T q^)
    __shared__ float wsum[4][3];                              // warp sums: |q|^2, |k|^2, q.k
    const int tid = threadIdx.x, v = tid & (kHead - 1), half = tid >> 7;
    const int warp = tid >> 5, lane = tid & 31;
    const size_t unit = blockIdx.x;  // sequence * H + head
    const int64_t h = (int64_t)(unit % (size_t)p.H);
    const size_t vec = unit * kHead;

    // ---- channel c = tid (first 128 threads): activations and norms ----
    float qc = 0.f, kc = 0.f;
    if (tid < kHead) {
        qc = bf(p.q, vec + tid);
        kc = bf(p.k, vec + tid);
        const float x = bf(p.g, vec + tid) + p.dt_bias[h * kHead + tid];
        const float sp = fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));  // softplus
        const float lam = fmaxf(p.lower_bound, -expf(p.A_log[h]) * sp);
        al_s[tid] = expf(lam);
        float s0 = qc * qc, s1 = kc * kc, s2 = qc * kc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        }
        if (lane == 0) {
            wsum[warp][0] = s0;
            wsum[warp][1] = s1;
            wsum[warp][2] = s2;
        }
    }
    __syncthreads();
    const float sqq = (wsum[0][0] + wsum[1][0]) + (wsum[2][0] + wsum[3][0]);
    const float skk = (wsum[0][1] + wsum[1][1]) + (wsum[2][1] + wsum[3][1]);
    const float sqk = (wsum[0][2] + wsum[1][2]) + (wsum[2][2] + wsum[3][2]);
    const float rq = rsqrtf(sqq + 1e-6f), rk = rsqrtf(skk + 1e-6f);
    if (tid < kHead) {
        qh_s[tid] = qc * rq;
        kh_s[tid] = kc * rk;
    }
    const float b = 1.f / (1.f + expf(-bf(p.beta, unit)));
    const float kq = sqk * rq * rk;  // k^ . q^
    __syncthreads();

    // ---- read pass: S' = Diag(alpha) S on this thread's rows, and its contractions.
    //      S[k][v]: row k of the state is contiguous across the threads v (coalesced
    //      element loads); S[v][k]: thread v reads its own 64 contiguous entries with
    //      16-byte loads.  bf16 states are promoted exactly. ----
    const size_t ubase = unit * (size_t)kHead * kHead;
    const int c0 = half * RH;
    float s[RH];
    if (!VK) {
        const size_t sb = ubase + v;
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            const size_t e = sb + (size_t)(c0 + i) * kHead;
            s[i] = IN_BF16 ? __bfloat162float(__ldcs(reinterpret_cast<const __nv_bfloat16 *>(p.state_in) + e))
                           : __ldcs(reinterpret_cast<const float *>(p.state_in) + e);
        }
    } else {
        const size_t sb = ubase + (size_t)v * kHead + c0;
        if (IN_BF16) {
            const uint4 *src = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.state_in) + sb);
#pragma unroll
            for (int i = 0; i < RH / 8; ++i) {
                const uint4 w = __ldcs(src + i);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s[8 * i + 2 * e] = __uint_as_float(ww[e] << 16);
                    s[8 * i + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
                }
            }
        } else {
            const float4 *src = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.state_in) + sb);
#pragma unroll
            for (int i = 0; i < RH / 4; ++i) {
                const float4 w = __ldcs(src + i);
                s[4 * i] = w.x; s[4 * i + 1] = w.y; s[4 * i + 2] = w.z; s[4 * i + 3] = w.w;
            }
        }
    }
    float dk = 0.f, dq = 0.f;
#pragma unroll
    for (int i = 0; i < RH; ++i) {
        s[i] *= al_s[c0 + i];
        dk += s[i] * kh_s[c0 + i];
        dq += s[i] * qh_s[c0 + i];
    }
    part[half][v] = make_float2(dk, dq);
    __syncthreads();
    const float2 pa = part[0][v], pb = part[1][v];
    const float r = bf(p.v, vec + v) - (pa.x + pb.x);  // delta: v - S'^T k^
    if (half == 0) p.out[vec + v] = __float2bfloat16_rn(p.scale * ((pa.y + pb.y) + b * r * kq));

    // ---- write pass: S = S' + b k^ r^T (bf16 out: round to nearest even) ----
    const float br = b * r;
#pragma unroll
    for (int i = 0; i < RH; ++i) s[i] += br * kh_s[c0 + i];
    if (!VK) {
        const size_t sb = ubase + v;
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            const size_t e = sb + (size_t)(c0 + i) * kHead;
            if (OUT_BF16) __stcs(reinterpret_cast<__nv_bfloat16 *>(p.state_out) + e, __float2bfloat16_rn(s[i]));
            else __stcs(reinterpret_cast<float *>(p.state_out) + e, s[i]);
        }
    } else {
        const size_t sb = ubase + (size_t)v * kHead + c0;
        if (OUT_BF16) {
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.state_out) + sb);
#pragma unroll
            for (int i = 0; i < RH / 8; ++i) {
                uint32_t ww[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 hh = __floats2bfloat162_rn(s[8 * i + 2 * e], s[8 * i + 2 * e + 1]);
                    ww[e] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                __stcs(dst + i, make_uint4(ww[0], ww[1], ww[2], ww[3]));
            }
        } else {
            float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.state_out) + sb);
#pragma unroll
            for (int i = 0; i < RH / 4; ++i) __stcs(dst + i, make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]));
        }
    }
}

}  // namespace

int launch_decode(const DecodeParams &p, cudaStream_t stream)
{
    const int64_t ctas = p.N * p.H;
    if (ctas <= 0) return 0;
    if (ctas > (int64_t)INT32_MAX) return KDA_ERR_SHAPE;
    const bool vk = p.state_layout == KDA_LAYOUT_VK;
    const bool ib = p.in_dtype == KDA_STATE_BF16, ob = p.out_dtype == KDA_STATE_BF16;
    auto kern = vk ? (ib ? (ob ? decode_kernel<true, true, true> : decode_kernel<true, true, false>)
                         : (ob ? decode_kernel<true, false, true> : decode_kernel<true, false, false>))
                   : (ib ? (ob ? decode_kernel<false, true, true> : decode_kernel<false, true, false>)
                         : (ob ? decode_kernel<false, false, true> : decode_kernel<false, false, false>));
    kern<<<(unsigned)ctas, DT, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 1 : KDA_ERR_CUDA;
}

}  // namespace kda
