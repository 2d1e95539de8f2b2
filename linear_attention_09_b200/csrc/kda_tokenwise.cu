// Token-serial KDA forward kernel (fp32 on CUDA cores).
//
// One CTA per (sequence, head); thread v owns column v of the state S (K = 128
// fp32 registers), so the recurrence of the Kimi Delta Attention operator
// (FlashKDA de código abierto de Moonshot AI, section "¿Qué es la atención Kimi
// Delta...?": a gated delta rule with channel-wise decay) is thread-local:
//   S[:,v] *= alpha;  r = b (v_t[v] - S[:,v].kh);  S[:,v] += kh r;  o_v = S[:,v].qh
// The per-token activations (L2 norms, sigmoid, gate) are computed cooperatively
// for blocks of 16 tokens and broadcast through shared memory.
//
// This kernel is the parity scaffold of the C ABI: it is launched only for the
// shapes the chunked tensor-core kernel does not take.
#include "kda_internal.cuh"
#include "kda.h"

namespace kda {
namespace {

constexpr int kTB = 16;  // tokens per activation block

struct TokenwiseSmem {
    float qh[kTB][kHead];
    float kh[kTB][kHead];
    float alpha[kTB][kHead];
    float b[kTB];
};

__device__ __forceinline__ float softplus_f(float x)
{
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

__device__ __forceinline__ void load4_bf16(const __nv_bfloat16 *src, float f[4])
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(src);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    f[0] = fa.x; f[1] = fa.y; f[2] = fb.x; f[3] = fb.y;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__global__ void __launch_bounds__(128) tokenwise_kernel(const FwdParams p)
{
    __shared__ __align__(16) TokenwiseSmem sm;
    const int64_t s = blockIdx.x / p.H, h = blockIdx.x % p.H;
    int64_t tok0, len;
    if (p.cu) {
        tok0 = p.cu[s];
        len = p.cu[s + 1] - tok0;
        if (len < 0) len = 0;
    } else {
        tok0 = s * p.T;
        len = p.T;
    }
    const int vcol = threadIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t soff = (size_t)(s * p.H + h) * kHead * kHead;

    float S[kHead];
    if (p.init && p.init_dtype == KDA_STATE_F32) {
        const float *src = reinterpret_cast<const float *>(p.init) + soff;
#pragma unroll
        for (int k = 0; k < kHead; ++k) S[k] = src[k * kHead + vcol];
    } else if (p.init && p.init_dtype == KDA_STATE_BF16) {
        const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(p.init) + soff;
#pragma unroll
        for (int k = 0; k < kHead; ++k) S[k] = __bfloat162float(src[k * kHead + vcol]);
    } else {
#pragma unroll
        for (int k = 0; k < kHead; ++k) S[k] = 0.f;
    }
    const float decay = expf(p.A_log[h]);

    for (int64_t t0 = 0; t0 < len; t0 += kTB) {
        const int n = (int)((len - t0) < kTB ? (len - t0) : kTB);
        for (int tt = warp; tt < n; tt += 4) {
            const int64_t tok = tok0 + t0 + tt;
            const size_t row = (size_t)(tok * p.H + h) * kHead + lane * 4;
            float qf[4], kf[4], gf[4];
            load4_bf16(p.q + row, qf);
            load4_bf16(p.k + row, kf);
            load4_bf16(p.g + row, gf);
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) { sq += qf[i] * qf[i]; sk += kf[i] * kf[i]; }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            const float rq = 1.f / sqrtf(sq + 1e-6f), rk = 1.f / sqrtf(sk + 1e-6f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = lane * 4 + i;
                sm.qh[tt][c] = qf[i] * rq;
                sm.kh[tt][c] = kf[i] * rk;
                const float x = gf[i] + p.dt_bias[h * kHead + c];
                sm.alpha[tt][c] = expf(fmaxf(p.lower_bound, -decay * softplus_f(x)));
            }
            if (lane == 0) {
                const float bl = __bfloat162float(p.beta[tok * p.H + h]);
                sm.b[tt] = 1.f / (1.f + expf(-bl));
            }
        }
        __syncthreads();
        for (int tt = 0; tt < n; ++tt) {
            const int64_t tok = tok0 + t0 + tt;
            const size_t vo = (size_t)(tok * p.H + h) * kHead + vcol;
            const float vv = __bfloat162float(p.v[vo]);
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < kHead; k += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(&sm.alpha[tt][k]);
                const float4 kk = *reinterpret_cast<const float4 *>(&sm.kh[tt][k]);
                S[k] *= a.x; S[k + 1] *= a.y; S[k + 2] *= a.z; S[k + 3] *= a.w;
                acc += S[k] * kk.x + S[k + 1] * kk.y + S[k + 2] * kk.z + S[k + 3] * kk.w;
            }
            const float r = sm.b[tt] * (vv - acc);
            float o = 0.f;
#pragma unroll
            for (int k = 0; k < kHead; k += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&sm.kh[tt][k]);
                const float4 qq = *reinterpret_cast<const float4 *>(&sm.qh[tt][k]);
                S[k] += kk.x * r; S[k + 1] += kk.y * r; S[k + 2] += kk.z * r; S[k + 3] += kk.w * r;
                o += S[k] * qq.x + S[k + 1] * qq.y + S[k + 2] * qq.z + S[k + 3] * qq.w;
            }
            p.out[vo] = __float2bfloat16_rn(p.scale * o);
        }
        __syncthreads();
    }
    if (p.final_state) {
        float *dst = p.final_state + soff;
#pragma unroll
        for (int k = 0; k < kHead; ++k) dst[k * kHead + vcol] = S[k];
    }
}

}  // namespace

int launch_tokenwise(const FwdParams &p, cudaStream_t stream)
{
    const int64_t ctas = p.N * p.H;
    if (ctas <= 0) return 0;
    if (ctas > (int64_t)INT32_MAX) return KDA_ERR_SHAPE;
    tokenwise_kernel<<<(unsigned)ctas, 128, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 1 : KDA_ERR_CUDA;
}

}  // namespace kda
