// Host side of libkda.so: argument validation, kernel dispatch and the
// host-buffer (end-to-end) entry point.  See include/kda.h for the contract.
#include <cmath>
#include <cstring>

#include "kda.h"
#include "kda_internal.cuh"

namespace {

thread_local int g_last_launches = 0;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Compute capability check, cached per device (the product path runs on sm_100 only).
int check_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return KDA_ERR_DEVICE;
    }
    static int cached[64];  // 0 unknown, 1 ok, -1 unsupported
    if (dev < 64 && cached[dev] != 0) return cached[dev] > 0 ? KDA_OK : KDA_ERR_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_DEVICE;
    }
    const int ok = (major == 10) ? 1 : -1;
    if (dev < 64) cached[dev] = ok;
    return ok > 0 ? KDA_OK : KDA_ERR_DEVICE;
}

// Validation shared by kda_fwd and kda_fwd_host (pointer kinds aside).
int validate(const void *q, const void *k, const void *v, const void *g, const void *beta,
             float scale, const float *A_log, const float *dt_bias, float lower_bound,
             const void *init, int init_dtype, const void *final_state, const int64_t *cu,
             int64_t num_seqs, const void *out, int64_t B, int64_t T, int64_t H, int64_t K,
             int64_t V, int64_t *N_out)
{
    if (K != kda::kHead || V != kda::kHead) return KDA_ERR_HEAD_DIM;
    if (B < 1 || T < 0 || H < 1) return KDA_ERR_SHAPE;
    // keep every element index comfortably inside int64
    if (B > (int64_t(1) << 40) / (T + 1) || H > 65536 || B * (T + 1) * H > (int64_t(1) << 40))
        return KDA_ERR_SHAPE;
    if (cu && B != 1) return KDA_ERR_VARLEN_BATCH;
    if (cu && num_seqs < 1) return KDA_ERR_NUM_SEQS;
    const int64_t N = cu ? num_seqs : B;
    if (N * H > (int64_t(1) << 31) - 1) return KDA_ERR_SHAPE;
    if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_LOWER_BOUND;
    if (!std::isfinite(scale)) return KDA_ERR_SCALE;
    if (init_dtype != KDA_STATE_NONE && init_dtype != KDA_STATE_F32 && init_dtype != KDA_STATE_BF16)
        return KDA_ERR_STATE_DTYPE;
    if ((init != nullptr) != (init_dtype != KDA_STATE_NONE)) return KDA_ERR_STATE_DTYPE;
    const bool any_tokens = B * T > 0;
    if (any_tokens && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_NULL;
    if (any_tokens && (!A_log || !dt_bias)) return KDA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
        !aligned(out, 16) || !aligned(beta, 2) || !aligned(A_log, 4) || !aligned(dt_bias, 16) ||
        !aligned(init, 16) || !aligned(final_state, 16) || !aligned(cu, 8))
        return KDA_ERR_ALIGN;
    *N_out = N;
    return KDA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Byte sizes of every buffer of a call (for the host entry point's workspace).
struct HostSizes {
    size_t qk, vv, beta, alog, dt, init, fin, cu;
};

HostSizes host_sizes(int64_t B, int64_t T, int64_t H, int64_t N, int init_dtype, int want_final,
                     bool varlen)
{
    HostSizes s{};
    const size_t toks = (size_t)B * (size_t)T * (size_t)H;
    s.qk = toks * kda::kHead * 2;
    s.vv = toks * kda::kHead * 2;
    s.beta = toks * 2;
    s.alog = (size_t)H * 4;
    s.dt = (size_t)H * kda::kHead * 4;
    const size_t st = (size_t)N * H * kda::kHead * kda::kHead;
    s.init = init_dtype == KDA_STATE_F32 ? st * 4 : init_dtype == KDA_STATE_BF16 ? st * 2 : 0;
    s.fin = want_final ? st * 4 : 0;
    s.cu = varlen ? (size_t)(N + 1) * 8 : 0;
    return s;
}

size_t host_total(const HostSizes &s)
{
    const size_t a = 256;
    return 3 * round_up(s.qk, a) + 2 * round_up(s.vv, a) + round_up(s.beta, a) +
           round_up(s.alog, a) + round_up(s.dt, a) + round_up(s.init, a) + round_up(s.fin, a) +
           round_up(s.cu, a);
}

}  // namespace

extern "C" const char *kda_strerror(int code)
{
    switch (code) {
    case KDA_OK: return "ok";
    case KDA_ERR_HEAD_DIM: return "K and V must both be 128";
    case KDA_ERR_NULL: return "a required pointer is NULL";
    case KDA_ERR_VARLEN_BATCH: return "cu_seqlens requires B == 1";
    case KDA_ERR_NUM_SEQS: return "cu_seqlens requires num_seqs >= 1";
    case KDA_ERR_LOWER_BOUND: return "lower_bound must lie in [-5, 0]";
    case KDA_ERR_STATE_DTYPE: return "bad initial_state dtype / pointer combination";
    case KDA_ERR_ALIGN: return "misaligned pointer (16 bytes for tensors, 8 for cu_seqlens)";
    case KDA_ERR_SHAPE: return "bad shape (B >= 1, T >= 0, H >= 1, sizes within range)";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_DEVICE: return "no usable sm_100 (B200) device";
    case KDA_ERR_SCALE: return "scale must be finite";
    case KDA_ERR_LAYOUT: return "state_layout must be KDA_LAYOUT_KV or KDA_LAYOUT_VK";
    default: return "unknown kda error code";
    }
}

extern "C" int kda_last_launch_count(void) { return g_last_launches; }

extern "C" int kda_device_status(int reset) { return kda::chunked_device_error(reset != 0); }

extern "C" int kda_fwd_ex(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                          const kda_bf16 *g, const kda_bf16 *beta, float scale,
                          const float *A_log, const float *dt_bias, float lower_bound,
                          const void *initial_state, int initial_state_dtype, void *final_state,
                          int final_state_dtype, int state_layout, const int64_t *cu_seqlens,
                          int64_t num_seqs, kda_bf16 *out, int64_t B, int64_t T, int64_t H,
                          int64_t K, int64_t V, kda_stream_t stream)
{
    int64_t N = 0;
    int rc = validate(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state,
                      initial_state_dtype, final_state, cu_seqlens, num_seqs, out, B, T, H, K, V,
                      &N);
    if (rc != KDA_OK) return rc;
    if (state_layout != KDA_LAYOUT_KV && state_layout != KDA_LAYOUT_VK) return KDA_ERR_LAYOUT;
    if (final_state && final_state_dtype != KDA_STATE_F32 && final_state_dtype != KDA_STATE_BF16)
        return KDA_ERR_STATE_DTYPE;
    if ((rc = check_device()) != KDA_OK) return rc;
    kda::FwdParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    p.k = reinterpret_cast<const __nv_bfloat16 *>(k);
    p.v = reinterpret_cast<const __nv_bfloat16 *>(v);
    p.g = reinterpret_cast<const __nv_bfloat16 *>(g);
    p.beta = reinterpret_cast<const __nv_bfloat16 *>(beta);
    p.A_log = A_log;
    p.dt_bias = dt_bias;
    p.init = initial_state;
    p.init_dtype = initial_state_dtype;
    p.final_state = final_state;
    p.final_dtype = final_state_dtype;
    p.state_layout = state_layout;
    p.cu = cu_seqlens;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.scale = scale;
    p.lower_bound = lower_bound;
    p.B = B;
    p.T = T;
    p.H = H;
    p.N = N;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Nothing to do at all: no tokens and no state requested.
    if (B * T == 0 && !final_state) {
        g_last_launches = 0;
        return KDA_OK;
    }
    const int n = kda::launch_chunked(p, st);
    if (n < 0) return n;
    g_last_launches = n;
    return KDA_OK;
}

extern "C" int kda_fwd(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
                       const kda_bf16 *beta, float scale, const float *A_log,
                       const float *dt_bias, float lower_bound, const void *initial_state,
                       int initial_state_dtype, float *final_state, const int64_t *cu_seqlens,
                       int64_t num_seqs, kda_bf16 *out, int64_t B, int64_t T, int64_t H,
                       int64_t K, int64_t V, kda_stream_t stream)
{
    return kda_fwd_ex(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state,
                      initial_state_dtype, final_state, KDA_STATE_F32, KDA_LAYOUT_KV, cu_seqlens,
                      num_seqs, out, B, T, H, K, V, stream);
}

extern "C" int kda_decode(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                          const kda_bf16 *g, const kda_bf16 *beta, float scale,
                          const float *A_log, const float *dt_bias, float lower_bound,
                          const float *state_in, float *state_out, kda_bf16 *out, int64_t N,
                          int64_t H, int64_t K, int64_t V, kda_stream_t stream)
{
    if (K != kda::kHead || V != kda::kHead) return KDA_ERR_HEAD_DIM;
    if (N < 0 || H < 1 || N > (int64_t(1) << 40) / H || N * H > (int64_t(1) << 31) - 1)
        return KDA_ERR_SHAPE;
    if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_LOWER_BOUND;
    if (!std::isfinite(scale)) return KDA_ERR_SCALE;
    if (N == 0) {
        g_last_launches = 0;
        return KDA_OK;
    }
    if (!q || !k || !v || !g || !beta || !A_log || !dt_bias || !state_in || !state_out || !out)
        return KDA_ERR_NULL;
    if (!aligned(q, 2) || !aligned(k, 2) || !aligned(v, 2) || !aligned(g, 2) || !aligned(beta, 2) ||
        !aligned(out, 2) || !aligned(A_log, 4) || !aligned(dt_bias, 4) || !aligned(state_in, 16) ||
        !aligned(state_out, 16))
        return KDA_ERR_ALIGN;
    int rc = check_device();
    if (rc != KDA_OK) return rc;
    kda::DecodeParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    p.k = reinterpret_cast<const __nv_bfloat16 *>(k);
    p.v = reinterpret_cast<const __nv_bfloat16 *>(v);
    p.g = reinterpret_cast<const __nv_bfloat16 *>(g);
    p.beta = reinterpret_cast<const __nv_bfloat16 *>(beta);
    p.A_log = A_log;
    p.dt_bias = dt_bias;
    p.state_in = state_in;
    p.state_out = state_out;
    p.out = reinterpret_cast<__nv_bfloat16 *>(out);
    p.scale = scale;
    p.lower_bound = lower_bound;
    p.N = N;
    p.H = H;
    const int n = kda::launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
    if (n < 0) return n;
    g_last_launches = n;
    return KDA_OK;
}

extern "C" size_t kda_fwd_host_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K,
                                              int64_t V, int64_t num_seqs,
                                              int initial_state_dtype, int want_final_state)
{
    if (K != kda::kHead || V != kda::kHead || B < 1 || T < 0 || H < 1) return 0;
    const bool varlen = num_seqs > 0;
    const int64_t N = varlen ? num_seqs : B;
    return host_total(host_sizes(B, T, H, N, initial_state_dtype, want_final_state, varlen));
}

extern "C" int kda_fwd_host(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                            const kda_bf16 *g, const kda_bf16 *beta, float scale,
                            const float *A_log, const float *dt_bias, float lower_bound,
                            const void *initial_state, int initial_state_dtype,
                            float *final_state, const int64_t *cu_seqlens, int64_t num_seqs,
                            kda_bf16 *out, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream)
{
    int64_t N = 0;
    int rc = validate(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state,
                      initial_state_dtype, final_state, cu_seqlens, num_seqs, out, B, T, H, K, V,
                      &N);
    if (rc != KDA_OK) return rc;
    if ((rc = check_device()) != KDA_OK) return rc;
    const HostSizes s = host_sizes(B, T, H, N, initial_state_dtype, final_state != nullptr,
                                   cu_seqlens != nullptr);
    if (!workspace || workspace_bytes < host_total(s) || !aligned(workspace, 256))
        return KDA_ERR_WORKSPACE;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    auto take = [&](size_t bytes) {
        char *r = w;
        w += round_up(bytes, 256);
        return r;
    };
    char *dq = take(s.qk), *dk = take(s.qk), *dg = take(s.qk), *dv = take(s.vv),
         *dout = take(s.vv), *dbeta = take(s.beta), *dalog = take(s.alog), *ddt = take(s.dt),
         *dinit = take(s.init), *dfin = take(s.fin), *dcu = take(s.cu);
    auto h2d = [&](void *dst, const void *src, size_t n) {
        return n == 0 || cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, st) == cudaSuccess;
    };
    if (!h2d(dq, q, s.qk) || !h2d(dk, k, s.qk) || !h2d(dg, g, s.qk) || !h2d(dv, v, s.vv) ||
        !h2d(dbeta, beta, s.beta) || !h2d(dalog, A_log, s.alog) || !h2d(ddt, dt_bias, s.dt) ||
        !h2d(dinit, initial_state, s.init) || !h2d(dcu, cu_seqlens, s.cu))
        return KDA_ERR_CUDA;
    rc = kda_fwd(reinterpret_cast<const kda_bf16 *>(dq), reinterpret_cast<const kda_bf16 *>(dk),
                 reinterpret_cast<const kda_bf16 *>(dv), reinterpret_cast<const kda_bf16 *>(dg),
                 reinterpret_cast<const kda_bf16 *>(dbeta), scale,
                 reinterpret_cast<const float *>(dalog), reinterpret_cast<const float *>(ddt),
                 lower_bound, initial_state ? dinit : nullptr, initial_state_dtype,
                 final_state ? reinterpret_cast<float *>(dfin) : nullptr,
                 cu_seqlens ? reinterpret_cast<const int64_t *>(dcu) : nullptr, num_seqs,
                 reinterpret_cast<kda_bf16 *>(dout), B, T, H, K, V, stream);
    if (rc != KDA_OK) return rc;
    if (s.vv && cudaMemcpyAsync(out, dout, s.vv, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (s.fin &&
        cudaMemcpyAsync(final_state, dfin, s.fin, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return KDA_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
