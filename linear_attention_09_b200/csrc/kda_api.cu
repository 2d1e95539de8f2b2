// Host side of libkda.so: argument validation, kernel dispatch and the
// host-buffer (end-to-end) entry point.  See include/kda.h for the contract.
#include <cmath>
#include <cstring>

#include "kda.h"
#include "kda_internal.cuh"

namespace {

thread_local int g_last_launches = 0;
int g_checks = 0;  // kda_set_checks level

// cu_seqlens check of the debug level: bad |= 1 unless 0 <= cu[0] <= ... <= cu[n] <= rows.
__global__ void check_offsets_kernel(const int64_t *cu, int64_t n, int64_t rows, int *bad)
{
    for (int64_t i = threadIdx.x; i <= n; i += blockDim.x) {
        const int64_t c = cu[i];
        if (c < 0 || c > rows || (i > 0 && cu[i - 1] > c)) atomicOr(bad, 1);
    }
}

// Runs the check on `stream` and waits for it; KDA_OK, KDA_ERR_SEQLENS or KDA_ERR_CUDA.
int check_offsets(const int64_t *cu, int64_t n, int64_t rows, cudaStream_t stream)
{
    int *bad = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void **>(&bad), sizeof(int), stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    int host = 0;
    bool ok = cudaMemsetAsync(bad, 0, sizeof(int), stream) == cudaSuccess;
    if (ok) {
        check_offsets_kernel<<<1, 256, 0, stream>>>(cu, n, rows, bad);
        ok = cudaGetLastError() == cudaSuccess &&
             cudaMemcpyAsync(&host, bad, sizeof(int), cudaMemcpyDeviceToHost, stream) == cudaSuccess;
    }
    ok = (cudaFreeAsync(bad, stream) == cudaSuccess) && ok;
    ok = ok && cudaStreamSynchronize(stream) == cudaSuccess;
    if (!ok) return KDA_ERR_CUDA;
    return host ? KDA_ERR_SEQLENS : KDA_OK;
}

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

// The validation and device check above, for the other host files of the library.
namespace kda {
int validate_args(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  float scale, const float *A_log, const float *dt_bias, float lower_bound,
                  const void *init, int init_dtype, const void *final_state, const int64_t *cu,
                  int64_t num_seqs, const void *out, int64_t B, int64_t T, int64_t H, int64_t K,
                  int64_t V, int64_t *N_out)
{
    return validate(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, init, init_dtype,
                    final_state, cu, num_seqs, out, B, T, H, K, V, N_out);
}

int device_supported() { return check_device(); }
}  // namespace kda

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
    case KDA_ERR_SEQLENS: return "cu_seqlens must be non-decreasing within [0, B*T] (device check)";
    case KDA_ERR_ARG: return "argument outside its documented range";
    default: return "unknown kda error code";
    }
}

extern "C" int kda_last_launch_count(void) { return g_last_launches; }

extern "C" int kda_set_checks(int level)
{
    const int old = g_checks;
    g_checks = level;
    return old;
}

extern "C" int kda_device_status(int reset) { return kda::chunked_device_error(reset != 0); }

extern "C" int kda_inject_error(int code) { return kda::chunked_inject_error(code); }

extern "C" int kda_set_schedule(int mode) { return kda::chunked_set_schedule(mode); }

extern "C" int kda_last_schedule(void) { return kda::chunked_last_schedule(); }

extern "C" int kda_set_bwd_schedule(int mode) { return kda::bwd_set_schedule(mode); }

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
    if (g_checks && cu_seqlens &&
        (rc = check_offsets(cu_seqlens, N, B * T, reinterpret_cast<cudaStream_t>(stream))) != KDA_OK)
        return rc;
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

extern "C" int kda_decode_ex(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                             const kda_bf16 *g, const kda_bf16 *beta, float scale,
                             const float *A_log, const float *dt_bias, float lower_bound,
                             const void *state_in, int state_in_dtype, void *state_out,
                             int state_out_dtype, int state_layout, kda_bf16 *out, int64_t N,
                             int64_t H, int64_t K, int64_t V, kda_stream_t stream)
{
    if (K != kda::kHead || V != kda::kHead) return KDA_ERR_HEAD_DIM;
    if (N < 0 || H < 1 || N > (int64_t(1) << 40) / H || N * H > (int64_t(1) << 31) - 1)
        return KDA_ERR_SHAPE;
    if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_LOWER_BOUND;
    if (!std::isfinite(scale)) return KDA_ERR_SCALE;
    if (state_layout != KDA_LAYOUT_KV && state_layout != KDA_LAYOUT_VK) return KDA_ERR_LAYOUT;
    const auto dtype_ok = [](int d) { return d == KDA_STATE_F32 || d == KDA_STATE_BF16; };
    if (!dtype_ok(state_in_dtype) || !dtype_ok(state_out_dtype)) return KDA_ERR_STATE_DTYPE;
    // an update in place needs one element type
    if (state_in == state_out && state_in_dtype != state_out_dtype) return KDA_ERR_STATE_DTYPE;
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
    p.in_dtype = state_in_dtype;
    p.out_dtype = state_out_dtype;
    p.state_layout = state_layout;
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

extern "C" int kda_decode(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                          const kda_bf16 *g, const kda_bf16 *beta, float scale,
                          const float *A_log, const float *dt_bias, float lower_bound,
                          const float *state_in, float *state_out, kda_bf16 *out, int64_t N,
                          int64_t H, int64_t K, int64_t V, kda_stream_t stream)
{
    return kda_decode_ex(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, state_in,
                         KDA_STATE_F32, state_out, KDA_STATE_F32, KDA_LAYOUT_KV, out, N, H, K, V,
                         stream);
}

extern "C" size_t kda_bwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                         int64_t num_seqs)
{
    if (K != kda::kHead || V != kda::kHead || B < 1 || T < 0 || H < 1) return 0;
    const int64_t N = num_seqs > 0 ? num_seqs : B;
    return kda::bwd_layout(B * T, N, H, nullptr);
}

extern "C" int kda_bwd(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
                       const kda_bf16 *beta, float scale, const float *A_log,
                       const float *dt_bias, float lower_bound, const void *initial_state,
                       int initial_state_dtype, const kda_bf16 *d_out,
                       const float *d_final_state, const int64_t *cu_seqlens, int64_t num_seqs,
                       float *dq, float *dk, float *dv, float *dg, float *dbeta, float *dA_log,
                       float *ddt_bias, float *d_initial_state, void *workspace,
                       size_t workspace_bytes, int64_t B, int64_t T, int64_t H, int64_t K,
                       int64_t V, kda_stream_t stream)
{
    int64_t N = 0;
    int rc = validate(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state,
                      initial_state_dtype, nullptr, cu_seqlens, num_seqs, d_out, B, T, H, K, V,
                      &N);
    if (rc != KDA_OK) return rc;
    const bool any_tokens = B * T > 0;
    if (any_tokens && (!dq || !dk || !dv || !dg || !dbeta)) return KDA_ERR_NULL;
    if (!dA_log || !ddt_bias || !A_log || !dt_bias) return KDA_ERR_NULL;
    if (!aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(dg, 16) ||
        !aligned(dbeta, 4) || !aligned(dA_log, 4) || !aligned(ddt_bias, 4) ||
        !aligned(d_final_state, 4) || !aligned(d_initial_state, 4))
        return KDA_ERR_ALIGN;
    kda::BwdLayout lay{};
    const size_t need = kda::bwd_layout(B * T, N, H, &lay);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return KDA_ERR_ALIGN;
    if ((rc = check_device()) != KDA_OK) return rc;
    if (g_checks && cu_seqlens &&
        (rc = check_offsets(cu_seqlens, N, B * T, reinterpret_cast<cudaStream_t>(stream))) != KDA_OK)
        return rc;
    kda::BwdParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16 *>(q);
    p.k = reinterpret_cast<const __nv_bfloat16 *>(k);
    p.v = reinterpret_cast<const __nv_bfloat16 *>(v);
    p.g = reinterpret_cast<const __nv_bfloat16 *>(g);
    p.beta = reinterpret_cast<const __nv_bfloat16 *>(beta);
    p.dout = reinterpret_cast<const __nv_bfloat16 *>(d_out);
    p.A_log = A_log;
    p.dt_bias = dt_bias;
    p.init = initial_state;
    p.init_dtype = initial_state_dtype;
    p.dfinal = d_final_state;
    p.cu = cu_seqlens;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dg = dg;
    p.dbeta = dbeta;
    p.dA_log = dA_log;
    p.ddt_bias = ddt_bias;
    p.dinit = d_initial_state;
    char *ws = static_cast<char *>(workspace);
    p.ckpt = reinterpret_cast<float *>(ws);
    p.scratch = reinterpret_cast<float *>(ws + lay.ckpt_bytes);
    p.part = reinterpret_cast<float *>(ws + lay.ckpt_bytes + lay.scratch_bytes);
    p.scale = scale;
    p.lower_bound = lower_bound;
    p.B = B;
    p.T = T;
    p.H = H;
    p.N = N;
    const int n = kda::launch_backward(p, lay, reinterpret_cast<cudaStream_t>(stream));
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

namespace {

// Pieces of a host-buffer call: contiguous token ranges with their contiguous state
// ranges (batch entries, or consecutive sequences of a varlen batch of about equal
// token counts), so that the copies of one piece overlap the kernel of another.
struct Piece {
    int64_t tok0, toks;  // rows of the [tokens, H, *] tensors
    int64_t seq0, seqs;  // states [seq0, seq0 + seqs)
};

int plan_pieces(int64_t B, int64_t T, const int64_t *cu_host, int64_t num_seqs, Piece *out,
                int max_pieces)
{
    int n = 0;
    if (!cu_host) {
        const int64_t per = (B + max_pieces - 1) / max_pieces;
        for (int64_t b = 0; b < B; b += per) {
            const int64_t nb = (B - b < per) ? B - b : per;
            out[n++] = Piece{b * T, nb * T, b, nb};
        }
        return n;
    }
    const int64_t total = cu_host[num_seqs] - cu_host[0];
    const int64_t target = (total + max_pieces - 1) / max_pieces;
    int64_t s0 = 0;
    while (s0 < num_seqs) {
        int64_t s1 = s0 + 1;
        while (s1 < num_seqs && cu_host[s1] - cu_host[s0] < target && n < max_pieces - 1) ++s1;
        if (n == max_pieces - 1) s1 = num_seqs;
        out[n++] = Piece{cu_host[s0], cu_host[s1] - cu_host[s0], s0, s1 - s0};
        s0 = s1;
    }
    return n;
}

// Helper streams and events of the pipelined host path, per host thread and device
// (created once; a thread's calls on one device are serialised by the final sync).
struct HostPipe {
    cudaStream_t comp = nullptr, d2h = nullptr;
    cudaEvent_t ev[2 * 8 + 1] = {};
    bool ok = false;
};

HostPipe *host_pipe()
{
    static thread_local HostPipe pipes[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    HostPipe &hp = pipes[dev];
    if (!hp.ok) {
        if (cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess)
            return nullptr;
        for (auto &e : hp.ev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        hp.ok = true;
    }
    return &hp;
}

}  // namespace

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
    // cu_seqlens is in host memory here, so it is checked before anything uses it: the
    // piece plan and the copy offsets come from it
    if (cu_seqlens) {
        const int64_t rows = B * T;
        for (int64_t i = 0; i <= num_seqs; ++i) {
            const int64_t c = cu_seqlens[i];
            if (c < 0 || c > rows || (i > 0 && cu_seqlens[i - 1] > c)) return KDA_ERR_SEQLENS;
        }
    }
    if ((rc = check_device()) != KDA_OK) return rc;
    const HostSizes s = host_sizes(B, T, H, N, initial_state_dtype, final_state != nullptr,
                                   cu_seqlens != nullptr);
    if (!workspace || workspace_bytes < host_total(s) || !aligned(workspace, 256))
        return KDA_ERR_WORKSPACE;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    HostPipe *hp = host_pipe();
    if (!hp) return KDA_ERR_CUDA;
    char *w = static_cast<char *>(workspace);
    auto take = [&](size_t bytes) {
        char *r = w;
        w += round_up(bytes, 256);
        return r;
    };
    char *dq = take(s.qk), *dk = take(s.qk), *dg = take(s.qk), *dv = take(s.vv),
         *dout = take(s.vv), *dbeta = take(s.beta), *dalog = take(s.alog), *ddt = take(s.dt),
         *dinit = take(s.init), *dfin = take(s.fin), *dcu = take(s.cu);
    auto copy = [&](void *dst, const void *src, size_t n, cudaMemcpyKind kind, cudaStream_t on) {
        return n == 0 || cudaMemcpyAsync(dst, src, n, kind, on) == cudaSuccess;
    };
    const size_t row = (size_t)H * kda::kHead * 2;                 // bytes per token row
    const size_t st_in = s.init / (size_t)(N > 0 ? N : 1), st_out = s.fin / (size_t)(N > 0 ? N : 1);
    // parameters first, then the pieces: copy in (stream st) -> kernel (comp) -> copy out (d2h)
    if (!copy(dalog, A_log, s.alog, cudaMemcpyHostToDevice, st) ||
        !copy(ddt, dt_bias, s.dt, cudaMemcpyHostToDevice, st) ||
        !copy(dcu, cu_seqlens, s.cu, cudaMemcpyHostToDevice, st))
        return KDA_ERR_CUDA;
    Piece pcs[8];
    const int np = (B * T == 0) ? 0 : plan_pieces(B, T, cu_seqlens, num_seqs, pcs, 8);
    int launches = 0;
    for (int i = 0; i < np; ++i) {
        const Piece &pc = pcs[i];
        const size_t o = (size_t)pc.tok0 * row, nb = (size_t)pc.toks * row;
        const size_t ob = (size_t)pc.tok0 * H * 2, nbb = (size_t)pc.toks * H * 2;
        if (!copy(dq + o, (const char *)q + o, nb, cudaMemcpyHostToDevice, st) ||
            !copy(dk + o, (const char *)k + o, nb, cudaMemcpyHostToDevice, st) ||
            !copy(dg + o, (const char *)g + o, nb, cudaMemcpyHostToDevice, st) ||
            !copy(dv + o, (const char *)v + o, nb, cudaMemcpyHostToDevice, st) ||
            !copy(dbeta + ob, (const char *)beta + ob, nbb, cudaMemcpyHostToDevice, st) ||
            !copy(dinit + pc.seq0 * st_in, (const char *)initial_state + pc.seq0 * st_in,
                  pc.seqs * st_in, cudaMemcpyHostToDevice, st) ||
            cudaEventRecord(hp->ev[2 * i], st) != cudaSuccess ||
            cudaStreamWaitEvent(hp->comp, hp->ev[2 * i], 0) != cudaSuccess)
            return KDA_ERR_CUDA;
        // the piece as its own call: a batch slice, or a range of varlen sequences
        // (cu_seqlens holds absolute token offsets, so only its start moves)
        const bool varlen = cu_seqlens != nullptr;
        rc = kda_fwd(reinterpret_cast<const kda_bf16 *>(varlen ? dq : dq + o),
                     reinterpret_cast<const kda_bf16 *>(varlen ? dk : dk + o),
                     reinterpret_cast<const kda_bf16 *>(varlen ? dv : dv + o),
                     reinterpret_cast<const kda_bf16 *>(varlen ? dg : dg + o),
                     reinterpret_cast<const kda_bf16 *>(varlen ? dbeta : dbeta + ob), scale,
                     reinterpret_cast<const float *>(dalog), reinterpret_cast<const float *>(ddt),
                     lower_bound, initial_state ? dinit + pc.seq0 * st_in : nullptr,
                     initial_state_dtype,
                     final_state ? reinterpret_cast<float *>(dfin + pc.seq0 * st_out) : nullptr,
                     varlen ? reinterpret_cast<const int64_t *>(dcu) + pc.seq0 : nullptr,
                     varlen ? pc.seqs : 0,
                     reinterpret_cast<kda_bf16 *>(varlen ? dout : dout + o),
                     varlen ? 1 : pc.seqs, varlen ? B * T : T, H, K, V,
                     reinterpret_cast<kda_stream_t>(hp->comp));
        if (rc != KDA_OK) return rc;
        launches += g_last_launches;
        if (cudaEventRecord(hp->ev[2 * i + 1], hp->comp) != cudaSuccess ||
            cudaStreamWaitEvent(hp->d2h, hp->ev[2 * i + 1], 0) != cudaSuccess ||
            !copy((char *)out + o, dout + o, nb, cudaMemcpyDeviceToHost, hp->d2h) ||
            !copy((char *)final_state + pc.seq0 * st_out, dfin + pc.seq0 * st_out,
                  final_state ? pc.seqs * st_out : 0, cudaMemcpyDeviceToHost, hp->d2h))
            return KDA_ERR_CUDA;
    }
    if (np == 0 && final_state) {  // no tokens: the final state is the initial one
        if (!copy(dinit, initial_state, s.init, cudaMemcpyHostToDevice, st)) return KDA_ERR_CUDA;
        rc = kda_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, scale, nullptr, nullptr,
                     lower_bound, initial_state ? dinit : nullptr, initial_state_dtype,
                     reinterpret_cast<float *>(dfin),
                     cu_seqlens ? reinterpret_cast<const int64_t *>(dcu) : nullptr,
                     cu_seqlens ? num_seqs : 0, nullptr, B, T, H, K, V, stream);
        if (rc != KDA_OK) return rc;
        launches = g_last_launches;
        if (!copy(final_state, dfin, s.fin, cudaMemcpyDeviceToHost, st)) return KDA_ERR_CUDA;
    }
    g_last_launches = launches;
    // the caller's stream waits for the copies out, then everything is complete
    if (cudaEventRecord(hp->ev[16], hp->d2h) != cudaSuccess ||
        cudaStreamWaitEvent(st, hp->ev[16], 0) != cudaSuccess)
        return KDA_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
