// kda_bwd_noalloc: the backward pass for callers that cannot allocate device memory.
//
// kda_bwd needs a workspace (the state before every 64-token chunk, 1 MB of
// sub-chunk states per CTA, and per-(sequence, head) partial sums), which the caller
// normally allocates.  Some callers cannot: code that runs inside a memory pool or
// allocator that must not be re-entered, a plugin of a host framework that hands it
// tensors but no allocator, or a process whose memory budget is fixed before the
// first call.  For them this entry point takes its workspace from a fixed array in
// the library's own device memory, kNoallocBytes long, which every GPU that loads
// the library holds until the process exits.
//
// There is no counterpart of this entry point on the FlashKDA pages; it is a
// deployment convenience of this library.
#include <mutex>

#include "kda.h"
#include "kda_internal.cuh"

namespace {

constexpr size_t kNoallocBytes = KDA_BWD_NOALLOC_MAX_BYTES;

// The workspace of every kda_bwd_noalloc call (shared: calls whose work overlaps on
// the GPU race on it).  Nothing in it has to start at zero: the backward kernel
// writes every checkpoint, sub-chunk state and partial sum before it reads it.
static __device__ __align__(256) unsigned char g_noalloc_ws[kNoallocBytes];

// Device address of g_noalloc_ws on the current device.  In host code the array's
// name only stands for the variable; the address a kernel can use comes from
// cudaGetSymbolAddress, taken once per device with that device current (the first
// kda_bwd_noalloc call on the device does it, which loads this module there).
void *noalloc_workspace(int *rc)
{
    static std::mutex mu;
    static void *addr[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        *rc = KDA_ERR_DEVICE;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) {
            cudaGetLastError();
            *rc = KDA_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    *rc = KDA_OK;
    return addr[dev];
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int kda_bwd_noalloc(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v,
                               const kda_bf16 *g, const kda_bf16 *beta, float scale,
                               const float *A_log, const float *dt_bias, float lower_bound,
                               const void *initial_state, int initial_state_dtype,
                               const kda_bf16 *d_out, const float *d_final_state,
                               const int64_t *cu_seqlens, int64_t num_seqs, float *dq, float *dk,
                               float *dv, float *dg, float *dbeta, float *dA_log,
                               float *ddt_bias, float *d_initial_state, int64_t B, int64_t T,
                               int64_t H, int64_t K, int64_t V, kda_stream_t stream)
{
    // the argument checks of kda_bwd, in the same order
    int64_t N = 0;
    int rc = kda::validate_args(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound,
                                initial_state, initial_state_dtype, nullptr, cu_seqlens,
                                num_seqs, d_out, B, T, H, K, V, &N);
    if (rc != KDA_OK) return rc;
    if (B * T > 0 && (!dq || !dk || !dv || !dg || !dbeta)) return KDA_ERR_NULL;
    if (!dA_log || !ddt_bias || !A_log || !dt_bias) return KDA_ERR_NULL;
    if (!aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(dg, 16) ||
        !aligned(dbeta, 4) || !aligned(dA_log, 4) || !aligned(ddt_bias, 4) ||
        !aligned(d_final_state, 4) || !aligned(d_initial_state, 4))
        return KDA_ERR_ALIGN;
    kda::BwdLayout lay{};
    if (kda::bwd_layout(B * T, N, H, &lay) > kNoallocBytes) return KDA_ERR_WORKSPACE;
    if ((rc = kda::device_supported()) != KDA_OK) return rc;
    char *ws = static_cast<char *>(noalloc_workspace(&rc));
    if (rc != KDA_OK) return rc;

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
    return n < 0 ? n : KDA_OK;
}
