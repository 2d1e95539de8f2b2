// Internal declarations shared by the libkda host code and its kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace kda {

constexpr int kHead = 128;  // K = V = 128 (the pages' only supported head size)

// Arguments of one forward call, already validated on the host.
struct FwdParams {
    const __nv_bfloat16 *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    const void *init;        // fp32 or bf16 state per (sequence, head) or nullptr
    int init_dtype;          // KDA_STATE_*
    void *final_state;       // fp32 or bf16 state per (sequence, head) or nullptr
    int final_dtype;         // KDA_STATE_F32 / KDA_STATE_BF16
    int state_layout;        // KDA_LAYOUT_KV / KDA_LAYOUT_VK (both states)
    const int64_t *cu;       // [N+1] or nullptr
    __nv_bfloat16 *out;
    float scale, lower_bound;
    int64_t B, T, H, N;      // N = number of sequences
    uint32_t epoch;          // set by the launcher: tags the launch's error word
    // Backward pass only: when set, the launch stores the fp32 state S[k][v] before
    // every 64-token chunk of unit (sequence s, head h) starting at token bos, chunk n,
    // at slot (bos / 64 + s + n) * H + h (64 KB each), and writes no output.
    float *ckpt;
};

// One decode step: one token per (sequence, head), state updated in HBM.
struct DecodeParams {
    const __nv_bfloat16 *q, *k, *v, *g, *beta;  // [N,H,K], [N,H,K], [N,H,V], [N,H,K], [N,H]
    const float *A_log, *dt_bias;
    const void *state_in;    // [N,H,K,V] (S[k][v]) or [N,H,V,K] (S[v][k]), fp32 or bf16
    void *state_out;         // same layout, fp32 or bf16; may equal state_in (same dtype)
    int in_dtype, out_dtype; // KDA_STATE_F32 / KDA_STATE_BF16
    int state_layout;        // KDA_LAYOUT_KV / KDA_LAYOUT_VK
    __nv_bfloat16 *out;      // [N,H,V]
    float scale, lower_bound;
    int64_t N, H;
};

int launch_decode(const DecodeParams &p, cudaStream_t stream);

// Backward pass: gradients of <dO, out> + <dS_final, S_final>.
struct BwdParams {
    const __nv_bfloat16 *q, *k, *v, *g, *beta, *dout;
    const float *A_log, *dt_bias;
    const void *init;        // fp32 or bf16 initial state or nullptr
    int init_dtype;
    const float *dfinal;     // fp32 [N,H,K,V] or nullptr (zero)
    const int64_t *cu;
    float *dq, *dk, *dv, *dg, *dbeta;  // fp32, layouts of q, k, v, g, beta
    float *dA_log, *ddt_bias;          // fp32 [H], [H,K]
    float *dinit;                      // fp32 [N,H,K,V] or nullptr
    float *ckpt, *scratch, *part;      // workspace regions
    float scale, lower_bound;
    int64_t B, T, H, N;
};

constexpr int kBwdMaxCtas = 148;  // persistent grid of the backward kernel

struct BwdLayout {
    int grid;
    size_t ckpt_bytes, scratch_bytes, part_bytes;
};

// Workspace bytes of a backward call (and the split into regions).
size_t bwd_layout(int64_t total_tokens, int64_t N, int64_t H, BwdLayout *out);
// The backward pass in the schedule set by bwd_set_schedule (KDA_BWD_*): the number of
// kernels enqueued or a negative KDA_ERR_* code.
int launch_backward(const BwdParams &p, const BwdLayout &l, cudaStream_t stream);
int launch_backward_token(const BwdParams &p, const BwdLayout &l, cudaStream_t stream);
int launch_param_reduce(const BwdParams &p, cudaStream_t stream);  // dA_log, ddt_bias
int bwd_set_schedule(int mode);  // the previous mode or KDA_ERR_ARG
size_t bwd_chunked_scratch_bytes_per_cta();

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per device (the
// attribute belongs to the device's context); `done` is the caller's per-device flags.
template <typename Kernel>
inline bool set_smem_limit_once(Kernel kernel, int bytes, int (&done)[64])
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const bool cached = dev >= 0 && dev < 64;
    if (cached && done[dev]) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    if (cached) done[dev] = 1;
    return true;
}

// Host-side argument validation of the forward/backward calls (KDA_OK or a negative
// code; *N_out = number of sequences) and the sm_100 device check, shared by the
// entry points of the library's host files.
int validate_args(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  float scale, const float *A_log, const float *dt_bias, float lower_bound,
                  const void *init, int init_dtype, const void *final_state, const int64_t *cu,
                  int64_t num_seqs, const void *out, int64_t B, int64_t T, int64_t H, int64_t K,
                  int64_t V, int64_t *N_out);
int device_supported();

// Kernel launcher; returns the number of kernels it enqueued (>= 0) or a negative
// KDA_ERR_* code.
int launch_chunked(const FwdParams &p, cudaStream_t stream);
// Error word the chunked kernel sets when a bounded wait gives up (0 = none).
int chunked_device_error(bool reset);
int chunked_inject_error(int code);  // the next launch starts failed with `code`
int chunked_set_schedule(int mode);  // KDA_SCHEDULE_*; the previous mode or KDA_ERR_ARG
int chunked_last_schedule();         // schedule of this thread's last forward launch

}  // namespace kda
