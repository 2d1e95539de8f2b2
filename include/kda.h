/*
 * kda.h -- C ABI of libkda.so, the B200 (sm_100a) Kimi Delta Attention forward pass.
 *
 * The operation (FlashKDA de código abierto de Moonshot AI, 7minutos.es, sections
 * "¿Qué es la atención Kimi Delta...?" and "Debajo del capó: CUTLASS en Hopper";
 * flags from the chunk_kda call on github.zuobiaodaohang.com "FlashKDA：用CUTLASS
 * fused kernel 给 Kimi Delta Attention 提速 3-5 倍", section "作为 FLA 后端的用法"):
 *
 *   for each sequence s and head h, S (K x V, fp32) = initial_state[s,h] or 0;
 *   for each token t of s:
 *     qh = q_t / sqrt(|q_t|^2 + 1e-6),  kh = k_t / sqrt(|k_t|^2 + 1e-6)
 *     b  = sigmoid(beta_t)
 *     lam[c] = max(lower_bound, -exp(A_log[h]) * softplus(g_t[c] + dt_bias[h,c]))
 *     S = (I - b kh kh^T) Diag(exp(lam)) S + b kh v_t^T
 *     out_t = scale * S^T qh
 *   final_state[s,h] = S
 *
 * The pages do not print the gate formula; the one above (natural log,
 * lower_bound in [-5, 0] as the pages state) is this library's reading.
 *
 * Layouts: every tensor is row-major and contiguous (the pages require contiguous
 * inputs on one GPU):
 *   q, k, g      [B, T, H, K]  bf16      v, out  [B, T, H, V]  bf16
 *   beta         [B, T, H]     bf16 (logits; the sigmoid is applied inside)
 *   A_log        [H]           fp32      dt_bias [H, K]        fp32
 *   states       [N, H, K, V]  S[k][v] at ((n*H + h)*K + k)*V + v, N = B, or
 *                               num_seqs with cu_seqlens
 *   cu_seqlens   [num_seqs+1]  int64, cumulative token offsets; requires B == 1,
 *                               cu_seqlens[0] == 0 and cu_seqlens[num_seqs] == T.
 * K = V = 128 is the only head size (the pages' current restriction).
 *
 * Ownership: the caller owns every buffer; the library keeps no pointer after a
 * call returns and allocates no device memory on the kda_fwd path.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 element (raw IEEE bfloat16 bits). */
typedef uint16_t kda_bf16;
/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *kda_stream_t;

/* initial_state element types */
#define KDA_STATE_NONE 0
#define KDA_STATE_F32 1
#define KDA_STATE_BF16 2

/* Return codes.  Every negative code except KDA_ERR_CUDA and KDA_ERR_SEQLENS is
 * detected on the host before anything is launched. */
#define KDA_OK 0
#define KDA_ERR_HEAD_DIM (-1)     /* K != 128 or V != 128 */
#define KDA_ERR_NULL (-2)         /* a required pointer is NULL */
#define KDA_ERR_VARLEN_BATCH (-3) /* cu_seqlens given with B != 1 */
#define KDA_ERR_NUM_SEQS (-4)     /* cu_seqlens given with num_seqs < 1 */
#define KDA_ERR_LOWER_BOUND (-5)  /* lower_bound outside [-5, 0] or NaN */
#define KDA_ERR_STATE_DTYPE (-6)  /* initial_state_dtype not NONE/F32/BF16, or a
                                     state pointer without a matching dtype */
#define KDA_ERR_ALIGN (-7)        /* a pointer is not 16-byte aligned (4 for fp32
                                     vectors, 8 for cu_seqlens, 2 for beta) */
#define KDA_ERR_SHAPE (-8)        /* B < 1, T < 0, H < 1, or sizes overflow */
#define KDA_ERR_CUDA (-9)         /* a CUDA call or launch failed */
#define KDA_ERR_WORKSPACE (-10)   /* workspace missing or too small */
#define KDA_ERR_DEVICE (-11)      /* no usable sm_100 device for this call */
#define KDA_ERR_SCALE (-12)       /* scale is not finite */
#define KDA_ERR_LAYOUT (-13)      /* state_layout is not KV / VK */
#define KDA_ERR_SEQLENS (-14)     /* cu_seqlens is not non-decreasing within [0, B*T]:
                                     always checked by kda_fwd_host (host offsets), by the
                                     device entry points with checks on (kda_set_checks);
                                     nothing was run */
#define KDA_ERR_ARG (-15)         /* an argument outside its documented range */

/* State layouts (kda_fwd_ex).  The FLA call on the pages passes
 * transpose_state_layout=True, i.e. per (sequence, head) the state stored value-major. */
#define KDA_LAYOUT_KV 0 /* S[k][v] at ((n*H + h)*K + k)*V + v   (kda_fwd's layout) */
#define KDA_LAYOUT_VK 1 /* S[v][k] at ((n*H + h)*V + v)*K + k   (transposed)       */

/*
 * kda_fwd -- the forward/prefill pass on device buffers.
 *
 * q, k, v, g, beta, A_log, dt_bias, out: device pointers (layouts above).
 * scale, lower_bound: host scalars (lower_bound in [-5, 0]).
 * initial_state: device pointer or NULL; initial_state_dtype says KDA_STATE_F32
 *   or KDA_STATE_BF16 (KDA_STATE_NONE when NULL).
 * final_state: device fp32 [N,H,K,V] or NULL when not wanted.
 * cu_seqlens: device int64 [num_seqs+1] or NULL (then B sequences of length T).
 *   It is not read on the host (that would need a synchronisation); a sequence
 *   of length 0 returns its initial state (or zeros) as final state and writes
 *   no output; tokens outside [cu_seqlens[0], cu_seqlens[num_seqs]) are not
 *   written.
 * The kernel reads q, k, v, g, beta in tiles of 64 tokens, so the last tile of a
 *   sequence also reads up to 63 rows after it (the next sequence's, or rows that
 *   belong to no sequence).  Those rows are cleared on chip before any use, so
 *   their bits (NaN and Inf included) never reach a result.
 * stream: the work is enqueued on it; the call does not synchronise.
 * T == 0 is valid: only final_state is written.
 * Returns KDA_OK or a negative code (see above).  Never traps the GPU.
 */
int kda_fwd(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
            const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
            float lower_bound, const void *initial_state, int initial_state_dtype,
            float *final_state, const int64_t *cu_seqlens, int64_t num_seqs, kda_bf16 *out,
            int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, kda_stream_t stream);

/*
 * kda_fwd_ex -- kda_fwd with the state variants of the operator statement (FlashKDA de
 * código abierto de Moonshot AI, 7minutos.es, section "Debajo del capó: CUTLASS en
 * Hopper": optional initial and final states in bf16 or fp32; the transposed layout
 * is the transpose_state_layout flag of the chunk_kda call on
 * github.zuobiaodaohang.com, section "作为 FLA 后端的用法").
 *
 * final_state: device pointer or NULL; final_state_dtype is KDA_STATE_F32 or
 *   KDA_STATE_BF16 (bf16 is the fp32 state rounded to nearest even).
 * state_layout: KDA_LAYOUT_KV or KDA_LAYOUT_VK, for both initial and final state.
 * Everything else as kda_fwd; kda_fwd(...) == kda_fwd_ex(..., final_state,
 * KDA_STATE_F32, KDA_LAYOUT_KV, ...).  Extra return code: KDA_ERR_LAYOUT; a
 * final_state_dtype other than F32/BF16 with a final_state gives KDA_ERR_STATE_DTYPE.
 */
int kda_fwd_ex(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
               const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
               float lower_bound, const void *initial_state, int initial_state_dtype,
               void *final_state, int final_state_dtype, int state_layout,
               const int64_t *cu_seqlens, int64_t num_seqs, kda_bf16 *out, int64_t B, int64_t T,
               int64_t H, int64_t K, int64_t V, kda_stream_t stream);

/*
 * kda_fwd_host_workspace_size -- bytes of device memory kda_fwd_host needs for a
 * call of this shape (all inputs, out, and the states it copies).  Returns 0 for
 * invalid sizes.
 */
size_t kda_fwd_host_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                   int64_t num_seqs, int initial_state_dtype,
                                   int want_final_state);

/*
 * kda_fwd_host -- the same pass on HOST buffers (end-to-end path).
 *
 * Every pointer except workspace is a host pointer (pinned memory gives
 * asynchronous copies; pageable memory works but copies synchronously).  The
 * call copies the inputs into `workspace` (a device buffer of at least
 * kda_fwd_host_workspace_size(...) bytes, owned by the caller), runs the pass and
 * copies out (and final_state) back, and synchronises `stream` before returning,
 * so the host buffers are ready on return.  The work is pipelined over up to 8
 * pieces (batch entries, or consecutive varlen sequences of about equal token
 * counts): the copies in of one piece (on `stream`), the kernel of another and the
 * copies out of a third (two library-owned streams per host thread and device)
 * overlap.  Output rows of tokens outside every sequence are not written.
 * cu_seqlens is a host pointer here and is checked before anything is copied: offsets
 * that are not non-decreasing within [0, B*T] give KDA_ERR_SEQLENS.  Same return codes
 * as kda_fwd, plus KDA_ERR_WORKSPACE.
 */
int kda_fwd_host(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
                 const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
                 float lower_bound, const void *initial_state, int initial_state_dtype,
                 float *final_state, const int64_t *cu_seqlens, int64_t num_seqs,
                 kda_bf16 *out, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                 void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_decode -- one decode step: a single new token for each of N sequences, the
 * same operator as kda_fwd with T = 1 and the state carried in HBM between calls
 * (the generation step that follows prefill; FlashKDA pages, 7minutos.es, "¿Qué es
 * la atención Kimi Delta y por qué es importante?").
 *
 *   q, k, g   [N, H, K] bf16     v, out  [N, H, V] bf16     beta  [N, H] bf16
 *   A_log [H], dt_bias [H, K] fp32; scale and lower_bound as kda_fwd
 *   state_in  fp32 [N, H, K, V], S[k][v]; state_out fp32 [N, H, K, V], may be the
 *             same buffer as state_in (update in place)
 * Device pointers; asynchronous on stream.  N == 0 is a no-op.  Returns KDA_OK or a
 * negative code (head size, NULL pointers, alignment: 16 bytes for the states, 2 for
 * the bf16 vectors, 4 for A_log / dt_bias; lower_bound; scale; shape; device).
 */
int kda_decode(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
               const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
               float lower_bound, const float *state_in, float *state_out, kda_bf16 *out,
               int64_t N, int64_t H, int64_t K, int64_t V, kda_stream_t stream);

/*
 * kda_decode_ex -- kda_decode with the state variants of kda_fwd_ex, so that a prefill
 * in either layout or element type hands its final state straight to decode (initial
 * and final states bf16 or fp32: FlashKDA de código abierto de Moonshot AI,
 * 7minutos.es, "Debajo del capó"; the transposed layout is the chunk_kda call's
 * transpose_state_layout on github.zuobiaodaohang.com, "作为 FLA 后端的用法").
 *
 * state_in_dtype / state_out_dtype: KDA_STATE_F32 or KDA_STATE_BF16 (a bf16 state is
 *   promoted exactly; a bf16 result is the fp32 state rounded to nearest even).
 * state_layout: KDA_LAYOUT_KV ([N,H,K,V], S[k][v]) or KDA_LAYOUT_VK ([N,H,V,K]).
 * state_out may equal state_in (update in place) only when the two dtypes are equal,
 *   else KDA_ERR_STATE_DTYPE.  Everything else as kda_decode; kda_decode(...) ==
 *   kda_decode_ex(..., KDA_STATE_F32, ..., KDA_STATE_F32, KDA_LAYOUT_KV, ...).
 */
int kda_decode_ex(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
                  const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
                  float lower_bound, const void *state_in, int state_in_dtype, void *state_out,
                  int state_out_dtype, int state_layout, kda_bf16 *out, int64_t N, int64_t H,
                  int64_t K, int64_t V, kda_stream_t stream);

/*
 * kda_bwd -- backward pass of kda_fwd: the gradients of
 *   L = sum over tokens of <d_out_t, out_t>  +  <d_final_state, final_state>
 * with respect to every input (reverse mode through the recurrence of the FlashKDA
 * pages, 7minutos.es "¿Qué es la atención Kimi Delta...?"; the training step the
 * FLA integration on github.zuobiaodaohang.com, section "作为 FLA 后端的用法", calls
 * for).
 *
 * Inputs: q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state /
 * initial_state_dtype, cu_seqlens / num_seqs, B, T, H, K, V exactly as kda_fwd
 * (states in the S[k][v] layout), and
 *   d_out          [B, T, H, V] bf16   dL/dout
 *   d_final_state  [N, H, K, V] fp32   dL/dS_final, or NULL (zero)
 * Outputs (fp32, device, written by this call):
 *   dq, dk, dg     [B, T, H, K]       dv  [B, T, H, V]       dbeta  [B, T, H]
 *   dA_log         [H]                ddt_bias  [H, K]  (sums over all sequences)
 *   d_initial_state [N, H, K, V] or NULL (not requested)
 * Token rows outside every sequence (varlen with cu_seqlens[0] > 0 or
 * cu_seqlens[N] < T) are not written.  The gradient of the gate clamp
 * lam = max(lower_bound, z) is taken as zero where z < lower_bound.
 *
 * workspace: device memory of at least kda_bwd_workspace_size(...) bytes, 256-byte
 * aligned, owned by the caller and free for reuse once the call's work on stream
 * is done.  It holds the state before every 64-token chunk (64 KB per chunk and
 * head) and per-CTA scratch.
 * The call is asynchronous on stream.  Returns KDA_OK or the codes of kda_fwd
 * (d_out takes the place of out in the checks), plus KDA_ERR_NULL for a missing
 * gradient output, KDA_ERR_ALIGN (16 bytes for dq, dk, dv, dg; 4 for the other fp32
 * buffers; 256 for the workspace) and KDA_ERR_WORKSPACE.
 */
size_t kda_bwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                              int64_t num_seqs);
int kda_bwd(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
            const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
            float lower_bound, const void *initial_state, int initial_state_dtype,
            const kda_bf16 *d_out, const float *d_final_state, const int64_t *cu_seqlens,
            int64_t num_seqs, float *dq, float *dk, float *dv, float *dg, float *dbeta,
            float *dA_log, float *ddt_bias, float *d_initial_state, void *workspace,
            size_t workspace_bytes, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
            kda_stream_t stream);

/*
 * kda_bwd_noalloc -- kda_bwd for callers that cannot allocate device memory: code
 * running inside a memory pool or allocator that must not be re-entered, a plugin
 * that is handed tensors but no allocator, or a process whose device memory budget
 * is fixed before the first call.  The FlashKDA pages have no counterpart of it; it
 * is a deployment convenience of this library.
 *
 * Arguments, results and return codes are those of kda_bwd without the workspace
 * pair.  The workspace is instead a fixed array in the library's own device memory,
 * KDA_BWD_NOALLOC_MAX_BYTES (64 MiB) long, which every GPU that loads the library
 * holds until the process exits.  The call allocates nothing (no cudaMalloc, no
 * cudaMallocAsync, no library allocator) and frees nothing.
 *   - A call whose workspace need (kda_bwd_workspace_size of the same shape) exceeds
 *     KDA_BWD_NOALLOC_MAX_BYTES returns KDA_ERR_WORKSPACE and launches nothing.
 *   - The first call on a device looks up the array's device address there (once
 *     per device, with that device current); make that first call before any stream
 *     capture.
 *   - All calls share the one array, and its contents persist from call to call
 *     (the kernels write every part they read, so no clearing is needed).  Calls
 *     whose work overlaps on the GPU (other streams, other host threads) race on
 *     it: serialise them.
 *   - The optional device check of cu_seqlens (kda_set_checks) is not run here, as
 *     its result would need device memory; cu_seqlens is trusted as in kda_bwd with
 *     the checks off.
 */
#define KDA_BWD_NOALLOC_MAX_BYTES ((size_t)64 << 20)
int kda_bwd_noalloc(const kda_bf16 *q, const kda_bf16 *k, const kda_bf16 *v, const kda_bf16 *g,
                    const kda_bf16 *beta, float scale, const float *A_log, const float *dt_bias,
                    float lower_bound, const void *initial_state, int initial_state_dtype,
                    const kda_bf16 *d_out, const float *d_final_state, const int64_t *cu_seqlens,
                    int64_t num_seqs, float *dq, float *dk, float *dv, float *dg, float *dbeta,
                    float *dA_log, float *ddt_bias, float *d_initial_state, int64_t B, int64_t T,
                    int64_t H, int64_t K, int64_t V, kda_stream_t stream);

/*
 * kda_set_checks -- debug checks of device-resident arguments, process-wide; returns
 * the previous level.  0 (default): none; the kernels trust cu_seqlens.  1: every call
 * with cu_seqlens (kda_fwd, kda_fwd_ex, kda_bwd) first checks on the device, on its
 * stream, that 0 <= cu_seqlens[0] <= ... <= cu_seqlens[num_seqs] <= B*T, reads the
 * result back (a stream synchronisation) and returns KDA_ERR_SEQLENS without
 * launching anything if it fails.  The [cu_seqlens[0], cu_seqlens[num_seqs]) range
 * may be any part of the rows (the host entry point passes sub-ranges).
 */
int kda_set_checks(int level);

/* Human-readable text of a return code (static storage; never NULL). */
const char *kda_strerror(int code);

/* Number of kernel launches the last successful kda_fwd call on this host
 * thread enqueued (for launch accounting in benchmarks). */
int kda_last_launch_count(void);

/* Diagnostic: the error word the kernels set when one of their bounded waits
 * gave up (0 = none; the kernel then skipped the rest of its work and returned
 * without trapping).  This covers the checkpoint launch of a chunked kda_bwd too, whose
 * gradients are then not valid.  Synchronous (reads device memory); reset != 0
 * clears it. */
int kda_device_status(int reset);

/* Schedule of the forward kernel, process-wide (returns the previous one, or
 * KDA_ERR_ARG):
 *   KDA_SCHEDULE_AUTO  (default) split when every unit fits the device as a cluster
 *                      and units average at least 4 chunks (256 tokens), else fused;
 *   KDA_SCHEDULE_FUSED one CTA per (sequence, head) runs both roles;
 *   KDA_SCHEDULE_SPLIT a cluster of 4 CTAs per (sequence, head) whenever all units
 *                      fit the device at once (else fused): 3 CTAs prepare every
 *                      third chunk each and one runs the state pass.
 * Both schedules run the same arithmetic in the same order: results are identical. */
#define KDA_SCHEDULE_AUTO 0
#define KDA_SCHEDULE_FUSED 1
#define KDA_SCHEDULE_SPLIT 2
int kda_set_schedule(int mode);

/* Schedule of the backward pass (kda_bwd, kda_bwd_noalloc), process-wide; returns the
 * previous one, or KDA_ERR_ARG:
 *   KDA_BWD_CHUNKED (default) the forward kernel stores the fp32 state before every
 *                   64-token chunk in the workspace (one launch), then one CTA per
 *                   (sequence, head) runs the chunks in reverse in the chunked matrix
 *                   form (the adjoint of the WY form of the forward);
 *   KDA_BWD_TOKEN   one CTA per (sequence, head) sweeps the token recurrence forward
 *                   for its own fp32 checkpoints and reverses it token by token.
 * Both take the same workspace and meet the same tolerances; their rounding differs. */
#define KDA_BWD_CHUNKED 0
#define KDA_BWD_TOKEN 1
int kda_set_bwd_schedule(int mode);

/* Schedule (KDA_SCHEDULE_FUSED or KDA_SCHEDULE_SPLIT) of the last forward launch this
 * host thread enqueued (for reports). */
int kda_last_schedule(void);

/* Testing hook for the failure path (no counterpart on the pages): the next forward
 * launch (kda_fwd, kda_fwd_ex, kda_fwd_host, or the checkpoint launch of a chunked
 * kda_bwd) starts as if one of its CTAs had
 * already given up a bounded wait with `code` (1..255).  Every CTA of that launch
 * then returns at its start without writing out or the final state, exactly as
 * the CTAs that start after a real failure do, and kda_device_status reports
 * `code`.  Process-wide, consumed by the next launch; code 0 cancels a pending
 * one.  KDA_OK, or KDA_ERR_ARG for a code outside 0..255. */
int kda_inject_error(int code);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
