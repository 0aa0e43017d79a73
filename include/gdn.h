/* libgdn — the gated delta rule (Gated DeltaNet token mixing) on one NVIDIA B200.
 *
 * Operation ("論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身",
 * Eq. (1), the ranges stated under it, and the one-token concept code beside it):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t                       (read after the update)
 *
 * per (sequence, value head), with alpha_t = exp(g_t) (the decay gate, in (0,1)
 * for g_t < 0) and beta_t the write strength.  S is a dk x dv fp32 matrix, row
 * index = key dimension, dv contiguous.
 *
 * Layouts (all row-major and contiguous; B sequences are folded into tokens):
 *   q, k       [T_total, H_qk, dk]     dtype (GDN_F32 or GDN_BF16)
 *   v, out     [T_total, H_v,  dv]     dtype
 *   g, beta    [T_total, H_v]          fp32
 *   S0/S_final [num_seqs, H_v, dk, dv] fp32
 * Value head h reads q/k head h / (H_v / H_qk) (grouped heads; H_v % H_qk == 0).
 *
 * Ownership: the caller owns every buffer (device memory unless stated).  No
 * entry point allocates, frees or synchronises, except gdn_get_device_error,
 * which synchronises the stream it is given.  Work is enqueued on `stream` and
 * completes asynchronously.
 *
 * Errors: argument checks run on the host before anything is enqueued and return
 * GDN_ERR_INVALID_ARG or GDN_ERR_UNSUPPORTED with nothing launched.  A failed
 * launch returns GDN_ERR_CUDA.  A device-side wait that runs out of its bounded
 * iteration budget records GDN_ERR_TIMEOUT in the workspace; read it with
 * gdn_get_device_error.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, bad offsets */
    GDN_ERR_UNSUPPORTED = 2,   /* a valid combination this build has no kernel for       */
    GDN_ERR_CUDA = 3,          /* a CUDA runtime call or a kernel launch failed          */
    GDN_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up (see the workspace)  */
} gdn_status;

typedef enum {
    GDN_F32 = 0,               /* q, k, v, out in fp32 (CUDA-core kernels)             */
    GDN_BF16 = 1               /* q, k, v, out in bf16 (tensor-core prefill for dk=dv=128;
                                  other head dims run on the CUDA-core kernels)         */
} gdn_dtype;

/* L2-normalise q and k per (token, head) inside the kernel: x / sqrt(sum x^2 + 1e-6). */
#define GDN_FLAG_QK_L2NORM 1u
/* Prefill: use the CUDA-core chunked kernel even where the tensor-core one applies. */
#define GDN_FLAG_FORCE_CUDA_CORE 2u
/* g and beta hold unconstrained logits a, b instead of the gates themselves: the
 * kernels form g = -softplus(a) (so alpha = exp(g) lies in (0, 1)) and
 * beta = sigmoid(b) (in (0, 1)) as they load them, in fp32. */
#define GDN_FLAG_GATE_LOGITS 4u

/* Bytes of device workspace that let gdn_prefill use its fastest schedule for these
 * sizes on the current device (at least 256).  The first 16 bytes hold the device
 * error word; they must be zero-filled before first use.  When few (sequence, value
 * head) pairs would leave most SMs idle (long sequences, few heads), the bf16 tensor-core
 * path splits each sequence into segments that run in parallel; the rest of this size
 * then holds each segment's state transfer and start state (three dk x dv fp32 matrices
 * per segment and value head) and the transfer chains' per-token outputs Psi
 * (T_total x H_v x dk bf16: 1.07 GB for 262,144 tokens x 16 heads).  gdn_prefill
 * accepts any workspace of at least 256 bytes: a smaller one
 * than this size makes it run one unit per sequence (same results, less parallelism).
 * The workspace must stay allocated while work that uses it is in flight, and calls
 * that share one must not overlap on the GPU.
 * Besides the workspace, the library's module holds 20 MB of static device memory on
 * every GPU that loads it: the four-CTA cluster kernel's ring of prepared chunks
 * (64 cluster slots of 320 KB).  A cluster claims one slot for its lifetime; 64 is more
 * than the clusters one B200 can hold at once, so concurrent calls never share a slot. */
size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t T_total, int32_t H_v, int32_t dk,
                                  int32_t dv);

/* Chunked prefill over whole sequences: Eq. (1) for every token, all outputs, and
 * the final state.  Chunks of 64 tokens are re-associated exactly (the WY / UT
 * form of the rule); results equal the token-by-token recurrence up to rounding.
 *
 *   q, k, v, g, beta : inputs in the layouts above (T_total tokens).
 *   S0               : initial state per sequence, or NULL for zero.
 *   out              : [T_total, H_v, dv] outputs, written.
 *   S_final          : final state per sequence, or NULL to skip.  May equal S0.
 *   cu_seqlens       : DEVICE int32[num_seqs + 1] token offsets (non-decreasing,
 *                      cu_seqlens[0] = 0, cu_seqlens[num_seqs] = T), or NULL for a
 *                      dense batch of B sequences of T tokens each.
 *   num_seqs         : number of sequences when cu_seqlens != NULL (then B must be 1);
 *                      ignored (taken as B) when cu_seqlens == NULL.
 *   B, T             : dense batch shape; T_total = B * T.
 *   H_qk, H_v, dk, dv: heads and head dims; dk, dv in {64, 128}; H_v % H_qk == 0.
 *   dtype            : element type of q, k, v, out.
 *   scale            : read-out multiplier (1.0 for the plain rule).
 *   flags            : GDN_FLAG_* bits.
 *   workspace        : device scratch of at least gdn_prefill_workspace_size bytes.
 * Pointers to q, k, v, out, S0, S_final must be 16-byte aligned; g, beta, cu_seqlens
 * 4-byte aligned.  When there are no tokens (T_total == 0) q, k, v, g, beta, out may be
 * NULL and only S_final is written (a copy of S0, or zero).  g must be finite (alpha = 0
 * is reached by a large negative g). */
gdn_status gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *S0, void *out, float *S_final,
                       const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int64_t T,
                       int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dtype,
                       float scale, uint32_t flags, void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/* One decode step: Eq. (1) applied once per (sequence, value head), in place.
 * The one-token concept code of the same section is this step; its erase term is
 * taken as in Eq. (1), i.e. u = beta (v - alpha S^T k), S <- alpha S + k u^T,
 * o = scale * S^T q, each state element read once and written once.
 *
 *   q, k    : [N, H_qk, dk] dtype;  v, out : [N, H_v, dv] dtype
 *   g, beta : [N, H_v] fp32
 *   S_inout : [N, H_v, dk, dv] fp32, updated in place
 * dk, dv in {64, 128}; H_v % H_qk == 0; q, k, v, out, S_inout 16-byte aligned.
 * N == 0 is a no-op (the pointers may then be NULL). */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float *S_inout, void *out, int32_t N,
                           int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dtype,
                           float scale, uint32_t flags, cudaStream_t stream);

/* Multi-token decode / draft verification: T consecutive tokens (1 <= T <= 8) of
 * every (sequence, value head) applied in one call, Eq. (1) once per token in order,
 * with the state read once and written at most once.  This is the sequential
 * recurrence over a short segment (the same rule as gdn_decode_step, applied T times);
 * it serves speculative decoding, where several drafted tokens (for instance from a
 * multi-token-prediction head) are checked at once and only an accepted prefix is
 * kept.
 *
 *   q, k     : [N, T, H_qk, dk] dtype;  v, out : [N, T, H_v, dv] dtype
 *   g, beta  : [N, T, H_v] fp32
 *   S_inout  : [N, H_v, dk, dv] fp32
 *   n_commit : device [N] int32 or NULL.  out[n, t] is o_t for every t < T (each token
 *              sees the state after all tokens before it).  S_inout[n] is replaced by
 *              the state after the first c = n_commit[n] tokens (clamped to [0, T];
 *              c = 0 leaves it unchanged); NULL means c = T for every sequence.
 * dk, dv in {64, 128}; H_v % H_qk == 0; q, k, v, out, S_inout 16-byte aligned.
 * GDN_ERR_UNSUPPORTED for T outside [1, 8].  N == 0 is a no-op (pointers may be NULL). */
gdn_status gdn_decode_multi(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *S_inout, void *out,
                            const int32_t *n_commit, int32_t N, int32_t T, int32_t H_qk,
                            int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dtype, float scale,
                            uint32_t flags, cudaStream_t stream);

/* Backward pass: gradients of a loss L with respect to q, k, v, g, beta and S0, given
 * d_out = dL/d out and dS_final = dL/d S_final, for the computation gdn_prefill performs
 * (same inputs, layouts, varlen and GVA rules, scale and flags).
 * Reverse-mode differentiation of Eq. (1) token by token; exact (no chunked
 * re-association), with the state checkpointed every 64 tokens in the workspace and each
 * chunk recomputed from its checkpoint.
 *
 *   d_out            : like out ([.., T, H_v, dv], dtype)
 *   dS_final         : [N, H_v, dk, dv] fp32 or NULL (= 0)
 *   dq, dk           : [.., T, H_qk, dk] fp32 (value heads sharing a q/k head are summed)
 *   dv               : [.., T, H_v, dv] fp32
 *   dg, dbeta        : [.., T, H_v] fp32; with GDN_FLAG_GATE_LOGITS the gradients with
 *                      respect to the logits passed in g and beta
 *   dS0              : [N, H_v, dk, dv] fp32 or NULL (not computed)
 *   workspace        : device scratch of at least gdn_backward_workspace_size bytes,
 *                      16-byte aligned, no initial contents required
 * The library zero-fills dq, dk, dg, dbeta itself (they are accumulated with atomic adds;
 * their summation order, and so their last bits, may vary from run to run).  dv % 32 == 0.
 * GDN_ERR_UNSUPPORTED with GDN_FLAG_QK_L2NORM.  Nothing to do when T_total == 0 except
 * dS0 = dS_final. */
size_t gdn_backward_workspace_size(int32_t num_seqs, int64_t T_total, int32_t H_v, int32_t dk,
                                   int32_t dv);
gdn_status gdn_backward(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *S0, const void *d_out,
                        const float *dS_final, float *dq, float *dk, float *dv, float *dg,
                        float *dbeta, float *dS0, const int32_t *cu_seqlens, int32_t num_seqs,
                        int32_t B, int64_t T, int32_t H_qk, int32_t H_v, int32_t dk_dim,
                        int32_t dv_dim, gdn_dtype dtype, float scale, uint32_t flags,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* gdn_prefill for callers that cannot allocate device memory: the same computation
 * and arguments, minus the workspace.  The paper has no counterpart; this is a
 * deployment convenience.  Some callers cannot call cudaMalloc (for instance code
 * running inside another runtime's memory pool, or in a context where allocation is
 * forbidden), so they cannot provide the few bytes of device scratch gdn_prefill
 * needs.  This entry point instead uses a scratch array of GDN_STATIC_SCRATCH_BYTES
 * that the library keeps in every GPU that loads it, for as long as the library is
 * loaded; it calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call asks the runtime for that array's device address in the current
 *     context (cudaGetSymbolAddress: a table lookup once the library's module is
 *     loaded, and right again after cudaDeviceReset makes a new primary context).
 *     Make the first call on a device before any stream capture, since it may load
 *     the module.
 *   - Every call on a device shares the one array: calls that may overlap on the GPU
 *     (different streams, or different host threads) race on it.
 *   - Each call clears the array's error word before it launches.  A device-side
 *     timeout on this path is recorded there but not reported back (there is no
 *     workspace to hand to gdn_get_device_error).
 *   - It always runs one unit per sequence (the segmented schedule would need a
 *     workspace that grows with the sizes), so it needs only the 256-byte error
 *     area; it returns GDN_ERR_UNSUPPORTED if that ever exceeded
 *     GDN_STATIC_SCRATCH_BYTES. */
#define GDN_STATIC_SCRATCH_BYTES 4096u
gdn_status gdn_prefill_static_scratch(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, const float *S0,
                                      void *out, float *S_final, const int32_t *cu_seqlens,
                                      int32_t num_seqs, int32_t B, int64_t T, int32_t H_qk,
                                      int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dtype,
                                      float scale, uint32_t flags, cudaStream_t stream);

/* Scheduling override for the bf16 tensor-core prefill (process-wide, for later calls).
 * There are two kernels: one CTA per (sequence or segment, value head) carrying all 128
 * value columns, and a cluster of four CTAs per (sequence, value head) that splits the
 * value columns and shares each chunk's preparation.
 *    0  automatic (default): a cost model of the device's SM count picks the kernel and,
 *       for the first, whether to cut long sequences into segments and into how many
 *       (segments of equal length);
 *   -1  the single-CTA kernel, one unit per sequence;
 *   -2  the four-CTA cluster kernel;
 *   >0  the single-CTA kernel with segments of exactly this many tokens (a multiple of
 *       64) whenever the workspace is large enough (gdn_prefill_workspace_size accounts
 *       for the override).
 * Results do not depend on the schedule beyond rounding.  GDN_ERR_INVALID_ARG for other
 * values. */
gdn_status gdn_set_prefill_segment_tokens(int32_t tokens);

/* The schedule gdn_prefill would use for these sizes on the current device (with the
 * override above and a workspace of workspace_bytes): *kernel is one of GDN_PREFILL_*,
 * *segment_tokens the segment length (0: one unit per sequence), *launches the number of
 * kernels one call enqueues.  varlen: nonzero when cu_seqlens is given.  Enqueues nothing. */
#define GDN_PREFILL_NONE 0          /* no tokens: only S_final is written */
#define GDN_PREFILL_CUDA_CORE 1     /* fp32 or head dims of 64 */
#define GDN_PREFILL_CHAIN 2         /* single-CTA tensor-core kernel */
#define GDN_PREFILL_CLUSTER 3       /* four-CTA cluster tensor-core kernel */
gdn_status gdn_prefill_schedule(int32_t num_seqs, int64_t T_total, int32_t H_v, int32_t dk,
                                int32_t dv, gdn_dtype dtype, int32_t varlen,
                                size_t workspace_bytes, uint32_t flags, int32_t *kernel,
                                int32_t *segment_tokens, int32_t *launches);

/* Every device-side wait of the tensor-core prefill polls its barrier at most this many
 * times (each poll suspends the thread for at most 2 microseconds, less when the awaited
 * phase completes) before the kernel gives up and records GDN_ERR_TIMEOUT: with the
 * default, a wait gives up after at most about 2 seconds.  gdn_set_wait_budget sets the process-wide limit for later launches and
 * returns the previous one; 0 makes every wait give up at once, which exercises the
 * recovery path (the kernel drains its own copies and MMAs and exits; the context stays
 * usable).  The drains after a timeout always use the default limit. */
#define GDN_DEFAULT_WAIT_BUDGET (1u << 20)
uint32_t gdn_set_wait_budget(uint32_t polls);

/* Synchronises `stream`, returns the first device-side error recorded in
 * `workspace` (GDN_OK if none) and clears it.  GDN_ERR_CUDA if the stream itself
 * reports an error. */
gdn_status gdn_get_device_error(void *workspace, cudaStream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *gdn_status_string(gdn_status status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
