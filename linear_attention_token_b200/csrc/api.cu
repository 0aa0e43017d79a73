// libgdn C ABI: argument checks, kernel choice, launch on the caller's stream.
// The operation and the contract of every entry point are stated in include/gdn.h.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "../../include/qsa.h"

#define GDN_API extern "C" __attribute__((visibility("default")))

namespace gdn {
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *S, void *out, int N, int H_qk, int H_v,
                          int dk, int dv, gdn_dtype dtype, float scale, int opts,
                          cudaStream_t stream);
cudaError_t launch_prefill_cc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S0, void *out, float *S_final,
                              const int32_t *cu, int N, long long T, int H_qk, int H_v, int dk,
                              int dv, gdn_dtype dtype, float scale, int opts,
                              cudaStream_t stream);
bool prefill_chain_supported(int dk, int dv, gdn_dtype dtype);
size_t chain_workspace_bytes(int N, long long T_total, int H_v, int sms, int override_tokens);
int device_sm_count();
void describe_prefill(int N, long long T_total, int H_v, int sms, int override_tokens,
                      size_t workspace_bytes, bool varlen, int *kind, int *seg_tokens, int *launches);
cudaError_t launch_prefill_chain(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *S0, void *out, float *S_final,
                                 const int32_t *cu, int N, long long T_dense, long long T_total,
                                 int H_qk, int H_v, float scale, int opts, void *workspace,
                                 size_t workspace_bytes, uint32_t budget, int seg_override,
                                 cudaStream_t stream);
cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *S, void *out, const int32_t *n_commit,
                                int N, int T, int H_qk, int H_v, int dk, int dv, gdn_dtype dtype,
                                float scale, int opts, cudaStream_t stream);
size_t backward_workspace_bytes(int N, long long T_total, int H_v, int dk, int dv);
cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, const void *d_out,
                            const float *dS_final, float *dq, float *dk, float *dv, float *dg,
                            float *dbeta, float *dS0, const int32_t *cu, int N, long long T_dense,
                            long long T_total, int H_qk, int H_v, int dkk, int dvv,
                            gdn_dtype dtype, float scale, int opts, void *ws, cudaStream_t stream);
size_t qsa_index_workspace_bytes(int N, long long total_blocks, int T);
cudaError_t launch_qsa_compress(const void *k, const int32_t *cu_seqlens, const int32_t *cu_blocks,
                                const int32_t *pos0, void *k_hat, int N, long long total_blocks,
                                float rope_base, cudaStream_t stream);
cudaError_t launch_qsa_index(const void *q, const int32_t *q_pos, const void *k_hat,
                             const int32_t *cu_blocks, int N, long long total_blocks, int T,
                             int budget, float rope_base, int32_t *block_idx,
                             float *block_score, int32_t *token_idx, void *workspace,
                             cudaStream_t stream);
size_t static_scratch_capacity();
cudaError_t static_scratch_ptr(void **out);
}  // namespace gdn

namespace {

constexpr size_t kWorkspaceBytes = 256;
constexpr int kDefaultSms = 148;          // B200; used to size a workspace with no device current
std::atomic<uint32_t> g_wait_budget{GDN_DEFAULT_WAIT_BUDGET};
std::atomic<int32_t> g_segment_tokens{0};

// per-call options for the kernels (common.cuh)
int options_of(uint32_t flags)
{
    return ((flags & GDN_FLAG_QK_L2NORM) ? gdn::kOptL2Norm : 0) |
           ((flags & GDN_FLAG_GATE_LOGITS) ? gdn::kOptGateLogits : 0);
}
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool head_dim_ok(int32_t d) { return d == 64 || d == 128; }

// `has_tokens` false: there is no token to read or write, so the token buffers may be
// NULL (an empty tensor has no storage).
gdn_status common_checks(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const void *out, int32_t H_qk, int32_t H_v,
                         int32_t dk, int32_t dv, gdn_dtype dtype, uint32_t flags,
                         bool has_tokens)
{
    if (has_tokens && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
    if (H_qk <= 0 || H_v <= 0 || H_v % H_qk != 0) return GDN_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (flags & ~(GDN_FLAG_QK_L2NORM | GDN_FLAG_FORCE_CUDA_CORE | GDN_FLAG_GATE_LOGITS))
        return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return GDN_ERR_INVALID_ARG;
    if (!aligned(g, 4) || !aligned(beta, 4)) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

}  // namespace

GDN_API size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t T_total, int32_t H_v,
                                          int32_t dk, int32_t dv)
{
    if (num_seqs <= 0 || T_total <= 0 || H_v <= 0 || !gdn::prefill_chain_supported(dk, dv, GDN_BF16))
        return kWorkspaceBytes;
    int sms = gdn::device_sm_count();
    if (sms <= 0) sms = kDefaultSms;
    const size_t n = gdn::chain_workspace_bytes(num_seqs, T_total, H_v, sms, g_segment_tokens.load());
    return n > kWorkspaceBytes ? n : kWorkspaceBytes;
}

GDN_API gdn_status gdn_prefill_schedule(int32_t num_seqs, int64_t T_total, int32_t H_v,
                                        int32_t dk, int32_t dv, gdn_dtype dtype, int32_t varlen,
                                        size_t workspace_bytes, uint32_t flags, int32_t *kernel,
                                        int32_t *segment_tokens, int32_t *launches)
{
    if (!kernel || !segment_tokens || !launches || num_seqs < 0 || T_total < 0 || H_v <= 0)
        return GDN_ERR_INVALID_ARG;
    *segment_tokens = 0;
    if (num_seqs == 0 || T_total == 0) { *kernel = GDN_PREFILL_NONE; *launches = 0; return GDN_OK; }
    if ((flags & GDN_FLAG_FORCE_CUDA_CORE) || !gdn::prefill_chain_supported(dk, dv, dtype)) {
        *kernel = GDN_PREFILL_CUDA_CORE;
        *launches = 1;
        return GDN_OK;
    }
    int sms = gdn::device_sm_count();
    if (sms <= 0) sms = kDefaultSms;
    int kind = 0, seg = 0, n = 0;
    gdn::describe_prefill(num_seqs, T_total, H_v, sms, g_segment_tokens.load(), workspace_bytes,
                          varlen != 0, &kind, &seg, &n);
    *kernel = kind == 1 ? GDN_PREFILL_CLUSTER : GDN_PREFILL_CHAIN;
    *segment_tokens = seg;
    *launches = n;
    return GDN_OK;
}

GDN_API gdn_status gdn_set_prefill_segment_tokens(int32_t tokens)
{
    if (tokens < -2 || (tokens > 0 && tokens % 64 != 0)) return GDN_ERR_INVALID_ARG;
    g_segment_tokens.store(tokens);
    return GDN_OK;
}

GDN_API uint32_t gdn_set_wait_budget(uint32_t polls)
{
    return g_wait_budget.exchange(polls);
}

GDN_API gdn_status gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *S0, void *out, float *S_final,
                               const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int64_t T,
                               int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                               gdn_dtype dtype, float scale, uint32_t flags, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    const bool has_tokens = (cu_seqlens ? (long long)T : (long long)B * T) > 0;
    gdn_status st = common_checks(q, k, v, g, beta, out, H_qk, H_v, dk, dv, dtype, flags,
                                  has_tokens);
    if (st != GDN_OK) return st;
    int N;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0 || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
        N = num_seqs;
    } else {
        N = B;
    }
    if (N > 0 && H_v > 65535) return GDN_ERR_UNSUPPORTED;
    if ((S0 && !aligned(S0, 16)) || (S_final && !aligned(S_final, 16))) return GDN_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kWorkspaceBytes || !aligned(workspace, 16))
        return GDN_ERR_INVALID_ARG;
    const long long T_total = cu_seqlens ? (long long)T : (long long)B * T;
    if (N == 0 || T_total == 0) {
        // nothing to compute; S_final = S0 (or zero) per sequence still has to be written
        if (S_final && N > 0) {
            const size_t bytes = (size_t)N * H_v * dk * dv * sizeof(float);
            cudaError_t e = S0 ? (S0 == S_final ? cudaSuccess
                                                : cudaMemcpyAsync(S_final, S0, bytes,
                                                                  cudaMemcpyDeviceToDevice, stream))
                               : cudaMemsetAsync(S_final, 0, bytes, stream);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }
    const int l2 = options_of(flags);
    cudaError_t e;
    if (!(flags & GDN_FLAG_FORCE_CUDA_CORE) && gdn::prefill_chain_supported(dk, dv, dtype)) {
        e = gdn::launch_prefill_chain(q, k, v, g, beta, S0, out, S_final, cu_seqlens, N,
                                      cu_seqlens ? 0 : (long long)T, T_total, H_qk, H_v, scale, l2,
                                      workspace, workspace_bytes, g_wait_budget.load(),
                                      g_segment_tokens.load(), stream);
    } else {
        e = gdn::launch_prefill_cc(q, k, v, g, beta, S0, out, S_final, cu_seqlens, N,
                                   cu_seqlens ? 0 : (long long)T, H_qk, H_v, dk, dv, dtype, scale,
                                   l2, stream);
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API gdn_status gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *S_inout, void *out, int32_t N,
                                   int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                                   gdn_dtype dtype, float scale, uint32_t flags,
                                   cudaStream_t stream)
{
    if (N < 0) return GDN_ERR_INVALID_ARG;
    gdn_status st = common_checks(q, k, v, g, beta, out, H_qk, H_v, dk, dv, dtype, flags, N > 0);
    if (st != GDN_OK) return st;
    if ((N > 0 && !S_inout) || !aligned(S_inout, 16)) return GDN_ERR_INVALID_ARG;
    if ((long long)N * H_v > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    const int l2 = options_of(flags);
    cudaError_t e = gdn::launch_decode(q, k, v, g, beta, S_inout, out, N, H_qk, H_v, dk, dv,
                                       dtype, scale, l2, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API gdn_status gdn_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, float *S_inout, void *out,
                                    const int32_t *n_commit, int32_t N, int32_t T, int32_t H_qk,
                                    int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dtype,
                                    float scale, uint32_t flags, cudaStream_t stream)
{
    if (N < 0) return GDN_ERR_INVALID_ARG;
    if (T < 1 || T > 8) return GDN_ERR_UNSUPPORTED;
    gdn_status st = common_checks(q, k, v, g, beta, out, H_qk, H_v, dk, dv, dtype, flags, N > 0);
    if (st != GDN_OK) return st;
    if ((N > 0 && !S_inout) || !aligned(S_inout, 16) || !aligned(n_commit, 4))
        return GDN_ERR_INVALID_ARG;
    if ((long long)N * H_v > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    const int l2 = options_of(flags);
    cudaError_t e = gdn::launch_decode_multi(q, k, v, g, beta, S_inout, out, n_commit, N, T,
                                             H_qk, H_v, dk, dv, dtype, scale, l2, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API size_t gdn_backward_workspace_size(int32_t num_seqs, int64_t T_total, int32_t H_v,
                                           int32_t dk, int32_t dv)
{
    if (num_seqs < 0 || T_total < 0 || H_v < 0 || !head_dim_ok(dk) || !head_dim_ok(dv)) return 0;
    return gdn::backward_workspace_bytes(num_seqs, T_total, H_v, dk, dv);
}

GDN_API gdn_status gdn_backward(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *S0, const void *d_out,
                                const float *dS_final, float *dq, float *dk, float *dv,
                                float *dg, float *dbeta, float *dS0,
                                const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                                int64_t T, int32_t H_qk, int32_t H_v, int32_t dk_dim,
                                int32_t dv_dim, gdn_dtype dtype, float scale, uint32_t flags,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    const bool has_tokens = (cu_seqlens ? (long long)T : (long long)B * T) > 0;
    gdn_status st = common_checks(q, k, v, g, beta, d_out, H_qk, H_v, dk_dim, dv_dim, dtype,
                                  flags, has_tokens);
    if (st != GDN_OK) return st;
    if (flags & GDN_FLAG_QK_L2NORM) return GDN_ERR_UNSUPPORTED;
    if (has_tokens && (!dq || !dk || !dv || !dg || !dbeta)) return GDN_ERR_INVALID_ARG;
    if (!aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(dg, 4) ||
        !aligned(dbeta, 4))
        return GDN_ERR_INVALID_ARG;
    int N;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0 || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
        N = num_seqs;
    } else {
        N = B;
    }
    if ((S0 && !aligned(S0, 16)) || (dS_final && !aligned(dS_final, 16)) || (dS0 && !aligned(dS0, 16)))
        return GDN_ERR_INVALID_ARG;
    const long long T_total = cu_seqlens ? (long long)T : (long long)B * T;
    if ((long long)N * H_v * (dv_dim / 32) > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    const size_t need = gdn_backward_workspace_size(N, T_total, H_v, dk_dim, dv_dim);
    if (N > 0 && T_total > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16)))
        return GDN_ERR_INVALID_ARG;
    if (N == 0) return GDN_OK;
    if (T_total == 0) {
        if (dS0) {
            const size_t bytes = (size_t)N * H_v * dk_dim * dv_dim * sizeof(float);
            cudaError_t e = dS_final ? cudaMemcpyAsync(dS0, dS_final, bytes,
                                                       cudaMemcpyDeviceToDevice, stream)
                                     : cudaMemsetAsync(dS0, 0, bytes, stream);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }
    // accumulated with atomic adds
    cudaError_t e = cudaMemsetAsync(dq, 0, (size_t)T_total * H_qk * dk_dim * sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, (size_t)T_total * H_qk * dk_dim * sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dg, 0, (size_t)T_total * H_v * sizeof(float), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, (size_t)T_total * H_v * sizeof(float), stream);
    if (e != cudaSuccess) return GDN_ERR_CUDA;
    e = gdn::launch_backward(q, k, v, g, beta, S0, d_out, dS_final, dq, dk, dv, dg, dbeta, dS0,
                             cu_seqlens, N, cu_seqlens ? 0 : (long long)T, T_total, H_qk, H_v,
                             dk_dim, dv_dim, dtype, scale, options_of(flags), workspace, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// gdn_prefill without a caller-provided workspace (see include/gdn.h): the kernels
// receive the library's static scratch instead.
GDN_API gdn_status gdn_prefill_static_scratch(const void *q, const void *k, const void *v,
                                              const float *g, const float *beta,
                                              const float *S0, void *out, float *S_final,
                                              const int32_t *cu_seqlens, int32_t num_seqs,
                                              int32_t B, int64_t T, int32_t H_qk, int32_t H_v,
                                              int32_t dk, int32_t dv, gdn_dtype dtype,
                                              float scale, uint32_t flags, cudaStream_t stream)
{
    if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
    const bool has_tokens = (cu_seqlens ? (long long)T : (long long)B * T) > 0;
    gdn_status st = common_checks(q, k, v, g, beta, out, H_qk, H_v, dk, dv, dtype, flags,
                                  has_tokens);
    if (st != GDN_OK) return st;
    int N;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0 || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
        N = num_seqs;
    } else {
        N = B;
    }
    if (N > 0 && H_v > 65535) return GDN_ERR_UNSUPPORTED;
    if ((S0 && !aligned(S0, 16)) || (S_final && !aligned(S_final, 16))) return GDN_ERR_INVALID_ARG;
    const long long T_total = cu_seqlens ? (long long)T : (long long)B * T;
    // this path needs only the workspace's error word, which must fit the library-held scratch
    if (kWorkspaceBytes > gdn::static_scratch_capacity()) return GDN_ERR_UNSUPPORTED;
    if (N == 0 || T_total == 0) {
        if (S_final && N > 0) {
            const size_t bytes = (size_t)N * H_v * dk * dv * sizeof(float);
            cudaError_t e = S0 ? (S0 == S_final ? cudaSuccess
                                                : cudaMemcpyAsync(S_final, S0, bytes,
                                                                  cudaMemcpyDeviceToDevice, stream))
                               : cudaMemsetAsync(S_final, 0, bytes, stream);
            if (e != cudaSuccess) return GDN_ERR_CUDA;
        }
        return GDN_OK;
    }
    void *scratch = nullptr;
    if (gdn::static_scratch_ptr(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
    // the error word must start at zero; earlier calls may have left one behind
    if (cudaMemsetAsync(scratch, 0, sizeof(gdn::DeviceError), stream) != cudaSuccess)
        return GDN_ERR_CUDA;
    const int l2 = options_of(flags);
    cudaError_t e;
    if (!(flags & GDN_FLAG_FORCE_CUDA_CORE) && gdn::prefill_chain_supported(dk, dv, dtype)) {
        // the static scratch holds the error word only: the one-pass schedule
        e = gdn::launch_prefill_chain(q, k, v, g, beta, S0, out, S_final, cu_seqlens, N,
                                      cu_seqlens ? 0 : (long long)T, T_total, H_qk, H_v, scale, l2,
                                      scratch, kWorkspaceBytes, g_wait_budget.load(), -1, stream);
    } else {
        e = gdn::launch_prefill_cc(q, k, v, g, beta, S0, out, S_final, cu_seqlens, N,
                                   cu_seqlens ? 0 : (long long)T, H_qk, H_v, dk, dv, dtype, scale,
                                   l2, stream);
    }
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API gdn_status gdn_get_device_error(void *workspace, cudaStream_t stream)
{
    if (!workspace || !aligned(workspace, 16)) return GDN_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
    gdn::DeviceError h{};
    if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (h.status != 0) {
        const gdn::DeviceError zero{};
        if (cudaMemcpy(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return GDN_ERR_CUDA;
    }
    return static_cast<gdn_status>(h.status);
}

// ------------------------------------------------------------ QSA indexer (qsa.h)
namespace {
bool rope_base_ok(float base) { return base > 0.f && base < INFINITY; }
}  // namespace

GDN_API gdn_status gdn_qsa_compress(const void *k, const int32_t *cu_seqlens,
                                    const int32_t *cu_blocks, const int32_t *pos0, void *k_hat,
                                    int32_t num_seqs, int64_t total_blocks, float rope_base,
                                    cudaStream_t stream)
{
    if (num_seqs < 0 || total_blocks < 0 || total_blocks > INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (!rope_base_ok(rope_base)) return GDN_ERR_INVALID_ARG;
    if (total_blocks == 0) return GDN_OK;
    if (num_seqs == 0) return GDN_ERR_INVALID_ARG;
    if (!k || !cu_seqlens || !cu_blocks || !k_hat) return GDN_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(k_hat, 16) || !aligned(cu_seqlens, 4) ||
        !aligned(cu_blocks, 4) || !aligned(pos0, 4))
        return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_qsa_compress(k, cu_seqlens, cu_blocks, pos0, k_hat, num_seqs,
                                                   total_blocks, rope_base, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API size_t gdn_qsa_index_workspace_size(int32_t num_seqs, int64_t total_blocks)
{
    if (num_seqs < 0 || total_blocks < 0) return 0;
    return gdn::qsa_index_workspace_bytes(num_seqs, total_blocks, 1);
}

GDN_API size_t gdn_qsa_index_multi_workspace_size(int32_t num_seqs, int64_t total_blocks,
                                                  int32_t n_queries)
{
    if (num_seqs < 0 || total_blocks < 0 || n_queries < 1 || n_queries > GDN_QSA_MAX_QUERIES)
        return 0;
    return gdn::qsa_index_workspace_bytes(num_seqs, total_blocks, n_queries);
}

namespace {
gdn_status qsa_index(const void *q, const int32_t *q_pos, const void *k_hat,
                     const int32_t *cu_blocks, int32_t num_seqs, int64_t total_blocks,
                     int32_t n_queries, int32_t budget_blocks, float rope_base,
                     int32_t *block_idx, float *block_score, int32_t *token_idx,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (n_queries < 1 || n_queries > GDN_QSA_MAX_QUERIES) return GDN_ERR_UNSUPPORTED;
    if (num_seqs < 0) return GDN_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * n_queries > GDN_QSA_MAX_SEQS) return GDN_ERR_UNSUPPORTED;
    if (total_blocks < 0 || total_blocks > INT32_MAX / GDN_QSA_MAX_QUERIES)
        return GDN_ERR_INVALID_ARG;
    if (budget_blocks < 1 || budget_blocks > GDN_QSA_MAX_BUDGET) return GDN_ERR_INVALID_ARG;
    if (!rope_base_ok(rope_base)) return GDN_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDN_OK;
    if (!q || !q_pos || !cu_blocks || !block_idx || !workspace) return GDN_ERR_INVALID_ARG;
    if (total_blocks > 0 && !k_hat) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_hat, 16) || !aligned(workspace, 16) || !aligned(q_pos, 4) ||
        !aligned(cu_blocks, 4) || !aligned(block_idx, 4) || !aligned(block_score, 4) ||
        !aligned(token_idx, 4))
        return GDN_ERR_INVALID_ARG;
    if (workspace_bytes < gdn::qsa_index_workspace_bytes(num_seqs, total_blocks, n_queries))
        return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_qsa_index(q, q_pos, k_hat, cu_blocks, num_seqs,
                                                total_blocks, n_queries, budget_blocks,
                                                rope_base, block_idx, block_score, token_idx,
                                                workspace, stream);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
}  // namespace

GDN_API gdn_status gdn_qsa_index_decode(const void *q, const int32_t *q_pos, const void *k_hat,
                                        const int32_t *cu_blocks, int32_t num_seqs,
                                        int64_t total_blocks, int32_t budget_blocks,
                                        float rope_base, int32_t *block_idx, float *block_score,
                                        int32_t *token_idx, void *workspace,
                                        size_t workspace_bytes, cudaStream_t stream)
{
    return qsa_index(q, q_pos, k_hat, cu_blocks, num_seqs, total_blocks, 1, budget_blocks,
                     rope_base, block_idx, block_score, token_idx, workspace, workspace_bytes,
                     stream);
}

GDN_API gdn_status gdn_qsa_index_multi(const void *q, const int32_t *q_pos, const void *k_hat,
                                       const int32_t *cu_blocks, int32_t num_seqs,
                                       int64_t total_blocks, int32_t n_queries,
                                       int32_t budget_blocks, float rope_base,
                                       int32_t *block_idx, float *block_score,
                                       int32_t *token_idx, void *workspace,
                                       size_t workspace_bytes, cudaStream_t stream)
{
    return qsa_index(q, q_pos, k_hat, cu_blocks, num_seqs, total_blocks, n_queries,
                     budget_blocks, rope_base, block_idx, block_score, token_idx, workspace,
                     workspace_bytes, stream);
}

GDN_API const char *gdn_status_string(gdn_status status)
{
    switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: no kernel for this combination";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA call or launch failed";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown gdn_status";
}
