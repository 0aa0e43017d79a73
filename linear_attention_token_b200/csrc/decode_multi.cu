// Multi-token decode / draft verification of the gated delta rule.
//
// "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身": Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t
// applied to T consecutive tokens of each (sequence, value head) in one pass over the
// state, as a speculative decoder's verification of T drafted tokens needs: the state
// stays in registers from the first token to the last, and is written back once, after
// the n_commit-th token (the accepted prefix).
#include "common.cuh"
#include "sm100.cuh"
#include "device_once.h"

namespace gdn {

// The single decode step (decode.cu) applied to T <= 8 consecutive tokens of each
// (sequence, value head), the state held in registers between them, so the state is read
// once and written once per call (after the n_commit-th token).  Per token, the
// arithmetic and its order are the single step's, so T tokens in one call reproduce T
// calls of the single step exactly.
//
// Mapping: a persistent grid of two 256-thread CTAs per SM, each taking (sequence, value
// head) pairs round-robin.  While a CTA computes one head from registers, the next head's
// state streams into its shared memory (one bulk copy) and the next head's token rows
// (cp.async), so the HBM latency of one head hides behind the compute of the previous.
constexpr int kMaxDecodeTokens = 8;

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"(sm100::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                 ::"r"(sm100::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <int DK, int DV, typename TIn>
constexpr int decode_multi_smem() {
    return DK * DV * 4 + 2 * kMaxDecodeTokens * (2 * DK + DV) * (int)sizeof(TIn) +
           2 * 2 * kMaxDecodeTokens * 4;
}

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(256, 2)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                    const float *__restrict__ g, const float *__restrict__ beta, float *S,
                    TIn *__restrict__ out, const int32_t *__restrict__ n_commit, int T, int H_qk,
                    int H_v, int num_heads, float scale, int opts)
{
    constexpr int NT = 256;
    constexpr int TPR = DV / 4;
    constexpr int RPP = NT / TPR;
    constexpr int PASSES = DK / RPP;
    constexpr int EQ = 16 / (int)sizeof(TIn);           // elements per 16-byte chunk
    static_assert(DK % RPP == 0 && DK % 32 == 0 && DK % EQ == 0 && DV % EQ == 0, "shape");
    constexpr int MT = kMaxDecodeTokens;

    extern __shared__ __align__(16) unsigned char dsm[];
    float4 *sst = reinterpret_cast<float4 *>(dsm);                       // next state, DK x DV
    TIn *tq = reinterpret_cast<TIn *>(dsm + DK * DV * 4);                // [2][MT][DK]
    TIn *tk = tq + 2 * MT * DK;                                          // [2][MT][DK]
    TIn *tv = tk + 2 * MT * DK;                                          // [2][MT][DV]
    float *tg = reinterpret_cast<float *>(tv + 2 * MT * DV);             // [2][MT]
    float *tb = tg + 2 * MT;                                             // [2][MT]
    __shared__ float u_s[DV];
    __shared__ float red_a[RPP][DV], red_b[RPP][DV];
    __shared__ float tok_s[MT][5];          // rk, rq, k.q (normalised), alpha, beta
    __shared__ uint64_t bar;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int col4 = tid % TPR, row0 = tid / TPR;

    // token rows of head `nh` into buffer `buf` (committed as one cp.async group)
    auto issue_tokens = [&](int buf, int nh) {
        if (nh < num_heads) {
            const int n = nh / H_v, h = nh - n * H_v, hq = h / (H_v / H_qk);
            for (int e = tid; e < T * (DK / EQ); e += NT) {
                const int t = e / (DK / EQ), c = e - t * (DK / EQ);
                const size_t row = (((size_t)n * T + t) * H_qk + hq) * DK + c * EQ;
                cp_async16(tq + (buf * MT + t) * DK + c * EQ, q + row);
                cp_async16(tk + (buf * MT + t) * DK + c * EQ, k + row);
            }
            for (int e = tid; e < T * (DV / EQ); e += NT) {
                const int t = e / (DV / EQ), c = e - t * (DV / EQ);
                cp_async16(tv + (buf * MT + t) * DV + c * EQ, v + (((size_t)n * T + t) * H_v + h) * DV + c * EQ);
            }
            if (tid < T) {
                const size_t gi = ((size_t)n * T + tid) * H_v + h;
                cp_async4(tg + buf * MT + tid, g + gi);
                cp_async4(tb + buf * MT + tid, beta + gi);
            }
        }
        cp_async_commit();
    };

    if (tid == 0) { sm100::mbar_init(&bar, 1); sm100::fence_mbar_init(); }
    __syncthreads();
    if (blockIdx.x < num_heads) {
        if (tid == 0) {
            sm100::mbar_arrive_expect_tx(&bar, DK * DV * 4);
            sm100::bulk_load_global(sst, S + (size_t)blockIdx.x * DK * DV, DK * DV * 4, &bar);
        }
        issue_tokens(0, blockIdx.x);
    }

    int it = 0;
#pragma unroll 1
    for (int nh = blockIdx.x; nh < num_heads; nh += gridDim.x, ++it) {
        const int buf = it & 1, nxt = nh + gridDim.x;
        const int n = nh / H_v;
        const int commit = n_commit ? min(max(n_commit[n], 0), T) : T;
        issue_tokens(buf ^ 1, nxt);              // the other buffer was released last round
        cp_async_wait_prev();                    // this head's tokens have landed
        sm100::mbar_wait(&bar, (uint32_t)(it & 1), 1u << 26);   // and its state
        __syncthreads();
        const TIn *kq_t = tk + buf * MT * DK, *qq_t = tq + buf * MT * DK, *vv_t = tv + buf * MT * DV;

        float4 s[PASSES];
#pragma unroll
        for (int p = 0; p < PASSES; ++p) s[p] = sst[(p * RPP + row0) * TPR + col4];
        // per token: k.k, q.q, k.q summed as the single step sums them (per 32-element warp
        // slice, then the slices in order), normalisation factors, alpha and beta
        if (warp < T) {
            const int t = warp;
            float skk = 0.f, sqq = 0.f, skq = 0.f;
#pragma unroll
            for (int w = 0; w < DK / 32; ++w) {
                const float kv = to_f32(kq_t[t * DK + 32 * w + lane]), qv = to_f32(qq_t[t * DK + 32 * w + lane]);
                skk += warp_sum(kv * kv); sqq += warp_sum(qv * qv); skq += warp_sum(kv * qv);
            }
            if (lane == 0) {
                float rk = 1.f, rq = 1.f;
                if (opts & kOptL2Norm) {
                    rk = rsqrtf(skk + 1e-6f);
                    rq = rsqrtf(sqq + 1e-6f);
                    skq *= rk * rq;
                }
                tok_s[t][0] = rk; tok_s[t][1] = rq; tok_s[t][2] = skq;
                tok_s[t][3] = expf(gate_log_decay(tg[buf * MT + t], opts));
                tok_s[t][4] = gate_strength(tb[buf * MT + t], opts);
            }
        }
        // every thread has its slice of the state: the buffer takes the next head's
        sm100::fence_proxy_async();
        __syncthreads();
        if (tid == 0 && nxt < num_heads) {
            sm100::mbar_arrive_expect_tx(&bar, DK * DV * 4);
            sm100::bulk_load_global(sst, S + (size_t)nxt * DK * DV, DK * DV * 4, &bar);
        }

        float4 *Sh = reinterpret_cast<float4 *>(S + (size_t)nh * DK * DV);
        const int h = nh - n * H_v;
#pragma unroll 1
        for (int t = 0; t < T; ++t) {
            const float rk = tok_s[t][0], rq = tok_s[t][1], skq = tok_s[t][2];
            const float alpha = tok_s[t][3], bt = tok_s[t][4];
            // partial a = S^T k_t and b = S^T q_t over this thread's rows
            float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
            for (int p = 0; p < PASSES; ++p) {
                const int r = p * RPP + row0;
                const float kr = to_f32(kq_t[t * DK + r]) * rk, qr = to_f32(qq_t[t * DK + r]) * rq;
                pa.x += s[p].x * kr; pa.y += s[p].y * kr; pa.z += s[p].z * kr; pa.w += s[p].w * kr;
                pb.x += s[p].x * qr; pb.y += s[p].y * qr; pb.z += s[p].z * qr; pb.w += s[p].w * qr;
            }
            *reinterpret_cast<float4 *>(&red_a[row0][4 * col4]) = pa;
            *reinterpret_cast<float4 *>(&red_b[row0][4 * col4]) = pb;
            __syncthreads();
            // per value column: u, o
            if (tid < DV) {
                float a = 0.f, b = 0.f;
#pragma unroll
                for (int r = 0; r < RPP; ++r) { a += red_a[r][tid]; b += red_b[r][tid]; }
                const float u = bt * (to_f32(vv_t[t * DV + tid]) - alpha * a);
                u_s[tid] = u;
                out[(((size_t)n * T + t) * H_v + h) * DV + tid] = from_f32<TIn>(scale * (alpha * b + skq * u));
            }
            __syncthreads();
            // S <- alpha S + k u^T in registers; written back after the commit-th token
            const float4 u4 = *reinterpret_cast<const float4 *>(&u_s[4 * col4]);
#pragma unroll
            for (int p = 0; p < PASSES; ++p) {
                const int r = p * RPP + row0;
                const float kr = to_f32(kq_t[t * DK + r]) * rk;
                s[p].x = alpha * s[p].x + kr * u4.x;
                s[p].y = alpha * s[p].y + kr * u4.y;
                s[p].z = alpha * s[p].z + kr * u4.z;
                s[p].w = alpha * s[p].w + kr * u4.w;
            }
            if (t + 1 == commit) {
#pragma unroll
                for (int p = 0; p < PASSES; ++p) __stcs(Sh + (size_t)(p * RPP + row0) * TPR + col4, s[p]);
            }
        }
        __syncthreads();                         // token buffer, red_a/b, u_s free for reuse
    }
}

// shared-memory opt-in and SM count, per device, per instantiation
template <int DK, int DV, typename TIn>
PerDevice g_multi_setup;

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_multi_t(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, float *S, void *out,
                                         const int32_t *n_commit, int N, int T, int H_qk,
                                         int H_v, float scale, int opts, cudaStream_t stream)
{
    const long long heads = (long long)N * H_v;
    if (heads == 0) return cudaSuccess;
    constexpr int smem = decode_multi_smem<DK, DV, TIn>();
    int sms = 0;
    cudaError_t e = g_multi_setup<DK, DV, TIn>.ensure(
        [] {
            return cudaFuncSetAttribute(decode_multi_kernel<DK, DV, TIn>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        decode_multi_smem<DK, DV, TIn>());
        },
        &sms);
    if (e != cudaSuccess) return e;
    const long long grid = heads < 2LL * sms ? heads : 2LL * sms;
    decode_multi_kernel<DK, DV, TIn><<<(unsigned)grid, 256, smem, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, S, (TIn *)out, n_commit, T,
        H_qk, H_v, (int)heads, scale, opts);
    return cudaGetLastError();
}

cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *S, void *out, const int32_t *n_commit,
                                int N, int T, int H_qk, int H_v, int dk, int dv, gdn_dtype dtype,
                                float scale, int opts, cudaStream_t stream)
{
    if (T < 1 || T > kMaxDecodeTokens) return cudaErrorInvalidValue;
#define GDN_DECODE_MULTI_CASE(DK, DV)                                                         \
    if (dk == DK && dv == DV) {                                                               \
        return dtype == GDN_BF16                                                              \
                   ? launch_decode_multi_t<DK, DV, __nv_bfloat16>(q, k, v, g, beta, S, out,   \
                                                                  n_commit, N, T, H_qk, H_v,  \
                                                                  scale, opts, stream)      \
                   : launch_decode_multi_t<DK, DV, float>(q, k, v, g, beta, S, out, n_commit, \
                                                          N, T, H_qk, H_v, scale, opts,     \
                                                          stream);                            \
    }
    GDN_DECODE_MULTI_CASE(128, 128)
    GDN_DECODE_MULTI_CASE(64, 64)
    GDN_DECODE_MULTI_CASE(128, 64)
    GDN_DECODE_MULTI_CASE(64, 128)
#undef GDN_DECODE_MULTI_CASE
    return cudaErrorInvalidValue;
}

}  // namespace gdn
