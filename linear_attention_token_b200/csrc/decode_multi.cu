// Multi-token decode / draft verification of the gated delta rule.
//
// "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身": Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t
// applied to T consecutive tokens of each (sequence, value head) in one pass over the
// state, as a speculative decoder's verification of T drafted tokens needs: the state
// stays in registers from the first token to the last, and is written back once, after
// the n_commit-th token (the accepted prefix).
#include "common.cuh"

namespace gdn {

// The single decode step (decode.cu) applied to T <= 8 consecutive tokens of each
// (sequence, value head), the state held in registers between them, so the state is read
// once and written once per call (after the n_commit-th token).  Mapping: one CTA of 256
// threads per (sequence, value head), as in the single step.  Per token, the arithmetic
// and its order are the single step's, so T tokens in one call reproduce T calls of the
// single step exactly.
constexpr int kMaxDecodeTokens = 8;

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(256, 2)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                    const float *__restrict__ g, const float *__restrict__ beta, float *S,
                    TIn *__restrict__ out, const int32_t *__restrict__ n_commit, int T, int H_qk,
                    int H_v, float scale, int l2norm)
{
    constexpr int NT = 256;
    constexpr int TPR = DV / 4;
    constexpr int RPP = NT / TPR;
    constexpr int PASSES = DK / RPP;
    static_assert(DK % RPP == 0 && DK % 32 == 0, "shape");

    __shared__ float k_s[kMaxDecodeTokens][DK], q_s[kMaxDecodeTokens][DK];
    __shared__ float v_s[kMaxDecodeTokens][DV], u_s[DV];
    __shared__ float red_a[RPP][DV], red_b[RPP][DV];
    __shared__ float tok_s[kMaxDecodeTokens][5];        // rk, rq, k.q (normalised), alpha, beta

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nh = blockIdx.x;                 // n * H_v + h
    const int n = nh / H_v, h = nh - n * H_v;
    const int hq = h / (H_v / H_qk);
    const int col4 = tid % TPR, row0 = tid / TPR;
    const int commit = n_commit ? min(max(n_commit[n], 0), T) : T;

    // 1. the whole state slice in flight, then every token's inputs into shared memory
    float4 *Sh = reinterpret_cast<float4 *>(S + (size_t)nh * DK * DV);
    float4 s[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) s[p] = __ldcs(Sh + (size_t)(p * RPP + row0) * TPR + col4);
    for (int e = tid; e < T * DK; e += NT) {
        const int t = e / DK, d = e - t * DK;
        const size_t tok = (size_t)n * T + t;
        k_s[t][d] = to_f32(k[(tok * H_qk + hq) * DK + d]);
        q_s[t][d] = to_f32(q[(tok * H_qk + hq) * DK + d]);
    }
    for (int e = tid; e < T * DV; e += NT) {
        const int t = e / DV, j = e - t * DV;
        v_s[t][j] = to_f32(v[(((size_t)n * T + t) * H_v + h) * DV + j]);
    }
    __syncthreads();
    // per token: k.k, q.q, k.q summed as the single step sums them (per 32-element warp
    // slice, then the slices in order), normalisation factors, alpha and beta
    if (warp < T) {
        const int t = warp;
        float skk = 0.f, sqq = 0.f, skq = 0.f;
#pragma unroll
        for (int w = 0; w < DK / 32; ++w) {
            const float kv = k_s[t][32 * w + lane], qv = q_s[t][32 * w + lane];
            skk += warp_sum(kv * kv); sqq += warp_sum(qv * qv); skq += warp_sum(kv * qv);
        }
        if (lane == 0) {
            float rk = 1.f, rq = 1.f;
            if (l2norm) {
                rk = rsqrtf(skk + 1e-6f);
                rq = rsqrtf(sqq + 1e-6f);
                skq *= rk * rq;
            }
            const size_t gi = ((size_t)n * T + t) * H_v + h;
            tok_s[t][0] = rk; tok_s[t][1] = rq; tok_s[t][2] = skq;
            tok_s[t][3] = expf(g[gi]); tok_s[t][4] = beta[gi];
        }
    }
    __syncthreads();

#pragma unroll 1
    for (int t = 0; t < T; ++t) {
        const float rk = tok_s[t][0], rq = tok_s[t][1], skq = tok_s[t][2];
        const float alpha = tok_s[t][3], bt = tok_s[t][4];
        // 2. partial a = S^T k_t and b = S^T q_t over this thread's rows
        float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const int r = p * RPP + row0;
            const float kr = k_s[t][r] * rk, qr = q_s[t][r] * rq;
            pa.x += s[p].x * kr; pa.y += s[p].y * kr; pa.z += s[p].z * kr; pa.w += s[p].w * kr;
            pb.x += s[p].x * qr; pb.y += s[p].y * qr; pb.z += s[p].z * qr; pb.w += s[p].w * qr;
        }
        *reinterpret_cast<float4 *>(&red_a[row0][4 * col4]) = pa;
        *reinterpret_cast<float4 *>(&red_b[row0][4 * col4]) = pb;
        __syncthreads();
        // 3. per value column: u, o
        if (tid < DV) {
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int r = 0; r < RPP; ++r) { a += red_a[r][tid]; b += red_b[r][tid]; }
            const float u = bt * (v_s[t][tid] - alpha * a);
            u_s[tid] = u;
            out[(((size_t)n * T + t) * H_v + h) * DV + tid] = from_f32<TIn>(scale * (alpha * b + skq * u));
        }
        __syncthreads();
        // 4. S <- alpha S + k u^T in registers; written back after the commit-th token
        const float4 u4 = *reinterpret_cast<const float4 *>(&u_s[4 * col4]);
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
            const int r = p * RPP + row0;
            const float kr = k_s[t][r] * rk;
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
}

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_multi_t(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta, float *S, void *out,
                                         const int32_t *n_commit, int N, int T, int H_qk,
                                         int H_v, float scale, int l2norm, cudaStream_t stream)
{
    const long long blocks = (long long)N * H_v;
    if (blocks == 0) return cudaSuccess;
    decode_multi_kernel<DK, DV, TIn><<<(unsigned)blocks, 256, 0, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, S, (TIn *)out, n_commit, T,
        H_qk, H_v, scale, l2norm);
    return cudaGetLastError();
}

cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *S, void *out, const int32_t *n_commit,
                                int N, int T, int H_qk, int H_v, int dk, int dv, gdn_dtype dtype,
                                float scale, int l2norm, cudaStream_t stream)
{
    if (T < 1 || T > kMaxDecodeTokens) return cudaErrorInvalidValue;
#define GDN_DECODE_MULTI_CASE(DK, DV)                                                         \
    if (dk == DK && dv == DV) {                                                               \
        return dtype == GDN_BF16                                                              \
                   ? launch_decode_multi_t<DK, DV, __nv_bfloat16>(q, k, v, g, beta, S, out,   \
                                                                  n_commit, N, T, H_qk, H_v,  \
                                                                  scale, l2norm, stream)      \
                   : launch_decode_multi_t<DK, DV, float>(q, k, v, g, beta, S, out, n_commit, \
                                                          N, T, H_qk, H_v, scale, l2norm,     \
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
