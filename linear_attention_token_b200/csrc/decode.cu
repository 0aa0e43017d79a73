// Fused single-token decode step of the gated delta rule.
//
// "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身": Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
// and the one-token concept code (difference against what the key currently
// reads, write it, read out with q).  Written as one pass over the state:
//   a = S^T k,  b = S^T q            (reductions over the key dimension)
//   u = beta (v - alpha a)           (Eq. (1): alpha also scales the erase term)
//   S <- alpha S + k u^T,  o = scale (alpha b + (k.q) u)  ( = scale * S_new^T q )
// Each fp32 state element is loaded once (streaming, evict-first) and stored
// once, in place.
//
// Mapping: one CTA of 256 threads per (sequence, value head).  A thread owns
// four consecutive value columns (one 16-byte vector) of DK*DV/1024 rows, so a
// warp's load instruction covers 512 contiguous bytes of a row (DV=128) and all
// of a head's state sits in registers between the load and the store.
#include "common.cuh"

namespace gdn {

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                   const float *__restrict__ g, const float *__restrict__ beta, float *S,
                   TIn *__restrict__ out, int H_qk, int H_v, float scale, int opts)
{
    constexpr int NT = 256;
    constexpr int TPR = DV / 4;        // threads per state row
    constexpr int RPP = NT / TPR;      // rows covered by one pass of the block
    constexpr int PASSES = DK / RPP;   // 16-byte vectors held per thread
    static_assert(DK % RPP == 0, "shape");

    __shared__ float k_s[DK], q_s[DK], u_s[DV];
    __shared__ float red_a[RPP][DV], red_b[RPP][DV];
    __shared__ float dots[3][NT / 32];

    const int tid = threadIdx.x;
    const int nh = blockIdx.x;                 // n * H_v + h
    const int n = nh / H_v, h = nh - n * H_v;
    const int hq = h / (H_v / H_qk);
    const int col4 = tid % TPR, row0 = tid / TPR;

    // 1. issue every state load first so the whole slice is in flight
    float4 *Sh = reinterpret_cast<float4 *>(S + (size_t)nh * DK * DV);
    float4 s[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) s[p] = __ldcs(Sh + (size_t)(p * RPP + row0) * TPR + col4);

    // 2. k, q to shared memory (fp32); k.k, q.q, k.q for normalisation and read-out
    float kk = 0.f, qq = 0.f, kq = 0.f;
    if (tid < DK) {
        const float kv = to_f32(k[((size_t)n * H_qk + hq) * DK + tid]);
        const float qv = to_f32(q[((size_t)n * H_qk + hq) * DK + tid]);
        k_s[tid] = kv;
        q_s[tid] = qv;
        kk = kv * kv; qq = qv * qv; kq = kv * qv;
    }
    kk = warp_sum(kk); qq = warp_sum(qq); kq = warp_sum(kq);
    if ((tid & 31) == 0) { dots[0][tid >> 5] = kk; dots[1][tid >> 5] = qq; dots[2][tid >> 5] = kq; }
    __syncthreads();
    float skk = 0.f, sqq = 0.f, skq = 0.f;
#pragma unroll
    for (int w = 0; w < DK / 32; ++w) { skk += dots[0][w]; sqq += dots[1][w]; skq += dots[2][w]; }
    float rk = 1.f, rq = 1.f;
    if (opts & kOptL2Norm) {
        rk = rsqrtf(skk + 1e-6f);
        rq = rsqrtf(sqq + 1e-6f);
        skq *= rk * rq;
    }

    // 3. partial a = S^T k and b = S^T q over this thread's rows, four columns each
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = p * RPP + row0;
        const float kr = k_s[r] * rk, qr = q_s[r] * rq;
        pa.x += s[p].x * kr; pa.y += s[p].y * kr; pa.z += s[p].z * kr; pa.w += s[p].w * kr;
        pb.x += s[p].x * qr; pb.y += s[p].y * qr; pb.z += s[p].z * qr; pb.w += s[p].w * qr;
    }
    *reinterpret_cast<float4 *>(&red_a[row0][4 * col4]) = pa;
    *reinterpret_cast<float4 *>(&red_b[row0][4 * col4]) = pb;
    __syncthreads();

    // 4. per value column: u, o
    const float alpha = expf(gate_log_decay(g[nh], opts));
    const float bt = gate_strength(beta[nh], opts);
    if (tid < DV) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int r = 0; r < RPP; ++r) { a += red_a[r][tid]; b += red_b[r][tid]; }
        const float vj = to_f32(v[(size_t)nh * DV + tid]);
        const float u = bt * (vj - alpha * a);
        u_s[tid] = u;
        out[(size_t)nh * DV + tid] = from_f32<TIn>(scale * (alpha * b + skq * u));
    }
    __syncthreads();

    // 5. S <- alpha S + k u^T, streamed back in place
    const float4 u4 = *reinterpret_cast<const float4 *>(&u_s[4 * col4]);
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = p * RPP + row0;
        const float kr = k_s[r] * rk;
        float4 x = s[p];
        x.x = alpha * x.x + kr * u4.x;
        x.y = alpha * x.y + kr * u4.y;
        x.z = alpha * x.z + kr * u4.z;
        x.w = alpha * x.w + kr * u4.w;
        __stcs(Sh + (size_t)r * TPR + col4, x);
    }
}

template <int DK, int DV, typename TIn>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *S, void *out, int N, int H_qk,
                                   int H_v, float scale, int opts, cudaStream_t stream)
{
    const long long blocks = (long long)N * H_v;
    if (blocks == 0) return cudaSuccess;
    decode_step_kernel<DK, DV, TIn><<<(unsigned)blocks, 256, 0, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, S, (TIn *)out, H_qk, H_v,
        scale, opts);
    return cudaGetLastError();
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *S, void *out, int N, int H_qk, int H_v,
                          int dk, int dv, gdn_dtype dtype, float scale, int opts,
                          cudaStream_t stream)
{
#define GDN_DECODE_CASE(DK, DV)                                                                \
    if (dk == DK && dv == DV) {                                                                \
        return dtype == GDN_BF16                                                               \
                   ? launch_decode_t<DK, DV, __nv_bfloat16>(q, k, v, g, beta, S, out, N, H_qk, \
                                                            H_v, scale, opts, stream)        \
                   : launch_decode_t<DK, DV, float>(q, k, v, g, beta, S, out, N, H_qk, H_v,    \
                                                    scale, opts, stream);                    \
    }
    GDN_DECODE_CASE(128, 128)
    GDN_DECODE_CASE(64, 64)
    GDN_DECODE_CASE(128, 64)
    GDN_DECODE_CASE(64, 128)
#undef GDN_DECODE_CASE
    return cudaErrorInvalidValue;
}

}  // namespace gdn
