// Chunked prefill of the gated delta rule on CUDA cores (fp32 arithmetic).
//
// Rule: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身", Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
// Chunked re-association (chunk C = 64 tokens, exact up to rounding): with
// G_i = sum_{s<=i} g_s, gamma_i = exp(G_i) inside the chunk and S the state entering it,
//   A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i),  T = (I + A)^-1   (unit lower)
//   R    = diag(beta) V - diag(beta gamma) K S,     U = T R
//   O    = diag(gamma) Q S + P U,  P_ij = exp(G_i - G_j) q_i.k_j (j <= i)
//   S   <- gamma_{C-1} S + sum_j exp(G_{C-1} - G_j) k_j u_j^T
// Only exp of non-positive arguments is ever taken, so strong in-chunk decay
// cannot overflow.
//
// This kernel serves fp32 inputs (where a 1e-4 relative bound rules out
// reduced-precision tensor-core operands), head dims of 64, and any shape the
// tensor-core kernel does not take.  One CTA of 256 threads owns one
// (sequence, value head, 32-wide value tile); value columns of S evolve
// independently, so tiles need no communication.  The state tile lives in
// shared memory for the whole sequence.
#include "common.cuh"
#include "tri_inverse.cuh"

namespace gdn {

namespace {
constexpr int CC_C = 64;        // chunk length
constexpr int CC_BV = 32;       // value columns per CTA
constexpr int CC_NT = 256;      // threads per CTA
constexpr int CC_TP = CC_C + 1; // padded row pitch of the 64x64 matrices

template <int DK> struct CcSmem {
    float K[CC_C][DK + 1];
    float Q[CC_C][DK + 1];
    float V[CC_C][CC_BV];
    float A[CC_C][CC_TP];
    float P[CC_C][CC_TP];
    float T[CC_C][CC_TP];
    float S[DK][CC_BV];
    float R[CC_C][CC_BV];
    float U[CC_C][CC_BV];
    float g[CC_C], b[CC_C], G[CC_C], decay_to_end[CC_C];
};
}  // namespace

template <int DK, typename TIn>
__global__ void __launch_bounds__(CC_NT, 1)
prefill_cc_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta,
                  const float *S0, TIn *__restrict__ out, float *S_final,
                  const int32_t *__restrict__ cu_seqlens, long long T_dense, int H_qk, int H_v,
                  int DV, float scale, int opts)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    CcSmem<DK> &sm = *reinterpret_cast<CcSmem<DK> *>(smem_raw);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = blockIdx.x, h = blockIdx.y, vt = blockIdx.z;
    const int hq = h / (H_v / H_qk);
    const int v0 = vt * CC_BV;
    long long t_begin, t_end;
    if (cu_seqlens) { t_begin = cu_seqlens[n]; t_end = cu_seqlens[n + 1]; }
    else { t_begin = (long long)n * T_dense; t_end = t_begin + T_dense; }

    // state tile S[:, v0:v0+32]
    const size_t s_off = ((size_t)n * H_v + h) * DK * DV;
    for (int e = tid; e < DK * CC_BV; e += CC_NT) {
        const int d = e / CC_BV, c = e % CC_BV;
        sm.S[d][c] = S0 ? S0[s_off + (size_t)d * DV + v0 + c] : 0.f;
    }

    // thread tilings used below
    const int gi0 = (tid / 16) * 4, gj0 = (tid % 16) * 4;       // 4x4 tile of a 64x64 product
    const int ri0 = (tid / 8) * 2, rc0 = (tid % 8) * 4;         // 2x4 tile of a 64x32 product
    constexpr int RD = DK / 32;                                 // state rows per thread
    const int sd0 = (tid / 8) * RD;                             // RDx4 tile of the DKx32 state

    for (long long c0 = t_begin; c0 < t_end; c0 += CC_C) {
        const int L = (int)min((long long)CC_C, t_end - c0);

        // 1. load the chunk (rows past the sequence end are zero; g = beta = 0 there)
        for (int i = warp; i < CC_C; i += CC_NT / 32) {
            const bool valid = i < L;
            const size_t kq_off = ((size_t)(c0 + i) * H_qk + hq) * DK;
            float ss_k = 0.f, ss_q = 0.f;
            for (int d = lane; d < DK; d += 32) {
                const float kv = valid ? to_f32(k[kq_off + d]) : 0.f;
                const float qv = valid ? to_f32(q[kq_off + d]) : 0.f;
                sm.K[i][d] = kv;
                sm.Q[i][d] = qv;
                ss_k += kv * kv;
                ss_q += qv * qv;
            }
            if (opts & kOptL2Norm) {
                const float rk = rsqrtf(warp_sum(ss_k) + 1e-6f), rq = rsqrtf(warp_sum(ss_q) + 1e-6f);
                for (int d = lane; d < DK; d += 32) { sm.K[i][d] *= rk; sm.Q[i][d] *= rq; }
            }
            sm.V[i][lane] = valid ? to_f32(v[((size_t)(c0 + i) * H_v + h) * DV + v0 + lane]) : 0.f;
        }
        if (tid < CC_C) {
            const bool valid = tid < L;
            sm.g[tid] = valid ? gate_log_decay(g[(size_t)(c0 + tid) * H_v + h], opts) : 0.f;
            sm.b[tid] = valid ? gate_strength(beta[(size_t)(c0 + tid) * H_v + h], opts) : 0.f;
        }
        __syncthreads();

        // 2. in-chunk inclusive cumsum of g (one warp, two tokens per lane)
        if (warp == 0) {
            const float a0 = sm.g[2 * lane], a1 = sm.g[2 * lane + 1];
            float s = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            const float excl = s - (a0 + a1);
            sm.G[2 * lane] = excl + a0;
            sm.G[2 * lane + 1] = s;
        }
        __syncthreads();
        const float G_end = sm.G[CC_C - 1];
        if (tid < CC_C) sm.decay_to_end[tid] = expf(G_end - sm.G[tid]);

        // 3. A (strictly lower) and P (lower incl. diagonal); T starts as I
        {
            float kk[4][4] = {}, qk[4][4] = {};
            if (gj0 <= gi0 + 3) {
                for (int d = 0; d < DK; ++d) {
                    float kr[4], qr[4], kc[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) { kr[r] = sm.K[gi0 + r][d]; qr[r] = sm.Q[gi0 + r][d]; kc[r] = sm.K[gj0 + r][d]; }
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int c = 0; c < 4; ++c) { kk[r][c] += kr[r] * kc[c]; qk[r][c] += qr[r] * kc[c]; }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = gi0 + r, j = gj0 + c;
                    const float decay = (j <= i) ? expf(sm.G[i] - sm.G[j]) : 0.f;
                    sm.A[i][j] = (j < i) ? sm.b[i] * decay * kk[r][c] : 0.f;
                    sm.P[i][j] = decay * qk[r][c];
                    sm.T[i][j] = (i == j) ? 1.f : 0.f;
                }
        }
        __syncthreads();

        // 4. T = (I + A)^-1 (blocked, fp32)
        invert_unit_lower_64<CC_TP>(&sm.A[0][0], &sm.T[0][0], tid);
        __syncthreads();

        // 5. K S and Q S (64x32 each); R = diag(beta) V - diag(beta gamma) K S
        float qs[2][4] = {};
        {
            float ks[2][4] = {};
            for (int d = 0; d < DK; ++d) {
                const float4 s4 = *reinterpret_cast<const float4 *>(&sm.S[d][rc0]);
                const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float kd = sm.K[ri0 + r][d], qd = sm.Q[ri0 + r][d];
#pragma unroll
                    for (int c = 0; c < 4; ++c) { ks[r][c] += kd * sv[c]; qs[r][c] += qd * sv[c]; }
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = ri0 + r;
                const float gam = expf(sm.G[i]), bi = sm.b[i];
#pragma unroll
                for (int c = 0; c < 4; ++c) sm.R[i][rc0 + c] = bi * (sm.V[i][rc0 + c] - gam * ks[r][c]);
            }
        }
        __syncthreads();

        // 6. U = T R
        {
            float u[2][4] = {};
            for (int j = 0; j <= ri0 + 1; ++j) {
                const float4 r4 = *reinterpret_cast<const float4 *>(&sm.R[j][rc0]);
                const float rv[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float t = sm.T[ri0 + r][j];
#pragma unroll
                    for (int c = 0; c < 4; ++c) u[r][c] += t * rv[c];
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) sm.U[ri0 + r][rc0 + c] = u[r][c];
        }
        __syncthreads();

        // 7. O = diag(gamma) Q S + P U  -> out
        {
            float pu[2][4] = {};
            for (int j = 0; j <= ri0 + 1; ++j) {
                const float4 u4 = *reinterpret_cast<const float4 *>(&sm.U[j][rc0]);
                const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float p = sm.P[ri0 + r][j];
#pragma unroll
                    for (int c = 0; c < 4; ++c) pu[r][c] += p * uv[c];
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = ri0 + r;
                if (i < L) {
                    const float gam = expf(sm.G[i]);
                    TIn *o = out + ((size_t)(c0 + i) * H_v + h) * DV + v0 + rc0;
#pragma unroll
                    for (int c = 0; c < 4; ++c) o[c] = from_f32<TIn>(scale * (gam * qs[r][c] + pu[r][c]));
                }
            }
        }

        // 8. S <- gamma_end S + sum_j exp(G_end - G_j) k_j u_j^T   (own RDx4 tile)
        {
            float acc[RD][4] = {};
            for (int j = 0; j < CC_C; ++j) {
                const float w = sm.decay_to_end[j];
                const float4 u4 = *reinterpret_cast<const float4 *>(&sm.U[j][rc0]);
                const float uv[4] = {u4.x * w, u4.y * w, u4.z * w, u4.w * w};
#pragma unroll
                for (int r = 0; r < RD; ++r) {
                    const float kd = sm.K[j][sd0 + r];
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[r][c] += kd * uv[c];
                }
            }
            const float gam_end = expf(G_end);
#pragma unroll
            for (int r = 0; r < RD; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) sm.S[sd0 + r][rc0 + c] = gam_end * sm.S[sd0 + r][rc0 + c] + acc[r][c];
        }
        __syncthreads();
    }

    if (S_final) {
        for (int e = tid; e < DK * CC_BV; e += CC_NT) {
            const int d = e / CC_BV, c = e % CC_BV;
            S_final[s_off + (size_t)d * DV + v0 + c] = sm.S[d][c];
        }
    }
}

template <int DK, typename TIn>
static cudaError_t launch_cc_t(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *S0, void *out, float *S_final,
                               const int32_t *cu, int N, long long T, int H_qk, int H_v, int dv,
                               float scale, int opts, cudaStream_t stream)
{
    const size_t smem = sizeof(CcSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(prefill_cc_kernel<DK, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)N, (unsigned)H_v, (unsigned)(dv / CC_BV));
    prefill_cc_kernel<DK, TIn><<<grid, CC_NT, smem, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, S0, (TIn *)out, S_final, cu, T,
        H_qk, H_v, dv, scale, opts);
    return cudaGetLastError();
}

cudaError_t launch_prefill_cc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S0, void *out, float *S_final,
                              const int32_t *cu, int N, long long T, int H_qk, int H_v, int dk,
                              int dv, gdn_dtype dtype, float scale, int opts,
                              cudaStream_t stream)
{
    if (N == 0) return cudaSuccess;
    if (dk == 128)
        return dtype == GDN_BF16
                   ? launch_cc_t<128, __nv_bfloat16>(q, k, v, g, beta, S0, out, S_final, cu, N, T, H_qk, H_v, dv, scale, opts, stream)
                   : launch_cc_t<128, float>(q, k, v, g, beta, S0, out, S_final, cu, N, T, H_qk, H_v, dv, scale, opts, stream);
    if (dk == 64)
        return dtype == GDN_BF16
                   ? launch_cc_t<64, __nv_bfloat16>(q, k, v, g, beta, S0, out, S_final, cu, N, T, H_qk, H_v, dv, scale, opts, stream)
                   : launch_cc_t<64, float>(q, k, v, g, beta, S0, out, S_final, cu, N, T, H_qk, H_v, dv, scale, opts, stream);
    return cudaErrorInvalidValue;
}

}  // namespace gdn
