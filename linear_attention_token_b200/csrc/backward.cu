// Backward pass of the gated delta rule: the gradients with respect to q, k, v, g, beta and
// S0, given dL/do_t and dL/dS_final.
//
// "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身", Eq. (1), per token:
//   alpha = exp(g), a = S_{t-1}^T k, u = beta (v - alpha a), S_t = alpha S_{t-1} + k u^T,
//   o_t = scale S_t^T q.
// Reverse-mode differentiation of those lines, from the last token to the first, with dS
// the gradient of the state after token t:
//   dS += scale q do^T;  dq = scale S_t do;  du = dS^T k;  dk = dS u + S_{t-1} da;
//   da = -alpha beta du;  dalpha = <dS, S_{t-1}> - beta <du, a>;  dbeta = <du, v - alpha a>;
//   dv = beta du;  dg = alpha dalpha;  dS <- alpha dS + k da^T;  dS0 = dS at the end.
//
// Exact and sequential (no chunked re-association): one CTA per (sequence, value head,
// 16-column slice of the value dimension), one thread per state row, so a thread holds
// its row of S (and of dS) in registers; two CTAs share an SM.  The value columns of S evolve independently, so
// the slices need no exchange; the gradients that sum over value columns (dq, dk, dalpha,
// dbeta) are accumulated across slices and grouped value heads with atomic adds.
//   Phase 1: the state is run forward over the sequence and stored at every chunk start
//            (checkpoints, workspace).
//   Phase 2: chunks in reverse; each is recomputed forward from its checkpoint with its
//            states kept in a per-CTA workspace area, then walked backward token by token.
#include "common.cuh"

namespace gdn {

namespace {

constexpr int BW_C = 64;     // chunk (checkpoint interval)
constexpr int BW_BV = 16;    // value columns per CTA

// BW_BV values per lane -> lane l holds the sum over the warp's 32 lanes of value
// (l mod BW_BV): halving exchanges (BW_BV - 1 shuffles), then the remaining lane halves
__device__ __forceinline__ float warp_transpose_sum(float (&x)[BW_BV], int lane)
{
#pragma unroll
    for (int m = BW_BV / 2; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = upper ? x[i] : x[i + m];
            const float keep = upper ? x[i + m] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
#pragma unroll
    for (int m = BW_BV; m < 32; m <<= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], m);
    return x[0];
}

template <int DK>
struct BwShared {
    float k[BW_C][DK], q[BW_C][DK];
    float v[BW_C][BW_BV], dout[BW_C][BW_BV];
    float a[BW_C][BW_BV], u[BW_C][BW_BV];
    float g[BW_C], beta[BW_C], dgate_g[BW_C], dgate_b[BW_C];   // gates and d(gate)/d(input)
    float red[DK / 32][BW_BV];
    float col[BW_BV];
    float scal[DK / 32][2];
    // the backward walk's per-token reductions, by token parity (a buffer is written again
    // two tokens later, after both barriers of the token in between)
    float bred[2][DK / 32][BW_BV];
    float bcol[2][BW_BV];
    float bscal[2][DK / 32];
};

}  // namespace

template <int DK, typename TIn>
__global__ void __launch_bounds__(DK, 2)
backward_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k, const TIn *__restrict__ v,
                const float *__restrict__ g, const float *__restrict__ beta, const float *S0,
                const TIn *__restrict__ d_out, const float *dS_final, float *dq, float *dk,
                float *dv, float *dg, float *dbeta, float *dS0, const int32_t *__restrict__ cu,
                long long T_dense, int H_qk, int H_v, int DV, float scale, int opts,
                float *ckpt, float *scratch, long long ckpt_stride)
{
    constexpr int NW = DK / 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwShared<DK> &sm = *reinterpret_cast<BwShared<DK> *>(smem_raw);
    const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
    const int NV = DV / BW_BV;
    const int slice = blockIdx.x % NV, nh = blockIdx.x / NV;
    const int n = nh / H_v, h = nh - n * H_v, hq = h / (H_v / H_qk);
    const int c0 = slice * BW_BV;
    long long t_begin, t_end;
    if (cu) { t_begin = cu[n]; t_end = cu[n + 1]; }
    else { t_begin = (long long)n * T_dense; t_end = t_begin + T_dense; }
    const int nch = (int)((t_end - t_begin + BW_C - 1) / BW_C);
    float *my_ckpt = ckpt + (size_t)blockIdx.x * ckpt_stride;           // [nch][DK][BV]
    float *my_scr = scratch + (size_t)blockIdx.x * (BW_C + 1) * DK * BW_BV;  // [C+1][DK][BV]
    const size_t s_off = ((size_t)n * H_v + h) * DK * DV;

    // the chunk's inputs into shared memory (fp32), gates formed, d(gate)/d(input) kept
    auto load_chunk = [&](long long t0, int L, bool with_grad_inputs) {
        for (int e = r; e < BW_C * DK; e += DK) {
            const int i = e / DK, d = e - i * DK;
            const bool ok = i < L;
            const size_t row = ((size_t)(t0 + i) * H_qk + hq) * DK + d;
            sm.k[i][d] = ok ? to_f32(k[row]) : 0.f;
            if (with_grad_inputs) sm.q[i][d] = ok ? to_f32(q[row]) : 0.f;
        }
        for (int e = r; e < BW_C * BW_BV; e += DK) {
            const int i = e / BW_BV, j = e - i * BW_BV;
            const bool ok = i < L;
            const size_t row = ((size_t)(t0 + i) * H_v + h) * DV + c0 + j;
            sm.v[i][j] = ok ? to_f32(v[row]) : 0.f;
            if (with_grad_inputs) sm.dout[i][j] = ok ? to_f32(d_out[row]) : 0.f;
        }
        for (int i = r; i < BW_C; i += DK) {
            const bool ok = i < L;
            const size_t gi = (size_t)(t0 + i) * H_v + h;
            const float x = ok ? g[gi] : 0.f, y = ok ? beta[gi] : 0.f;
            sm.g[i] = gate_log_decay(x, opts);
            sm.beta[i] = gate_strength(y, opts);
            // g = -softplus(x): dg/dx = -sigmoid(x);  beta = sigmoid(y): dbeta/dy = beta (1 - beta)
            sm.dgate_g[i] = (opts & kOptGateLogits) ? -1.f / (1.f + expf(-x)) : 1.f;
            sm.dgate_b[i] = (opts & kOptGateLogits) ? sm.beta[i] * (1.f - sm.beta[i]) : 1.f;
        }
        __syncthreads();
    };
    // one token forward on the row in registers: returns nothing, leaves a, u in sm
    auto step_forward = [&](float (&s)[BW_BV], int i) {
        const float kr = sm.k[i][r];
        float x[BW_BV];
#pragma unroll
        for (int j = 0; j < BW_BV; ++j) x[j] = s[j] * kr;
        const float part = warp_transpose_sum(x, lane);
        if (lane < BW_BV) sm.red[warp][lane] = part;
        __syncthreads();
        if (r < BW_BV) {
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) a += sm.red[w][r];
            const float al = expf(sm.g[i]);
            sm.a[i][r] = a;
            sm.u[i][r] = sm.beta[i] * (sm.v[i][r] - al * a);
        }
        __syncthreads();
        const float al = expf(sm.g[i]);
#pragma unroll
        for (int j = 0; j < BW_BV; ++j) s[j] = al * s[j] + kr * sm.u[i][j];
    };
    auto store_row = [&](float *dst, const float (&s)[BW_BV]) {
        float4 *p = reinterpret_cast<float4 *>(dst + (size_t)r * BW_BV);
#pragma unroll
        for (int j = 0; j < BW_BV; j += 4) p[j / 4] = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
    };
    auto load_row = [&](const float *src, float (&s)[BW_BV]) {
        const float4 *p = reinterpret_cast<const float4 *>(src + (size_t)r * BW_BV);
#pragma unroll
        for (int j = 0; j < BW_BV; j += 4) {
            const float4 f = p[j / 4];
            s[j] = f.x; s[j + 1] = f.y; s[j + 2] = f.z; s[j + 3] = f.w;
        }
    };

    // ---- phase 1: forward over the sequence, checkpoint at every chunk start
    float s[BW_BV];
    {
        const float *src = S0 ? S0 + s_off + (size_t)r * DV + c0 : nullptr;
#pragma unroll
        for (int j = 0; j < BW_BV; ++j) s[j] = src ? src[j] : 0.f;
    }
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
        const long long t0 = t_begin + (long long)c * BW_C;
        const int L = (int)min((long long)BW_C, t_end - t0);
        store_row(my_ckpt + (size_t)c * DK * BW_BV, s);
        if (c + 1 == nch) break;                 // the last chunk is recomputed in phase 2
        load_chunk(t0, L, false);
#pragma unroll 1
        for (int i = 0; i < L; ++i) step_forward(s, i);
        __syncthreads();                         // before the next chunk overwrites sm
    }

    // ---- phase 2: chunks in reverse
    float dS[BW_BV];
    {
        const float *src = dS_final ? dS_final + s_off + (size_t)r * DV + c0 : nullptr;
#pragma unroll
        for (int j = 0; j < BW_BV; ++j) dS[j] = src ? src[j] : 0.f;
    }
#pragma unroll 1
    for (int c = nch - 1; c >= 0; --c) {
        const long long t0 = t_begin + (long long)c * BW_C;
        const int L = (int)min((long long)BW_C, t_end - t0);
        __syncthreads();
        load_chunk(t0, L, true);
        // recompute: my_scr[i] = state before token i, my_scr[L] = state after the chunk
        load_row(my_ckpt + (size_t)c * DK * BW_BV, s);
        store_row(my_scr, s);
#pragma unroll 1
        for (int i = 0; i < L; ++i) {
            step_forward(s, i);
            store_row(my_scr + (size_t)(i + 1) * DK * BW_BV, s);
        }
        // backward over the chunk's tokens; s holds S_t (after token i).  S_{t-1} of the
        // next (earlier) token is loaded one step ahead, so its latency hides behind a step.
        float sp_next[BW_BV];
        if (L > 0) load_row(my_scr + (size_t)(L - 1) * DK * BW_BV, sp_next);
#pragma unroll 1
        for (int i = L - 1; i >= 0; --i) {
            const long long t = t0 + i;
            float sp[BW_BV];                                   // S_{t-1}
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) sp[j] = sp_next[j];
            if (i > 0) load_row(my_scr + (size_t)(i - 1) * DK * BW_BV, sp_next);
            const float al = expf(sm.g[i]), bt = sm.beta[i];
            const float qr = sm.q[i][r], kr = sm.k[i][r];
            // dS += scale q do^T ; dq_t (this slice's columns) = scale S_t do
            float dq_part = 0.f;
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) {
                const float dj = scale * sm.dout[i][j];
                dS[j] += qr * dj;
                dq_part += s[j] * dj;
            }
            atomicAdd(dq + ((size_t)t * H_qk + hq) * DK + r, dq_part);
            // du = dS^T k (over rows)
            const int pb = i & 1;
            float x[BW_BV];
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) x[j] = dS[j] * kr;
            {
                const float part = warp_transpose_sum(x, lane);
                if (lane < BW_BV) sm.bred[pb][warp][lane] = part;
            }
            // this row's share of <dS, S_{t-1}>
            float dal_part = 0.f;
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) dal_part += dS[j] * sp[j];
            dal_part = warp_sum(dal_part);
            if (lane == 0) sm.bscal[pb][warp] = dal_part;
            __syncthreads();
            if (r < BW_BV) {
                float du = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) du += sm.bred[pb][w][r];
                sm.bcol[pb][r] = du;
                dv[((size_t)t * H_v + h) * DV + c0 + r] = bt * du;
            }
            __syncthreads();
            // dk_t (slice share) = dS u + S_{t-1} da, da = -alpha beta du
            float dk_part = 0.f;
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) {
                const float du = sm.bcol[pb][j];
                dk_part += dS[j] * sm.u[i][j] - al * bt * du * sp[j];
            }
            atomicAdd(dk + ((size_t)t * H_qk + hq) * DK + r, dk_part);
            if (warp == 0) {
                // dbeta (slice share) = <du, v - alpha a>;  -beta <du, a> joins dalpha
                const bool on = lane < BW_BV;
                const float du = on ? sm.bcol[pb][lane] : 0.f, a = on ? sm.a[i][lane] : 0.f;
                const float db = warp_sum(on ? du * (sm.v[i][lane] - al * a) : 0.f);
                const float da_dot = warp_sum(du * a);
                if (lane == 0) {
                    float dal = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) dal += sm.bscal[pb][w];
                    dal -= bt * da_dot;
                    const size_t gi = (size_t)t * H_v + h;
                    atomicAdd(dg + gi, al * dal * sm.dgate_g[i]);
                    atomicAdd(dbeta + gi, db * sm.dgate_b[i]);
                }
            }
            // dS <- alpha dS + k da^T
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) dS[j] = al * dS[j] - kr * al * bt * sm.bcol[pb][j];
#pragma unroll
            for (int j = 0; j < BW_BV; ++j) s[j] = sp[j];
        }
    }
    if (dS0) {
        float *dst = dS0 + s_off + (size_t)r * DV + c0;
#pragma unroll
        for (int j = 0; j < BW_BV; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(dS[j], dS[j + 1], dS[j + 2], dS[j + 3]);
    }
}

size_t backward_workspace_bytes(int N, long long T_total, int H_v, int dk, int dv)
{
    // checkpoints: every CTA gets room for the longest possible sequence's chunk starts
    // (bounded by the total length), plus its chunk of recomputed states
    const long long nv = dv / BW_BV;
    const long long ctas = (long long)N * H_v * nv;
    const long long max_chunks = (T_total + BW_C - 1) / BW_C + 1;
    return (size_t)(ctas * (max_chunks + BW_C + 1) * dk * BW_BV * sizeof(float));
}

template <int DK, typename TIn>
static cudaError_t launch_bw_t(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *S0, const void *d_out,
                               const float *dS_final, float *dq, float *dk, float *dv, float *dg,
                               float *dbeta, float *dS0, const int32_t *cu, int N,
                               long long T_dense, long long T_total, int H_qk, int H_v, int DV,
                               float scale, int opts, void *ws, cudaStream_t stream)
{
    const long long ctas = (long long)N * H_v * (DV / BW_BV);
    if (ctas == 0) return cudaSuccess;
    const long long max_chunks = (T_total + BW_C - 1) / BW_C + 1;
    const long long ckpt_stride = max_chunks * DK * BW_BV;
    float *ckpt = reinterpret_cast<float *>(ws);
    float *scratch = ckpt + (size_t)ctas * ckpt_stride;
    const int smem = (int)sizeof(BwShared<DK>);
    cudaError_t e = cudaFuncSetAttribute(backward_kernel<DK, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    backward_kernel<DK, TIn><<<(unsigned)ctas, DK, smem, stream>>>(
        (const TIn *)q, (const TIn *)k, (const TIn *)v, g, beta, S0, (const TIn *)d_out,
        dS_final, dq, dk, dv, dg, dbeta, dS0, cu, T_dense, H_qk, H_v, DV, scale, opts, ckpt,
        scratch, ckpt_stride);
    return cudaGetLastError();
}

cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, const void *d_out,
                            const float *dS_final, float *dq, float *dk, float *dv, float *dg,
                            float *dbeta, float *dS0, const int32_t *cu, int N, long long T_dense,
                            long long T_total, int H_qk, int H_v, int dkk, int dvv,
                            gdn_dtype dtype, float scale, int opts, void *ws, cudaStream_t stream)
{
    if (dvv % BW_BV != 0) return cudaErrorInvalidValue;
#define GDN_BW_CASE(DK)                                                                        \
    if (dkk == DK) {                                                                           \
        return dtype == GDN_BF16                                                               \
                   ? launch_bw_t<DK, __nv_bfloat16>(q, k, v, g, beta, S0, d_out, dS_final, dq, \
                                                    dk, dv, dg, dbeta, dS0, cu, N, T_dense,    \
                                                    T_total, H_qk, H_v, dvv, scale, opts, ws,  \
                                                    stream)                                    \
                   : launch_bw_t<DK, float>(q, k, v, g, beta, S0, d_out, dS_final, dq, dk, dv, \
                                            dg, dbeta, dS0, cu, N, T_dense, T_total, H_qk,     \
                                            H_v, dvv, scale, opts, ws, stream);                \
    }
    GDN_BW_CASE(128)
    GDN_BW_CASE(64)
#undef GDN_BW_CASE
    return cudaErrorInvalidValue;
}

}  // namespace gdn
