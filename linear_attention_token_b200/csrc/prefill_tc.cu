// Chunked prefill of the gated delta rule on the sm_100a tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged by TMA), dk = dv = 128, bf16 I/O.
//
// Rule: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身", Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
// Chunk algebra (C = 64 tokens; G_i = in-chunk cumsum of g, gamma_i = exp G_i, S the
// state entering the chunk; exact re-association of the rule):
//   A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i);  T = (I + A)^-1
//   W    = T diag(beta gamma) K,  U~ = T diag(beta) V,  U = U~ - W S
//   O    = diag(gamma) Q S + P U,  P_ij = exp(G_i - G_j) q_i.k_j (j <= i)
//   S   <- gamma_end S + K~^T U,   K~_j = exp(G_end - G_j) k_j
//
// Everything is computed transposed so that every product has M = 128 on the
// tensor core and the 128 TMEM lanes map to the value (or key) index, which is
// also the row a thread owns in every epilogue:
//   P1  [K;Q] K^T        -> TMEM KQ  (lanes 0-63: K K^T, lanes 64-127: Q K^T)
//   P2  K^T T'^T  = W^T   -> TMEM W   (lane = key dim d)
//   P3  V^T T''^T = U~^T  -> TMEM U   (lane = value dim v)
//   S1  U~^T - S^T W^T    -> TMEM U   (negated B operand)       = U^T
//   S1' S^T Q^T           -> TMEM O   = (Q S)^T
//   S2  S^T += U^T K~     -> TMEM S   (the fp32 state, lane v, column d)
//   S2' U^T P^T           -> TMEM PU  = (P U)^T
// The fp32 state stays in TMEM for the whole sequence; a bf16 copy of S^T in
// shared memory is the A operand of S1/S1'.  T = (I + A)^-1 is solved on the CUDA
// cores in fp32 (four threads per column, no per-row barriers).
//
// One CTA (256 threads, 1 per SM) owns one (sequence, value head).  Rows past the
// end of a sequence are zeroed in shared memory with g = beta = 0, which makes
// them inert in every product.  Every mbarrier wait is bounded; a CTA whose wait
// runs out records GDN_ERR_TIMEOUT in the workspace, waits for its own copies and
// MMAs in flight, frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn {
using namespace sm100;

// Profiling aid, compiled in only with -DGDN_PHASE_TIMERS: CTA (0, 0) records
// clock64() at each phase boundary of its first 64 chunks.
#ifdef GDN_PHASE_TIMERS
__device__ unsigned long long g_phase_clock[64][32];
#define PHASE_MARK(k) gdn_phase_mark(tid, c, k)
__device__ __forceinline__ void gdn_phase_mark(int tid, int c, int k) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && c < 64) g_phase_clock[c][k] = clock64();
}
#define GDN_TRI_MARK(k) gdn_phase_mark(tid, dbg_chunk, k)
#else
#define PHASE_MARK(k) do { } while (0)
#define GDN_TRI_MARK(k) do { } while (0)
#endif

}  // namespace gdn
#include "tri_inverse.cuh"
namespace gdn {

namespace {

constexpr int TC_C = 64;
constexpr int TC_D = 128;
constexpr int TC_THREADS = 256;
constexpr uint32_t kDefaultBudget = 1u << 22;    // mbarrier polls before giving up

// TMEM columns (512 allocated; fp32 accumulators, lane = row of D)
constexpr uint32_t TM_S = 0, TM_KQ = 128, TM_W = 192, TM_U = 256, TM_O = 320, TM_PU = 384;

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t SM_KQ = 0;          // 32 KB [K cg0 | Q cg0 | K cg1 | Q cg1], rows = tokens
constexpr uint32_t SM_V = 32768;       // 2 x 16 KB, V [cg0 | cg1] per buffer
constexpr uint32_t SM_KT = 65536;      // 16 KB K~ [cg0 | cg1]
constexpr uint32_t SM_TP = 81920;      // 8 KB T' = T diag(beta gamma), K-major rows i
constexpr uint32_t SM_TPP = 90112;     // 8 KB T'' = T diag(beta)
constexpr uint32_t SM_P = 98304;       // 8 KB P, K-major rows i
constexpr uint32_t SM_WT = 106496;     // 16 KB W^T, rows d (MN-major B operand)
constexpr uint32_t SM_UT = 122880;     // 16 KB U^T, rows v (K-major A operand)
constexpr uint32_t SM_ST = 139264;     // 32 KB S^T bf16, rows v [cg0 | cg1]
constexpr uint32_t SM_AF = 172032;     // fp32 A, 64 x 65
constexpr uint32_t SM_TF = 188672;     // fp32 T, 64 x 65
constexpr uint32_t SM_VEC = 205312;    // g, beta, G, gamma, decay-to-end: 5 x 64 fp32
constexpr uint32_t SM_BAR = 206592;    // 4 mbarriers + TMEM base address
constexpr uint32_t SM_OST = 206848;    // 16 KB output staging, rows i x 128 bf16 (v contiguous)
constexpr uint32_t SM_END = SM_OST + 16384;
constexpr uint32_t SMEM_BYTES = SM_END + 1024;
constexpr int TP = 65;                 // fp32 matrix pitch

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t x) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x));
}

// Write 64 fp32 values (one TMEM row) as a 128-byte swizzled bf16 row.
__device__ __forceinline__ void store_row_bf16(unsigned char *tile, int r, const float *x) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = pack_bf16(x[8 * c + 0], x[8 * c + 1]);
        w.y = pack_bf16(x[8 * c + 2], x[8 * c + 3]);
        w.z = pack_bf16(x[8 * c + 4], x[8 * c + 5]);
        w.w = pack_bf16(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128(r, c)) = w;
    }
}

__device__ __forceinline__ void ld64(uint32_t taddr, float *x) {
    uint32_t a[32], b[32];
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) { x[j] = __uint_as_float(a[j]); x[32 + j] = __uint_as_float(b[j]); }
}

struct Pending {       // copies / MMAs in flight, tracked uniformly by every thread
    int kq_issued = 0, kq_done = 0;
    int v_issued[2] = {0, 0}, v_done[2] = {0, 0};
    int mma_issued = 0, mma_done = 0;
};

}  // namespace

__global__ void __launch_bounds__(TC_THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
                  const float *__restrict__ beta, const float *S0,
                  __nv_bfloat16 *__restrict__ out, float *S_final,
                  const int32_t *__restrict__ cu_seqlens, long long T_dense, int H_qk, int H_v,
                  float scale, int l2norm, DeviceError *err, uint32_t budget)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;                     // TMEM lane owned in epilogues
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int n = blockIdx.x, h = blockIdx.y;
    const int hq = h / (H_v / H_qk);
    long long t_begin, t_end;
    if (cu_seqlens) { t_begin = cu_seqlens[n]; t_end = cu_seqlens[n + 1]; }
    else { t_begin = (long long)n * T_dense; t_end = t_begin + T_dense; }
    const int nchunks = (int)((t_end - t_begin + TC_C - 1) / TC_C);
    const size_t s_off = ((size_t)n * H_v + h) * TC_D * TC_D;

    uint64_t *bar_kq = reinterpret_cast<uint64_t *>(sm + SM_BAR);
    uint64_t *bar_v = bar_kq + 1;                        // two buffers
    uint64_t *bar_mma = bar_kq + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SM_BAR + 32);
    float *gs = reinterpret_cast<float *>(sm + SM_VEC);
    float *bs = gs + 64, *Gs = gs + 128, *gam = gs + 192, *dte = gs + 256;
    float *Af = reinterpret_cast<float *>(sm + SM_AF);
    float *Tf = reinterpret_cast<float *>(sm + SM_TF);

    if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
    if (tid == 0) {
        mbar_init(bar_kq, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_v + 1, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    Pending pend;
    int fail_where = 0;

    auto issue_kq = [&](int c) {
        const int t0 = (int)(t_begin + (long long)c * TC_C);
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_kq, 32768);
            tma_load_3d(sm + SM_KQ, &tm_k, bar_kq, 0, hq, t0);
            tma_load_3d(sm + SM_KQ + 16384, &tm_k, bar_kq, 64, hq, t0);
            tma_load_3d(sm + SM_KQ + 8192, &tm_q, bar_kq, 0, hq, t0);
            tma_load_3d(sm + SM_KQ + 24576, &tm_q, bar_kq, 64, hq, t0);
        }
        ++pend.kq_issued;
    };
    auto issue_v = [&](int c) {
        const int b = c & 1;
        const int t0 = (int)(t_begin + (long long)c * TC_C);
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_v + b, 16384);
            tma_load_3d(sm + SM_V + b * 16384, &tm_v, bar_v + b, 0, h, t0);
            tma_load_3d(sm + SM_V + b * 16384 + 8192, &tm_v, bar_v + b, 64, h, t0);
        }
        ++pend.v_issued[b];
    };
    // CTA-uniform bounded wait
    auto cta_wait = [&](uint64_t *bar, int done_count) -> bool {
        const bool ok = mbar_wait(bar, (uint32_t)(done_count & 1), budget);
        return !__syncthreads_or(!ok);
    };
    auto mma_sync_wait = [&]() -> bool {
        const bool ok = cta_wait(bar_mma, pend.mma_done);
        if (ok) ++pend.mma_done;
        tc_fence_after();
        return ok;
    };
    auto commit_mma = [&]() {
        if (tid == 0) umma_commit(bar_mma);
        ++pend.mma_issued;
    };
    // make generic smem writes and TMEM accesses visible to the MMA issuer
    auto handoff = [&]() {
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    if (nchunks > 0) { issue_kq(0); issue_v(0); }

    // initial state: S0 (or 0) into TMEM (lane v, column d) and its bf16 copy S^T
    if (wg == 0) {
#pragma unroll 1
        for (int d0 = 0; d0 < TC_D; d0 += 32) {
            uint32_t r[32];
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x[j] = S0 ? S0[s_off + (size_t)(d0 + j) * TC_D + row] : 0.f;
                r[j] = __float_as_uint(x[j]);
            }
            tmem_st32(tmem + lane_off + TM_S + d0, r);
            unsigned char *st = sm + SM_ST + (d0 / 64) * 16384;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint4 w;
                w.x = pack_bf16(x[8 * cc + 0], x[8 * cc + 1]);
                w.y = pack_bf16(x[8 * cc + 2], x[8 * cc + 3]);
                w.z = pack_bf16(x[8 * cc + 4], x[8 * cc + 5]);
                w.w = pack_bf16(x[8 * cc + 6], x[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(st + sw128(row, (d0 % 64) / 8 + cc)) = w;
            }
        }
        tmem_wait_st();
    }
    handoff();

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const long long t0 = t_begin + (long long)c * TC_C;
        const int L = (int)min((long long)TC_C, t_end - t0);
        const int vb = c & 1;
        unsigned char *Vt = sm + SM_V + vb * 16384;
        PHASE_MARK(0);
        if (c + 1 < nchunks) issue_v(c + 1);          // its buffer was released by chunk c-1
        PHASE_MARK(16);

        // ---- A: inputs of the chunk
        {
            const bool ok = mbar_wait(bar_kq, (uint32_t)(pend.kq_done & 1), budget) &&
                            mbar_wait(bar_v + vb, (uint32_t)(pend.v_done[vb] & 1), budget);
            if (__syncthreads_or(!ok)) { fail_where = 1; break; }
        }
        ++pend.kq_done;
        PHASE_MARK(17);
        ++pend.v_done[vb];
        PHASE_MARK(1);
        if (L < TC_C) {            // zero rows L..63 of K, Q (both halves) and V
            const int zr = TC_C - L;
            for (int e = tid; e < 6 * zr * 8; e += TC_THREADS) {
                const int region = e / (zr * 8), rr = L + (e % (zr * 8)) / 8, cc = e % 8;
                unsigned char *base = region < 4 ? sm + SM_KQ + region * 8192 : Vt + (region - 4) * 8192;
                *reinterpret_cast<uint4 *>(base + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        if (l2norm) {              // rows of K (0..63) and Q (64..127), two threads per row
            const int rr = tid >> 1, half = tid & 1;
            unsigned char *rowp = sm + SM_KQ + half * 16384 + (rr >= 64 ? 8192 : 0) + (rr & 63) * 128;
            float ss = 0.f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint4 w = *reinterpret_cast<const uint4 *>(rowp + cc * 16);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) { const float2 f = unpack_bf16(ws[q2]); ss += f.x * f.x + f.y * f.y; }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float rn = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 w = *reinterpret_cast<const uint4 *>(rowp + cc * 16);
                uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) { const float2 f = unpack_bf16(ws[q2]); ws[q2] = pack_bf16(f.x * rn, f.y * rn); }
                *reinterpret_cast<uint4 *>(rowp + cc * 16) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
            }
        }
        if (tid < TC_C) {
            const bool valid = tid < L;
            gs[tid] = valid ? g[(size_t)(t0 + tid) * H_v + h] : 0.f;
            bs[tid] = valid ? beta[(size_t)(t0 + tid) * H_v + h] : 0.f;
        }
        __syncthreads();
        if (warp == 0) {
            const float a0 = gs[2 * lane], a1 = gs[2 * lane + 1];
            float s = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            const float G0 = s - a1, G1 = s;
            const float Gend = __shfl_sync(0xffffffffu, s, 31);
            Gs[2 * lane] = G0; Gs[2 * lane + 1] = G1;
            gam[2 * lane] = expf(G0); gam[2 * lane + 1] = expf(G1);
            dte[2 * lane] = expf(Gend - G0); dte[2 * lane + 1] = expf(Gend - G1);
        }
        handoff();
        PHASE_MARK(2);

        // ---- B: P1 = [K;Q] K^T and S1' (Q S)^T = S^T Q^T on the tensor core;
        //         meanwhile K~ = diag(decay-to-end) K on the CUDA cores
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, 64, false, false);
            const uint32_t kq = smem_u32(sm + SM_KQ), st = smem_u32(sm + SM_ST);
            const uint32_t qb = kq + 8192;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t a = kq + (s / 4) * 16384 + (s % 4) * 32;
                umma_bf16(tmem + TM_KQ, sdesc_kmajor(a), sdesc_kmajor(a), id, s > 0);
            }
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t o = (s / 4) * 16384 + (s % 4) * 32;
                umma_bf16(tmem + TM_O, sdesc_kmajor(st + o), sdesc_kmajor(qb + o), id, s > 0);
            }
        }
        commit_mma();
        for (int e = tid; e < 1024; e += TC_THREADS) {
            const int cg = e >> 9, r = (e >> 3) & 63, cc = e & 7;
            const uint4 w = *reinterpret_cast<const uint4 *>(sm + SM_KQ + cg * 16384 + r * 128 + cc * 16);
            const float s = dte[r];
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) { const float2 f = unpack_bf16(ws[q2]); o[q2] = pack_bf16(f.x * s, f.y * s); }
            *reinterpret_cast<uint4 *>(sm + SM_KT + cg * 8192 + r * 128 + cc * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async();
        if (!mma_sync_wait()) { fail_where = 3; break; }
        PHASE_MARK(3);

        // ---- C: A (fp32) from K K^T, P (bf16) from Q K^T; T := I
        if (wg == 0) {
            float x[64];
            ld64(tmem + lane_off + TM_KQ, x);
            PHASE_MARK(18);
            // loads of G are issued ahead of the stores (they may not be reordered
            // across stores to shared memory by the compiler)
            const bool is_a = quad < 2;
            const int i = is_a ? row : row - 64;
            const float Gi = Gs[i], wi = is_a ? bs[i] : 1.f;
#pragma unroll
            for (int j0 = 0; j0 < 64; j0 += 16) {
                float gj[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(Gs + j0 + 4 * u);
                    gj[4 * u] = t4.x; gj[4 * u + 1] = t4.y; gj[4 * u + 2] = t4.z; gj[4 * u + 3] = t4.w;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {   // branch-free: clamped exponent times a 0/1 mask
                    const int j = j0 + u;
                    const float keep = (is_a ? (j < i) : (j <= i)) ? 1.f : 0.f;
                    x[j] = (wi * keep) * __expf(fminf(Gi - gj[u], 0.f)) * x[j];
                }
            }
            if (is_a) {
#pragma unroll
                for (int j = 0; j < 64; ++j) Af[i * TP + j] = x[j];
            } else {
                store_row_bf16(sm + SM_P, i, x);
            }
            PHASE_MARK(19);
        } else {
            for (int e = tid - 128; e < 64 * 64; e += 128) {
                const int i = e >> 6, j = e & 63;
                Tf[i * TP + j] = (i == j) ? 1.f : 0.f;
            }
        }
        __syncthreads();
        PHASE_MARK(4);

        // ---- D: T = (I + A)^-1 (blocked; merges on the warp-level tensor cores in tf32)
        invert_unit_lower_64_tf32<TP>(Af, Tf, tid, c);
        __syncthreads();
        PHASE_MARK(5);
        {   // T' = T diag(beta gamma), T'' = T diag(beta): thread = (matrix, row i, 32 columns)
            const int which = tid >> 7, i = (tid >> 1) & 63, j0 = (tid & 1) * 32;
            float x[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) x[u] = Tf[i * TP + j0 + u];
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
                const float4 b4 = *reinterpret_cast<const float4 *>(bs + j0 + u);
                const float4 g4 = which == 0 ? *reinterpret_cast<const float4 *>(gam + j0 + u)
                                             : make_float4(1.f, 1.f, 1.f, 1.f);
                const float bb[4] = {b4.x * g4.x, b4.y * g4.y, b4.z * g4.z, b4.w * g4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) x[u + e] = (j0 + u + e <= i) ? x[u + e] * bb[e] : 0.f;
            }
            unsigned char *dst = sm + (which ? SM_TPP : SM_TP);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint4 w;
                w.x = pack_bf16(x[8 * cc + 0], x[8 * cc + 1]); w.y = pack_bf16(x[8 * cc + 2], x[8 * cc + 3]);
                w.z = pack_bf16(x[8 * cc + 4], x[8 * cc + 5]); w.w = pack_bf16(x[8 * cc + 6], x[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(dst + sw128(i, j0 / 8 + cc)) = w;
            }
        }
        handoff();
        PHASE_MARK(6);

        // ---- E: P2 W^T = K^T T'^T ; P3 U~^T = V^T T''^T
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, 64, true, false);
            const uint32_t kq = smem_u32(sm + SM_KQ), vt = smem_u32(Vt);
            const uint32_t tp = smem_u32(sm + SM_TP), tpp = smem_u32(sm + SM_TPP);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                umma_bf16(tmem + TM_W, sdesc_mnmajor(kq + s * 2048, 16384), sdesc_kmajor(tp + s * 32), id, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                umma_bf16(tmem + TM_U, sdesc_mnmajor(vt + s * 2048, 8192), sdesc_kmajor(tpp + s * 32), id, s > 0);
        }
        commit_mma();
        if (!mma_sync_wait()) { fail_where = 4; break; }
        PHASE_MARK(7);
        if (c + 1 < nchunks) issue_kq(c + 1);        // K and Q of this chunk are no longer read

        // ---- F: W^T (lane d) -> bf16 rows d of the MN-major B operand
        if (wg == 0) {
            float x[64];
            ld64(tmem + lane_off + TM_W, x);
            store_row_bf16(sm + SM_WT, row, x);
        }
        handoff();
        PHASE_MARK(8);

        // ---- G: S1 U^T = U~^T - S^T W^T
        if (tid == 0) {
            const uint32_t st = smem_u32(sm + SM_ST), wt = smem_u32(sm + SM_WT);
            const uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t a = sdesc_kmajor(st + (s / 4) * 16384 + (s % 4) * 32);
                umma_bf16(tmem + TM_U, a, sdesc_mnmajor(wt + s * 2048, 16384), id_neg, 1);
            }
        }
        commit_mma();
        if (!mma_sync_wait()) { fail_where = 5; break; }
        PHASE_MARK(9);

        // ---- H: U^T -> bf16 A operand (WG0); state scaled by gamma_end in TMEM (WG1)
        if (wg == 0) {
            float x[64];
            ld64(tmem + lane_off + TM_U, x);
            store_row_bf16(sm + SM_UT, row, x);
        } else {
            const float ge = gam[TC_C - 1];
#pragma unroll 1
            for (int d0 = 0; d0 < TC_D; d0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + TM_S + d0, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * ge);
                tmem_st32(tmem + lane_off + TM_S + d0, r);
            }
            tmem_wait_st();
        }
        handoff();
        PHASE_MARK(10);

        // ---- I: S2 S^T += U^T K~ ; S2' (P U)^T = U^T P^T
        if (tid == 0) {
            const uint32_t ut = smem_u32(sm + SM_UT), kt = smem_u32(sm + SM_KT), p = smem_u32(sm + SM_P);
            const uint32_t id_s = idesc_bf16(128, 128, false, true);
            const uint32_t id_p = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t a = sdesc_kmajor(ut + s * 32);
                umma_bf16(tmem + TM_S, a, sdesc_mnmajor(kt + s * 2048, 8192), id_s, 1);
                umma_bf16(tmem + TM_PU, a, sdesc_kmajor(p + s * 32), id_p, s > 0);
            }
        }
        commit_mma();
        if (!mma_sync_wait()) { fail_where = 6; break; }
        PHASE_MARK(11);

        // ---- J: new state -> bf16 S^T (or S_final); outputs
        const bool last = (c + 1 == nchunks);
        if (wg == 0) {
#pragma unroll 1
            for (int d0 = 0; d0 < TC_D; d0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + TM_S + d0, r);
                tmem_wait_ld();
                if (last) {
                    if (S_final) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            S_final[s_off + (size_t)(d0 + j) * TC_D + row] = __uint_as_float(r[j]);
                    }
                } else {
                    unsigned char *st = sm + SM_ST + (d0 / 64) * 16384;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(r[8 * cc + 0]), __uint_as_float(r[8 * cc + 1]));
                        w.y = pack_bf16(__uint_as_float(r[8 * cc + 2]), __uint_as_float(r[8 * cc + 3]));
                        w.z = pack_bf16(__uint_as_float(r[8 * cc + 4]), __uint_as_float(r[8 * cc + 5]));
                        w.w = pack_bf16(__uint_as_float(r[8 * cc + 6]), __uint_as_float(r[8 * cc + 7]));
                        *reinterpret_cast<uint4 *>(st + sw128(row, (d0 % 64) / 8 + cc)) = w;
                    }
                }
            }
            PHASE_MARK(21);
        } else {
            // o_i = scale (gamma_i (Q S)_i + (P U)_i): column v of the chunk's outputs,
            // staged row-major in shared memory, then written as 16-byte row pieces
            const int v = row;
            __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(sm + SM_OST);
#pragma unroll 1
            for (int i0 = 0; i0 < TC_C; i0 += 32) {
                uint32_t o[32], pu[32];
                tmem_ld32(tmem + lane_off + TM_O + i0, o);
                tmem_ld32(tmem + lane_off + TM_PU + i0, pu);
                tmem_wait_ld();
                float gg[32];
#pragma unroll
                for (int u = 0; u < 32; u += 4) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(gam + i0 + u);
                    gg[u] = g4.x; gg[u + 1] = g4.y; gg[u + 2] = g4.z; gg[u + 3] = g4.w;
                }
                __nv_bfloat16 ov[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    ov[j] = __float2bfloat16_rn(scale * (gg[j] * __uint_as_float(o[j]) + __uint_as_float(pu[j])));
#pragma unroll
                for (int j = 0; j < 32; ++j) ost[(i0 + j) * TC_D + v] = ov[j];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");       // the four output warps
            for (int e = tid - 128; e < L * 16; e += 128) {
                const int i = e >> 4, cc = e & 15;
                const uint4 val = *reinterpret_cast<const uint4 *>(ost + i * TC_D + cc * 8);
                *reinterpret_cast<uint4 *>(out + ((size_t)(t0 + i) * H_v + h) * TC_D + cc * 8) = val;
            }
        }
        handoff();
        PHASE_MARK(12);
    }

    if (fail_where) {
        if (tid == 0) record_error(err, GDN_ERR_TIMEOUT, fail_where);
        // let this CTA's own copies and MMAs land before its shared memory and TMEM go
        if (tid == 0) {
            if (pend.kq_issued > pend.kq_done) mbar_wait(bar_kq, pend.kq_done & 1, kDefaultBudget);
            for (int b = 0; b < 2; ++b)
                if (pend.v_issued[b] > pend.v_done[b]) mbar_wait(bar_v + b, pend.v_done[b] & 1, kDefaultBudget);
            if (pend.mma_issued > pend.mma_done) mbar_wait(bar_mma, pend.mma_done & 1, kDefaultBudget);
        }
    } else if (nchunks == 0 && S_final && wg == 0) {
        for (int d = 0; d < TC_D; ++d)
            S_final[s_off + (size_t)d * TC_D + row] = S0 ? S0[s_off + (size_t)d * TC_D + row] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [T_total, H, 128] bf16 -> boxes of 64 tokens x 64 elements (128 B), 128-byte swizzle
bool make_map(CUtensorMap *map, const void *base, long long T_total, int H) {
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T_total};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Poll budget of the kernel's bounded waits.  Test hook: the environment variable
// GDN_TEST_WAIT_BUDGET overrides it (0 makes every wait give up at once, which
// exercises the timeout path without a real hang).
uint32_t wait_budget() {
    const char *env = getenv("GDN_TEST_WAIT_BUDGET");
    return env ? (uint32_t)strtoul(env, nullptr, 10) : kDefaultBudget;
}

}  // namespace

// ------------------------------------------- library-held scratch (no-allocation path)
// Scratch for gdn_prefill_static_scratch: callers that cannot allocate device memory
// still need somewhere for the kernel's error word.  Every GPU that loads the library
// holds this array until the library is unloaded; all calls on a device share it.
static __device__ __align__(256) unsigned char g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};
}  // namespace

size_t static_scratch_capacity() { return GDN_STATIC_SCRATCH_BYTES; }

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) with cudaGetSymbolAddress and cached.
cudaError_t static_scratch_ptr(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

#ifdef GDN_PHASE_TIMERS
extern "C" __attribute__((visibility("default"))) int gdn_debug_phase_clock(void *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_phase_clock, sizeof(g_phase_clock));
}
#endif

bool prefill_tc_supported(int dk, int dv, gdn_dtype dtype)
{
    return dk == TC_D && dv == TC_D && dtype == GDN_BF16;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S0, void *out, float *S_final,
                              const int32_t *cu, int N, long long T_dense, long long T_total,
                              int H_qk, int H_v, float scale, int l2norm, DeviceError *err,
                              cudaStream_t stream)
{
    if (T_total >= (1LL << 31)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, T_total, H_qk) || !make_map(&mk, k, T_total, H_qk) ||
        !make_map(&mv, v, T_total, H_v))
        return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid((unsigned)N, (unsigned)H_v);
    prefill_tc_kernel<<<grid, TC_THREADS, SMEM_BYTES, stream>>>(
        mq, mk, mv, g, beta, S0, (__nv_bfloat16 *)out, S_final, cu, T_dense, H_qk, H_v, scale,
        l2norm, err, wait_budget());
    return cudaGetLastError();
}

}  // namespace gdn
