// Chunked prefill of the gated delta rule, dk = dv = 128, bf16 I/O, on a cluster of
// four sm_100a CTAs per (sequence, value head).
//
// Rule: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身", Eq. (1)
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
// Chunk algebra (C = 64; G_i = in-chunk cumsum of g, gamma_i = exp G_i, S the state
// entering the chunk; an exact re-association of the rule):
//   A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i),  T = (I + A)^-1
//   W = T diag(beta gamma) K,  U~ = T diag(beta) V,  U = U~ - W S
//   O = diag(gamma) Q S + P U,  P_ij = exp(G_i - G_j) q_i.k_j (j <= i)
//   S <- gamma_end S + K~^T U,  K~_j = exp(G_end - G_j) k_j
//
// Work split.  The value columns of S evolve independently, so CTA r of the cluster
// owns columns [32r, 32r + 32) of S, U and O for the whole sequence and runs the
// sequential state chain for them:
//     WS = W S_r -> U_r = U~_r - WS -> S_r <- gamma_end S_r + K~^T U_r -> next chunk,
// with Q S_r and P U_r for the outputs off that chain.  The per-chunk quantities that
// do not depend on the value columns (P, the inverse T, W, U~) are computed once per
// chunk, by CTA (chunk mod 4), several chunks ahead of the state chain.  They travel
// through L2: the producer bulk-stores W, P and all four U~ slices (already in the
// shared-memory tile layout) into the chunk's slot of a small global ring, signals the
// four CTAs, and each bulk-loads W, P and its own slice into its two-slot ring.  (DSMEM
// copies from one SM run at about 20 B/cycle, which capped the producer; L2 does not.)
//
// Roles inside a CTA (448 threads):
//   warps 0-3    chain group:  U epilogue and state epilogue; its first thread issues
//                              the chain's MMAs WS = W S_r and S2 = K~^T U_r; thread 32
//                              issues PU = P U_r
//   warps 4-7    prep group:   inputs fix-up, A/P epilogue, triangular inverse, T'/T'',
//                              W/U~ epilogue into the store staging
//   warp 8       chain issuer: TMA for Q, MMA QS = Q S_r (queued behind WS), the ring
//                              (bulk loads of ready chunks, receipts to the producers)
//   warp 9       prep issuer:  TMA for the prepared chunk, MMAs P1 ([K;Q]K^T), W, U~,
//                              bulk stores into the L2 ring, ready signals
//   warps 10-13  aux group:    per-chunk vectors, K~ build, output epilogue
// Accumulators live in TMEM; the state slice S_r (128 x 32 fp32) stays in TMEM for the
// whole sequence.  Every wait is bounded; a CTA whose wait runs out records
// GDN_ERR_TIMEOUT, raises its abort flag so its other roles stop, drains its own
// copies and MMAs, and leaves through the final cluster barrier.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "tri_inverse.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int K4_C = 64;                 // chunk
constexpr int K4_D = 128;                // dk = dv
constexpr int K4_SL = 32;                // value columns per CTA
constexpr int K4_THREADS = 448;
constexpr uint32_t K4_DEFAULT_BUDGET = 1u << 22;
constexpr uint32_t K4_RING_BYTES = 28672;    // W 16 KB + P 8 KB + U~ slice 4 KB
// Prepared chunks travel through L2: the producer writes W, P and all four U~ slices of a
// chunk into one 40 KB global chunk slot (already in the shared-memory tile layout), and
// each consumer bulk-loads W, P and its own slice into its ring.  A cluster owns 8 chunk
// slots (chunk p uses slot p mod 8), taken from a library-held pool.
constexpr uint32_t K4_GCHUNK = 40960;        // W 16 KB | P 8 KB | U~ 4 x 4 KB
constexpr uint32_t K4_GCLUSTER = 8 * K4_GCHUNK;
constexpr int K4_POOL = 64;                  // cluster slots (more than can be resident)

// TMEM columns (512 allocated)
constexpr uint32_t T4_S = 0;       // 32: S_r (lane = key dim d, col = value v)
constexpr uint32_t T4_WS = 32;     // 32: W S_r      (M = 64 layout)
constexpr uint32_t T4_QS = 64;     // 2 x 32: Q S_r  (M = 64 layout, double-buffered)
constexpr uint32_t T4_PU = 128;    // 2 x 32: P U_r  (M = 64 layout, double-buffered)
constexpr uint32_t T4_KQ = 192;    // 64: [K;Q] K^T (M = 128)
constexpr uint32_t T4_W = 256;     // 128: T' K     (M = 64 layout)
constexpr uint32_t T4_U = 384;     // 128: T'' V    (M = 64 layout)

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t S4_CQ = 0;          // 16 KB Q of the chain's chunk [cg0 | cg1]
constexpr uint32_t S4_CK = 16384;      // 16 KB K of the chain's chunk
constexpr uint32_t S4_CKT = 32768;     // 16 KB K~
constexpr uint32_t S4_ST = 49152;      // 8 KB S_r bf16, rows d of 64 B (MN-major B, 64-byte swizzle)
constexpr uint32_t S4_UT = 57344;      // 4 KB U_r bf16, rows i of 64 B (MN-major B, 64-byte swizzle)
constexpr uint32_t S4_RING = 61440;    // 2 slots x 28 KB: W (16 KB) | P (8 KB) | U~_r (4 KB)
constexpr uint32_t S4_PKQ = 118784;    // 32 KB [K cg0 | Q cg0 | K cg1 | Q cg1] of the prepared chunk
constexpr uint32_t S4_PV = 151552;     // 16 KB V of the prepared chunk
constexpr uint32_t S4_TP = 167936;     // 8 KB T' = T diag(beta gamma)
constexpr uint32_t S4_TPP = 176128;    // 8 KB T'' = T diag(beta)
constexpr uint32_t S4_PSTG = 184320;   // 8 KB P staging (store source)
constexpr uint32_t S4_AF = 192512;     // fp32 A 64 x 65 (overlaid later by the W staging)
constexpr uint32_t S4_TF = 209152;     // fp32 T 64 x 65 (overlaid later by the U~ staging)
constexpr uint32_t S4_WSTG = 192512;   // 16 KB W staging
constexpr uint32_t S4_USTG = 208896;   // 16 KB U~ staging, 4 slices x [64 rows x 32 v]
constexpr uint32_t S4_CVEC = 225792;   // chain vectors, 2 buffers x {g, beta, G, gamma, dte} x 64
constexpr uint32_t S4_PVEC = 228352;   // prep vectors {g, beta, G, gamma, exp(-G)} x 64
constexpr uint32_t S4_BAR = 229632;    // mbarriers
constexpr uint32_t S4_MISC = S4_BAR + 48 * 8;   // tmem base, abort flag, cluster's ring slot
constexpr uint32_t S4_END = S4_MISC + 16;
constexpr uint32_t K4_SMEM = S4_END + 1024;
constexpr int TP4 = 65;

enum Bar {
    B_CQ = 0, B_CK, B_FULL0, B_FULL1, B_QS, B_WS, B_S2, B_KT, B_OFREE0, B_OFREE1,
    B_PKQ, B_PV, B_P1, B_TT, B_WU, B_PIN, B_CQN, B_VEC0, B_VEC1, B_PU0, B_PU1, B_WSI,
    B_STG,                                 // producer: staging written
    B_SFREE,                               // producer: staging read by the bulk stores
    B_GFREE0, B_GFREE1,                    // producer: all four CTAs loaded its chunk slot
    B_READY,                               // consumer: chunk p's slot written (8: p mod 8)
    B_COUNT = B_READY + 8
};
static_assert(B_COUNT <= 48, "barrier area holds 48");

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ float2 unpack2(uint32_t x) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x));
}
template <int ID>
__device__ __forceinline__ void group_sync() {
    asm volatile("bar.sync %0, 128;" ::"n"(ID) : "memory");
}
// all 128 threads of named barrier ID must call; returns the AND of `v`
template <int ID>
__device__ __forceinline__ bool group_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"(v ? 1u : 0u), "n"(ID) : "memory");
    return r != 0;
}
// row r (32 fp32 values, bit patterns) of a 64-byte-swizzled bf16 tile
__device__ __forceinline__ void store_row32(unsigned char *tile, int r, const uint32_t (&x)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4 *>(tile + sw64(r, c)) = make_uint4(
            pack2(__uint_as_float(x[8 * c]), __uint_as_float(x[8 * c + 1])),
            pack2(__uint_as_float(x[8 * c + 2]), __uint_as_float(x[8 * c + 3])),
            pack2(__uint_as_float(x[8 * c + 4]), __uint_as_float(x[8 * c + 5])),
            pack2(__uint_as_float(x[8 * c + 6]), __uint_as_float(x[8 * c + 7])));
}
// wait for the last of `issued` phases of `bar` (phases complete in order); used only
// while draining after an abort, so it ignores the abort flag
__device__ __forceinline__ void drain_bar(uint64_t *bar, int issued, bool cluster_scope,
                                          uint32_t budget = K4_DEFAULT_BUDGET) {
    if (issued <= 0) return;
    const uint32_t par = (uint32_t)((issued - 1) & 1);
    if (cluster_scope) mbar_wait_cluster(bar, par, budget);
    else mbar_wait(bar, par, budget);
}

}  // namespace

// Library-held L2 ring for prepared chunks (see K4_GCHUNK) and the pool of its cluster
// slots: a cluster claims a free slot when it starts and returns it when it ends.
static __device__ __align__(1024) unsigned char g4_ring[(size_t)K4_POOL * K4_GCLUSTER];
static __device__ int g4_pool[K4_POOL];


// Cold path, kept out of line so its code is not repeated at every wait: the first role
// of a CTA whose wait runs out records the error and raises the CTA's abort flag.
__device__ __noinline__ void raise_abort(volatile int *abort_flag, DeviceError *err, int where)
{
    if (!*abort_flag) {
        *abort_flag = 1;
        record_error(err, GDN_ERR_TIMEOUT, where);
    }
}

// L2N: q and k are L2-normalised in the kernel (a separate instantiation, so the common
// case carries none of that code)
template <bool L2N>
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(K4_THREADS, 1)
prefill_tc_cluster_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
                          const float *__restrict__ beta, const float *S0,
                          __nv_bfloat16 *__restrict__ out, float *S_final,
                          const int32_t *__restrict__ cu_seqlens, long long T_dense, int H_qk,
                          int H_v, float scale, int opts, DeviceError *err, uint32_t budget)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t r = cluster_rank();
    const int n = blockIdx.x >> 2, h = blockIdx.y;
    const int hq = h / (H_v / H_qk);
    long long t_begin, t_end;
    if (cu_seqlens) { t_begin = cu_seqlens[n]; t_end = cu_seqlens[n + 1]; }
    else { t_begin = (long long)n * T_dense; t_end = t_begin + T_dense; }
    const int nch = (int)((t_end - t_begin + K4_C - 1) / K4_C);
    const size_t s_off = ((size_t)n * H_v + h) * K4_D * K4_D;
    const int v0 = (int)r * K4_SL;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S4_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S4_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S4_MISC + 4);

    if (warp == 8) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
    if (tid == 256) {
        for (int b = 0; b < B_COUNT; ++b) mbar_init(bars + b, (b == B_GFREE0 || b == B_GFREE1) ? 4 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (r == 0) {                          // claim a ring slot for the cluster
            int slot = -1;
            for (int round = 0; round < 4096 && slot < 0; ++round) {
                for (int i = 0; i < K4_POOL && slot < 0; ++i)
                    if (atomicCAS(&g4_pool[i], 0, 1) == 0) slot = i;
                if (slot < 0) __nanosleep(1000);
            }
            *reinterpret_cast<volatile int *>(sm + S4_MISC + 8) = slot;
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int ring_slot = (int)ld_cluster_u32(map_to_rank(sm + S4_MISC + 8, 0));
    unsigned char *gring = g4_ring + (size_t)(ring_slot < 0 ? 0 : ring_slot) * K4_GCLUSTER;
    if (ring_slot < 0 && tid == 0) record_error(err, GDN_ERR_TIMEOUT, 90);

    // bounded wait; gives up early if another role of this CTA has aborted
    auto wait_bar = [&](int b, uint32_t parity, bool cluster_scope) -> bool {
        uint64_t *bar = bars + b;
        for (uint32_t i = 0; i < budget; ++i) {
            if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
            if (*abort_flag) return false;
        }
        return false;
    };
    auto fail = [&](int where) { raise_abort(abort_flag, err, where); };

    if (ring_slot < 0) {
        // no ring slot could be claimed: the error is recorded, nothing else runs
    } else if (warp < 4) {
        // =========================================================== chain group
        // The two CUDA-core steps of the state chain (U epilogue, state epilogue).  The
        // group's first thread also issues the chain's MMAs itself (W S_r, then K~^T U_r
        // with P U_r behind it), so no hand-off to another warp sits on the chain.
        const int t = tid, q = warp, l = lane;
        const int d = 32 * q + l;                        // TMEM lane = key dim of S_r
        const int i_row = 16 * q + l;                    // row of M = 64 results (l < 16)
        const uint32_t loff = (uint32_t)(32 * q) << 16;
        const float *cvec0 = reinterpret_cast<const float *>(sm + S4_CVEC);
        const unsigned char *ring = sm + S4_RING;
        const uint32_t st = smem_u32(sm + S4_ST), ut = smem_u32(sm + S4_UT), kt = smem_u32(sm + S4_CKT);
        const uint32_t id_m64 = idesc_bf16(64, 32, false, true);     // B = S_r or U_r rows
        const uint32_t id_s2 = idesc_bf16(128, 32, true, true);
        int ws_req = 0, s2_req = 0, pu_req0 = 0, pu_req1 = 0;    // MMA groups issued
        bool ok = true;
        // descriptors step by a fixed amount per 16-deep K slice (the address field is in
        // 16-byte units): K-major SW128 +32 B, 64-byte-row MN-major +1024 B, SW128
        // MN-major +2048 B; the second 64-wide K block of a K-major tile is +8192 B

        // W S_r for chunk cc once its ring slot has arrived (thread 0 only).  B_WSI tells
        // the issuer warp, which then queues Q S_r behind it.
        auto issue_ws = [&](int cc) -> bool {
            const int sc = cc & 1;
            if (!wait_bar(sc ? B_FULL1 : B_FULL0, (cc >> 1) & 1, false)) return false;
            tc_fence_after();
            const uint64_t d_w = sdesc_kmajor(smem_u32(sm + S4_RING + sc * K4_RING_BYTES));
            const uint64_t d_st = sdesc_mn_sw64(st);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16(tmem + T4_WS, d_w + (ks >> 2) * 512 + (ks & 3) * 2, d_st + ks * 64, id_m64, ks > 0);
            umma_commit(bars + B_WS);
            mbar_arrive_local(bars + B_WSI);
            ++ws_req;
            return true;
        };

        // initial state slice: D_S = gamma_end(0) S0_r, S_r (bf16) = S0_r
        float x[32];
        {
            const float *src = S0 ? S0 + s_off + (size_t)d * K4_D + v0 : nullptr;
#pragma unroll
            for (int v = 0; v < 32; v += 4) {
                const float4 f = src ? *reinterpret_cast<const float4 *>(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[v] = f.x; x[v + 1] = f.y; x[v + 2] = f.z; x[v + 3] = f.w;
            }
        }
        if (nch == 0) {
            if (S_final) {
                float *dst = S_final + s_off + (size_t)d * K4_D + v0;
#pragma unroll
                for (int v = 0; v < 32; v += 4) *reinterpret_cast<float4 *>(dst + v) = make_float4(x[v], x[v + 1], x[v + 2], x[v + 3]);
            }
        } else if (!group_all<1>(t != 0 || wait_bar(B_VEC0, 0, false))) {
            fail(15);
            ok = false;
        } else {
            const float ge0 = cvec0[192 + 63];
            uint32_t rr[32];
#pragma unroll
            for (int v = 0; v < 32; ++v) rr[v] = __float_as_uint(x[v]);
            store_row32(sm + S4_ST, d, rr);
#pragma unroll
            for (int v = 0; v < 32; ++v) rr[v] = __float_as_uint(ge0 * x[v]);
            tmem_st32(tmem + loff + T4_S, rr);
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            group_sync<1>();
            bool okw = true;
            if (t == 0) okw = issue_ws(0);
            if (!group_all<1>(okw)) { fail(31); ok = false; }
        }

#pragma unroll 1
        for (int c = 0; ok && c < nch; ++c) {
            const int s = c & 1;
            // ---- U_r = U~_r - W S_r  ->  U_r (bf16, rows i).  The previous chunk's P U_r
            // (issued by thread 32, so not covered by thread 0's commits) read U_r too.
            if (!group_all<1>(t != 0 || (wait_bar(B_WS, c & 1, false) &&
                                         (c == 0 || wait_bar((c & 1) ? B_PU0 : B_PU1, ((c - 1) >> 1) & 1, false))))) {
                fail(12);
                break;
            }
            tc_fence_after();
            {
                uint32_t ws[32];
                tmem_ld32(tmem + loff + T4_WS, ws);
                tmem_wait_ld();
                if (l < 16) {
                    const unsigned char *us = ring + s * K4_RING_BYTES + 24576 + i_row * 64;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(us + cc * 16);
                        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = unpack2(wv[e]);
                            ws[8 * cc + 2 * e] = __float_as_uint(f.x - __uint_as_float(ws[8 * cc + 2 * e]));
                            ws[8 * cc + 2 * e + 1] = __float_as_uint(f.y - __uint_as_float(ws[8 * cc + 2 * e + 1]));
                        }
                    }
                    store_row32(sm + S4_UT, i_row, ws);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<1>();

            // ---- S_r += K~^T U_r on the chain (thread 0) and P U_r -> D_PU[s] beside it
            // (thread 32).  gamma_end of the next chunk is waited for before S2, so this
            // group can never be lapped by the group that signals it.
            {
                bool oks = true;
                if (t == 0) {
                    oks = wait_bar(B_KT, c & 1, false) &&
                          (c + 1 >= nch || wait_bar(((c + 1) & 1) ? B_VEC1 : B_VEC0, ((c + 1) >> 1) & 1, false));
                    if (oks) {
                        tc_fence_after();
                        const uint64_t d_kt = sdesc_mnmajor(kt, 8192), d_ut = sdesc_mn_sw64(ut);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            umma_bf16(tmem + T4_S, d_kt + ks * 128, d_ut + ks * 64, id_s2, 1);
                        umma_commit(bars + B_S2);
                        ++s2_req;
                    }
                } else if (t == 32) {
                    oks = wait_bar(s ? B_OFREE1 : B_OFREE0, (c >> 1) & 1, false);
                    if (oks) {
                        tc_fence_after();
                        const uint64_t d_p = sdesc_kmajor(smem_u32(sm + S4_RING + s * K4_RING_BYTES + 16384));
                        const uint64_t d_ut = sdesc_mn_sw64(ut);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            umma_bf16(tmem + T4_PU + 32 * s, d_p + ks * 2, d_ut + ks * 64, id_m64, ks > 0);
                        umma_commit(bars + (s ? B_PU1 : B_PU0));
                        if (s) ++pu_req1; else ++pu_req0;
                    }
                }
                if (!group_all<1>(oks)) { fail(13); break; }
            }
            const float ge_next = (c + 1 < nch) ? cvec0[((c + 1) & 1) * 320 + 192 + 63] : 1.f;

            // ---- state: S_r (bf16) for the next chunk's products first (that is what the
            // next W S_r waits for), then D_S <- gamma_end(c+1) S_r (needed only by the next S2)
            if (!group_all<1>(t != 0 || wait_bar(B_S2, c & 1, false))) { fail(14); break; }
            tc_fence_after();
            uint32_t rs[32];
            tmem_ld32(tmem + loff + T4_S, rs);
            tmem_wait_ld();
            if (c + 1 == nch) {
                if (S_final) {
                    float *dst = S_final + s_off + (size_t)d * K4_D + v0;
#pragma unroll
                    for (int v = 0; v < 32; v += 4)
                        *reinterpret_cast<float4 *>(dst + v) = make_float4(
                            __uint_as_float(rs[v]), __uint_as_float(rs[v + 1]),
                            __uint_as_float(rs[v + 2]), __uint_as_float(rs[v + 3]));
                }
                break;
            }
            // Q S_r of this chunk reads the tile about to be replaced
            if (!group_all<1>(t != 0 || wait_bar(B_QS, c & 1, false))) { fail(17); break; }
            store_row32(sm + S4_ST, d, rs);
            fence_proxy_async();
            group_sync<1>();
            bool okw = true;
            if (t == 0) okw = issue_ws(c + 1);
#pragma unroll
            for (int v = 0; v < 32; ++v) rs[v] = __float_as_uint(ge_next * __uint_as_float(rs[v]));
            tmem_st32(tmem + loff + T4_S, rs);
            tmem_wait_st();
            tc_fence_before();
            if (!group_all<1>(okw)) { fail(18); break; }
        }
        if (*abort_flag) {
            if (t == 0) {
                drain_bar(bars + B_WS, ws_req, false);
                drain_bar(bars + B_S2, s2_req, false);
            } else if (t == 32) {
                drain_bar(bars + B_PU0, pu_req0, false);
                drain_bar(bars + B_PU1, pu_req1, false);
            }
        }
    } else if (warp >= 10) {
        // ============================================================ aux group
        // per-chunk vectors, K~ build, Q normalisation, output epilogue (all off the chain)
        const int t = tid - 320, qd = warp & 3, l = lane;
        const int i_row = 16 * qd + l;                   // row of M = 64 results (l < 16)
        const uint32_t loff = (uint32_t)(32 * qd) << 16;
        float *cvec0 = reinterpret_cast<float *>(sm + S4_CVEC);
        int k_issued = nch > 0 ? 1 : 0;                  // K tiles requested (the first by warp 8)
        float pre_g = 0.f, pre_b = 0.f;
        auto fetch_vectors = [&](int c) {                // g, beta of chunk c into registers
            const long long t0 = t_begin + (long long)c * K4_C;
            const int L = (int)min((long long)K4_C, t_end - t0);
            pre_g = (t < L) ? gate_log_decay(g[(size_t)(t0 + t) * H_v + h], opts) : 0.f;
            pre_b = (t < L) ? gate_strength(beta[(size_t)(t0 + t) * H_v + h], opts) : 0.f;
        };
        auto finish_vectors = [&](int c) {               // G, gamma, decay-to-end; then signal
            float *cv = cvec0 + (c & 1) * 320;
            float *cg = cv, *cb = cv + 64, *cG = cv + 128, *cgam = cv + 192, *cdte = cv + 256;
            if (t < K4_C) { cg[t] = pre_g; cb[t] = pre_b; }
            group_sync<3>();
            if (qd == 0 && warp == 12) {
                const float a0 = cg[2 * l], a1 = cg[2 * l + 1];
                float sc = a0 + a1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, sc, o);
                    if (l >= o) sc += y;
                }
                const float G0 = sc - a1, G1 = sc, Ge = __shfl_sync(0xffffffffu, sc, 31);
                cG[2 * l] = G0; cG[2 * l + 1] = G1;
                cgam[2 * l] = expf(G0); cgam[2 * l + 1] = expf(G1);
                cdte[2 * l] = expf(Ge - G0); cdte[2 * l + 1] = expf(Ge - G1);
            }
            group_sync<3>();
            if (t == 0) mbar_arrive_local(bars + ((c & 1) ? B_VEC1 : B_VEC0));
        };
        auto normalise_rows = [&](unsigned char *tile) {  // 64 rows x 128 bf16, two threads per row
            const int row = t >> 1, half = t & 1;
            unsigned char *rp = tile + half * 8192 + row * 128;
            float ss = 0.f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint4 w = *reinterpret_cast<const uint4 *>(rp + cc * 16);
                const uint32_t wsv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) { const float2 f = unpack2(wsv[e]); ss += f.x * f.x + f.y * f.y; }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float rn = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 w = *reinterpret_cast<const uint4 *>(rp + cc * 16);
                uint32_t wsv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) { const float2 f = unpack2(wsv[e]); wsv[e] = pack2(f.x * rn, f.y * rn); }
                *reinterpret_cast<uint4 *>(rp + cc * 16) = make_uint4(wsv[0], wsv[1], wsv[2], wsv[3]);
            }
        };

        if (nch > 0) {
            if (t < K4_C) fetch_vectors(0);
            finish_vectors(0);
        }
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const long long t0 = t_begin + (long long)c * K4_C;
            const int L = (int)min((long long)K4_C, t_end - t0);
            const int s = c & 1;
            const float *cv = cvec0 + s * 320;
            const float *cgam = cv + 192, *cdte = cv + 256;
            if (t < K4_C && c + 1 < nch) fetch_vectors(c + 1);   // lands while this chunk runs

            // ---- K~(c) = diag(decay to chunk end) K; rows past the end get weight 0
            if (!group_all<3>(t != 0 || wait_bar(B_CK, c & 1, false))) { fail(10); break; }
            if (c >= 1 && !group_all<3>(t != 0 || wait_bar(B_S2, (c - 1) & 1, false))) { fail(17); break; }
            if constexpr (L2N) { normalise_rows(sm + S4_CK); group_sync<3>(); }
#pragma unroll 2
            for (int u = 0; u < 8; ++u) {
                const int e = t + 128 * u;
                const int cg = e >> 9, row = (e >> 3) & 63, cc = e & 7;
                const uint4 w = *reinterpret_cast<const uint4 *>(sm + S4_CK + cg * 8192 + row * 128 + cc * 16);
                const float wt = row < L ? cdte[row] : 0.f;
                const uint32_t wsv[4] = {w.x, w.y, w.z, w.w};
                uint32_t o[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) { const float2 f = unpack2(wsv[e2]); o[e2] = pack2(f.x * wt, f.y * wt); }
                *reinterpret_cast<uint4 *>(sm + S4_CKT + cg * 8192 + row * 128 + cc * 16) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async();
            group_sync<3>();
            if (t == 0) {
                mbar_arrive_local(bars + B_KT);
                if (c + 1 < nch) {             // K of the next chunk into the free buffer
                    ++k_issued;
                    const int tn = (int)(t0 + K4_C);
                    mbar_arrive_expect_tx(bars + B_CK, 16384);
                    tma_load_3d(sm + S4_CK, &tm_k, bars + B_CK, 0, hq, tn);
                    tma_load_3d(sm + S4_CK + 8192, &tm_k, bars + B_CK, 64, hq, tn);
                }
            }
            if constexpr (L2N) {               // Q of this chunk, for Q S_r
                if (!group_all<3>(t != 0 || wait_bar(B_CQ, c & 1, false))) { fail(11); break; }
                normalise_rows(sm + S4_CQ);
                fence_proxy_async();
                group_sync<3>();
                if (t == 0) mbar_arrive_local(bars + B_CQN);
            }

            // ---- vectors of the next chunk (the chain scales the state by its gamma_end)
            if (c + 1 < nch) finish_vectors(c + 1);

            // ---- outputs: o_i = scale (gamma_i (Q S_r)_i + (P U_r)_i), columns [v0, v0 + 32)
            if (!group_all<3>(t != 0 || (wait_bar(B_QS, c & 1, false) &&
                                         wait_bar(s ? B_PU1 : B_PU0, (c >> 1) & 1, false)))) { fail(19); break; }
            tc_fence_after();
            {
                uint32_t qs[32], pu[32];
                tmem_ld32(tmem + loff + T4_QS + 32 * s, qs);
                tmem_ld32(tmem + loff + T4_PU + 32 * s, pu);
                tmem_wait_ld();
                if (l < 16 && i_row < L) {
                    const float gi = cgam[i_row];
                    __nv_bfloat16 *dst = out + ((size_t)(t0 + i_row) * H_v + h) * K4_D + v0;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint4 w;
                        uint32_t *pw = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int v = 8 * cc + 2 * e;
                            pw[e] = pack2(scale * (gi * __uint_as_float(qs[v]) + __uint_as_float(pu[v])),
                                          scale * (gi * __uint_as_float(qs[v + 1]) + __uint_as_float(pu[v + 1])));
                        }
                        *reinterpret_cast<uint4 *>(dst + 8 * cc) = w;
                    }
                }
            }
            tc_fence_before();
            group_sync<3>();
            if (t == 0) mbar_arrive_local(bars + (s ? B_OFREE1 : B_OFREE0));
        }
        if (*abort_flag && t == 0) drain_bar(bars + B_CK, k_issued, false);
    } else if (warp < 8) {
        // ============================================================= prep group
        const int t = tid - 128, q = warp - 4, l = lane;
        const int row = 32 * q + l;                        // TMEM lane
        const uint32_t loff = (uint32_t)(32 * q) << 16;
        float *pg = reinterpret_cast<float *>(sm + S4_PVEC);
        float *pb = pg + 64, *pG = pg + 128, *pgam = pg + 192, *pinv = pg + 256;
        float *Af = reinterpret_cast<float *>(sm + S4_AF);
        float *Tf = reinterpret_cast<float *>(sm + S4_TF);

        // g and beta of production k's chunk, loaded into registers one production ahead
        float nxt_g = 0.f, nxt_b = 0.f;
        auto fetch_gb = [&](int pp) {
            const long long tt = t_begin + (long long)pp * K4_C;
            const int LL = (int)min((long long)K4_C, t_end - tt);
            nxt_g = (t < LL) ? gate_log_decay(g[(size_t)(tt + t) * H_v + h], opts) : 0.f;
            nxt_b = (t < LL) ? gate_strength(beta[(size_t)(tt + t) * H_v + h], opts) : 0.f;
        };
        if ((int)r < nch && t < K4_C) fetch_gb((int)r);
#pragma unroll 1
        for (int k = 0;; ++k) {
            const int p = (int)r + 4 * k;
            if (p >= nch) break;
            const long long t0 = t_begin + (long long)p * K4_C;
            const int L = (int)min((long long)K4_C, t_end - t0);
            if (t < K4_C) { pg[t] = nxt_g; pb[t] = nxt_b; }
            group_sync<2>();
            if (q == 0) {
                const float a0 = pg[2 * l], a1 = pg[2 * l + 1];
                float s = a0 + a1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, o);
                    if (l >= o) s += y;
                }
                const float G0 = s - a1, G1 = s;
                pG[2 * l] = G0; pG[2 * l + 1] = G1;
                pgam[2 * l] = expf(G0); pgam[2 * l + 1] = expf(G1);
                pinv[2 * l] = expf(-G0); pinv[2 * l + 1] = expf(-G1);
            }
            // ---- inputs: rows past the end zeroed, optional q/k normalisation
            if (!group_all<2>(t != 0 || (wait_bar(B_PKQ, k & 1, false) && wait_bar(B_PV, k & 1, false)))) { fail(20); break; }
            if (L < K4_C) {
                const int zr = K4_C - L;
                for (int e = t; e < 6 * zr * 8; e += 128) {
                    const int region = e / (zr * 8), rr = L + (e % (zr * 8)) / 8, cc = e % 8;
                    unsigned char *base = region < 4 ? sm + S4_PKQ + region * 8192 : sm + S4_PV + (region - 4) * 8192;
                    *reinterpret_cast<uint4 *>(base + rr * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
                }
                group_sync<2>();
            }
            if constexpr (L2N) {           // thread t: row t of [K;Q] (both 128-byte halves)
                unsigned char *r0 = sm + S4_PKQ + (t >= 64 ? 8192 : 0) + (t & 63) * 128;
                float ss = 0.f;
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(r0 + half * 16384 + cc * 16);
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) { const float2 f = unpack2(ws[e]); ss += f.x * f.x + f.y * f.y; }
                    }
                const float rn = rsqrtf(ss + 1e-6f);
#pragma unroll
                for (int half = 0; half < 2; ++half)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        uint4 w = *reinterpret_cast<const uint4 *>(r0 + half * 16384 + cc * 16);
                        uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) { const float2 f = unpack2(ws[e]); ws[e] = pack2(f.x * rn, f.y * rn); }
                        *reinterpret_cast<uint4 *>(r0 + half * 16384 + cc * 16) = make_uint4(ws[0], ws[1], ws[2], ws[3]);
                    }
            }
            fence_proxy_async();
            group_sync<2>();
            if (t == 0) mbar_arrive_local(bars + B_PIN);

            // ---- the previous production's staging (overlaying A, T and P) has been read by
            // its bulk stores
            if (k >= 1 && !group_all<2>(t != 0 || wait_bar(B_SFREE, (k - 1) & 1, false))) { fail(21); break; }
            if (!group_all<2>(t != 0 || wait_bar(B_P1, k & 1, false))) { fail(22); break; }
            tc_fence_after();

            // ---- A (fp32, rows 0..63) and P (bf16, rows 64..127) from [K;Q] K^T
            {
                const bool is_a = q < 2;
                const int i = is_a ? row : row - 64;
                const float Gi = pG[i], wi = is_a ? pb[i] : 1.f;
                // exp(G_i - G_j) = exp(G_i) exp(-G_j) is exact enough and in range while the
                // chunk's total log-decay stays above -80 (the usual case, uniform across
                // the CTA); otherwise each factor is exponentiated from the clamped difference
                const bool factored = pG[63] > -80.f;
                const float wi_e = wi * pgam[i];
                const int jend = 32 * ((q & 1) + 1);         // columns past this are masked for the warp
#pragma unroll 1
                for (int j0 = 0; j0 < 64; j0 += 16) {
                    float xv[16];
                    if (j0 >= jend) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) xv[u] = 0.f;
                        if (is_a) continue;                  // the inverse never reads A above the diagonal
                    } else {
                        uint32_t kr[16];
                        tmem_ld16(tmem + loff + T4_KQ + j0, kr);
                        float fj[16];
                        const float *fsrc = factored ? pinv : pG;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float4 g4 = *reinterpret_cast<const float4 *>(fsrc + j0 + 4 * u);
                            fj[4 * u] = g4.x; fj[4 * u + 1] = g4.y; fj[4 * u + 2] = g4.z; fj[4 * u + 3] = g4.w;
                        }
                        tmem_wait_ld();
                        if (factored) {
#pragma unroll
                            for (int u = 0; u < 16; ++u) {
                                const int j = j0 + u;
                                const bool keep = is_a ? (j < i) : (j <= i);
                                xv[u] = keep ? wi_e * fj[u] * __uint_as_float(kr[u]) : 0.f;
                            }
                        } else {
#pragma unroll
                            for (int u = 0; u < 16; ++u) {
                                const int j = j0 + u;
                                const float keep = (is_a ? (j < i) : (j <= i)) ? 1.f : 0.f;
                                xv[u] = (wi * keep) * __expf(fminf(Gi - fj[u], 0.f)) * __uint_as_float(kr[u]);
                            }
                        }
                    }
                    if (is_a) {
#pragma unroll
                        for (int u = 0; u < 16; ++u) Af[i * TP4 + j0 + u] = xv[u];
                    } else {
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2)
                            *reinterpret_cast<uint4 *>(sm + S4_PSTG + sw128(i, (j0 >> 3) + h2)) = make_uint4(
                                pack2(xv[8 * h2 + 0], xv[8 * h2 + 1]), pack2(xv[8 * h2 + 2], xv[8 * h2 + 3]),
                                pack2(xv[8 * h2 + 4], xv[8 * h2 + 5]), pack2(xv[8 * h2 + 6], xv[8 * h2 + 7]));
                    }
                }
                // the inverse writes the diagonal 16 x 16 blocks and the blocks below them; of
                // the blocks above, it reads only T[0:16, 16:32] and T[32:48, 48:64]
#pragma unroll
                for (int e = t; e < 512; e += 128) {
                    const int blk = e >> 8, ii = (e >> 4) & 15, jj = e & 15;
                    Tf[(32 * blk + ii) * TP4 + 32 * blk + 16 + jj] = 0.f;
                }
            }
            tc_fence_before();
            group_sync<2>();

            if (p + 4 < nch && t < K4_C) fetch_gb(p + 4);    // lands during the inverse
            // ---- T = (I + A)^-1
            invert_unit_lower_64_tf32_wg<TP4>(Af, Tf, t, [] { group_sync<2>(); });
            group_sync<2>();

            // ---- T' = T diag(beta gamma), T'' = T diag(beta) (bf16, K-major rows i)
            {
                const int which = t >> 6, i = t & 63;
                unsigned char *dst = sm + (which ? S4_TPP : S4_TP);
#pragma unroll 2
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (8 * cc <= i) {                       // T is lower triangular
                        float w8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 8 * cc + e;
                            const float sc = which ? pb[j] : pb[j] * pgam[j];
                            w8[e] = (j <= i) ? Tf[i * TP4 + j] * sc : 0.f;
                        }
                        o = make_uint4(pack2(w8[0], w8[1]), pack2(w8[2], w8[3]), pack2(w8[4], w8[5]), pack2(w8[6], w8[7]));
                    }
                    *reinterpret_cast<uint4 *>(dst + sw128(i, cc)) = o;
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<2>();
            if (t == 0) mbar_arrive_local(bars + B_TT);

            // ---- W and U~ (M = 64 layout) into the staging
            if (!group_all<2>(t != 0 || wait_bar(B_WU, k & 1, false))) { fail(23); break; }
            tc_fence_after();
            const int i = 16 * q + l;                        // valid for l < 16
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t rw[32];
                tmem_ld32(tmem + loff + T4_W + 32 * cb, rw);
                tmem_wait_ld();
                if (l < 16) {
                    unsigned char *dst = sm + S4_WSTG + (cb >> 1) * 8192;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint32_t *f = rw + 8 * cc;
                        *reinterpret_cast<uint4 *>(dst + sw128(i, (cb & 1) * 4 + cc)) = make_uint4(
                            pack2(__uint_as_float(f[0]), __uint_as_float(f[1])), pack2(__uint_as_float(f[2]), __uint_as_float(f[3])),
                            pack2(__uint_as_float(f[4]), __uint_as_float(f[5])), pack2(__uint_as_float(f[6]), __uint_as_float(f[7])));
                    }
                }
                tmem_ld32(tmem + loff + T4_U + 32 * cb, rw);
                tmem_wait_ld();
                if (l < 16) {
                    unsigned char *dst = sm + S4_USTG + cb * 4096 + i * 64;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint32_t *f = rw + 8 * cc;
                        *reinterpret_cast<uint4 *>(dst + cc * 16) = make_uint4(
                            pack2(__uint_as_float(f[0]), __uint_as_float(f[1])), pack2(__uint_as_float(f[2]), __uint_as_float(f[3])),
                            pack2(__uint_as_float(f[4]), __uint_as_float(f[5])), pack2(__uint_as_float(f[6]), __uint_as_float(f[7])));
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<2>();
            if (t == 0) mbar_arrive_local(bars + B_STG);
        }
    } else if (warp == 8) {
        // ========================================================== chain issuer
        // Off the chain: Q tiles, Q S_r, and the ring: chunk c's prepared data is loaded
        // from its global chunk slot (once the producer has signalled it and ring slot c mod 2
        // is free), and the producer is told as soon as it has landed, so it may reuse the
        // global slot.  Every wait below also advances those two steps.
        if (lane == 0) {
            int q_req = 0, qs_req = 0, full_req0 = 0, full_req1 = 0;   // for draining after an abort
            const uint32_t id_m64 = idesc_bf16(64, 32, false, true);
            const uint64_t d_cq = sdesc_kmajor(smem_u32(sm + S4_CQ)), d_st = sdesc_mn_sw64(smem_u32(sm + S4_ST));
            int next_load = 0;                  // next chunk to load
            int load_limit = 1;                 // highest chunk whose ring slot is free
            int acked = -1;                     // last chunk acknowledged to its producer
            auto poll_ring = [&]() {
                const int a = next_load;
                if (a <= load_limit && a < nch &&
                    mbar_try_wait(bars + B_READY + (a & 7), (uint32_t)((a >> 3) & 1))) {
                    const int sa = a & 1;
                    const unsigned char *src = gring + (size_t)(a & 7) * K4_GCHUNK;
                    unsigned char *dst = sm + S4_RING + sa * K4_RING_BYTES;
                    uint64_t *fb = bars + (sa ? B_FULL1 : B_FULL0);
                    // polled at CTA scope (cheap); the cluster-scope acquire that pairs with
                    // the producer's release is this one fence, taken once the phase is seen
                    fence_release_cluster();
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(fb, K4_RING_BYTES);
                    bulk_load_global(dst, src, 24576, fb);                          // W | P
                    bulk_load_global(dst + 24576, src + 24576 + r * 4096, 4096, fb);  // U~_r
                    if (sa) ++full_req1; else ++full_req0;
                    next_load = a + 1;
                }
                const int k = acked + 1;
                if (k < next_load && mbar_try_wait(bars + ((k & 1) ? B_FULL1 : B_FULL0), (uint32_t)((k >> 1) & 1))) {
                    // the loads this covers have completed, so there is nothing to publish
                    mbar_arrive_remote_relaxed(map_to_rank(bars + B_GFREE0 + ((k >> 2) & 1), (uint32_t)(k & 3)));
                    acked = k;
                }
            };
            auto wait_ring = [&](int b, uint32_t parity) -> bool {
                for (uint32_t i = 0; i < budget; ++i) {
                    if (mbar_try_wait(bars + b, parity)) return true;
                    poll_ring();
                    if (*abort_flag) return false;
                }
                return false;
            };
            if (nch > 0) {
                q_req = 1;
                const int tb = (int)t_begin;
                mbar_arrive_expect_tx(bars + B_CQ, 16384);
                tma_load_3d(sm + S4_CQ, &tm_q, bars + B_CQ, 0, hq, tb);
                tma_load_3d(sm + S4_CQ + 8192, &tm_q, bars + B_CQ, 64, hq, tb);
                mbar_arrive_expect_tx(bars + B_CK, 16384);
                tma_load_3d(sm + S4_CK, &tm_k, bars + B_CK, 0, hq, tb);
                tma_load_3d(sm + S4_CK + 8192, &tm_k, bars + B_CK, 64, hq, tb);
                mbar_arrive_local(bars + B_OFREE0);     // both output buffers start free
                mbar_arrive_local(bars + B_OFREE1);
            }
#pragma unroll 1
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                // chunk c's prepared data has landed (and been acknowledged)
                {
                    bool okf = true;
                    for (uint32_t i = 0; acked < c; ++i) {
                        poll_ring();
                        if (*abort_flag || i >= budget) { okf = false; break; }
                    }
                    if (!okf) { fail(33); break; }
                }
                // Q S_r -> D_QS[s] right behind W S_r in the pipe (both read the same S_r tile)
                if (!wait_ring(B_WSI, c & 1)) { fail(35); break; }
                if (!wait_ring(L2N ? B_CQN : B_CQ, c & 1)) { fail(30); break; }
                if (!wait_ring(s ? B_OFREE1 : B_OFREE0, (c >> 1) & 1)) { fail(32); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16(tmem + T4_QS + 32 * s, d_cq + (ks >> 2) * 512 + (ks & 3) * 2, d_st + ks * 64, id_m64, ks > 0);
                umma_commit(bars + B_QS);
                ++qs_req;
                // Q of the next chunk into the buffer Q S_r has finished reading
                if (!wait_ring(B_QS, c & 1)) { fail(34); break; }
                if (c + 1 < nch) {
                    ++q_req;
                    const int tn = (int)(t_begin + (long long)(c + 1) * K4_C);
                    mbar_arrive_expect_tx(bars + B_CQ, 16384);
                    tma_load_3d(sm + S4_CQ, &tm_q, bars + B_CQ, 0, hq, tn);
                    tma_load_3d(sm + S4_CQ + 8192, &tm_q, bars + B_CQ, 64, hq, tn);
                }
                // ring slot s is free for chunk c + 2 once P U_r (the last MMA reading it) is done
                if (!wait_ring(s ? B_PU1 : B_PU0, (c >> 1) & 1)) { fail(38); break; }
                load_limit = c + 2;
                poll_ring();
            }
            if (*abort_flag) {
                // let this thread's loads land before shared memory goes away
                drain_bar(bars + B_CQ, q_req, false);
                drain_bar(bars + B_QS, qs_req, false);
                drain_bar(bars + B_FULL0, full_req0, false);
                drain_bar(bars + B_FULL1, full_req1, false);
            }
        }
        __syncwarp();
    } else {
        // =========================================================== prep issuer
        if (lane == 0) {
            int in_req = 0, p1_req = 0, wu_req = 0;
            const uint32_t id_p1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_wu = idesc_bf16(64, 128, false, true);
            auto load_inputs = [&](int p) {       // K, Q, V of chunk p into the prep buffers
                const int tp = (int)(t_begin + (long long)p * K4_C);
                ++in_req;
                mbar_arrive_expect_tx(bars + B_PKQ, 32768);
                tma_load_3d(sm + S4_PKQ, &tm_k, bars + B_PKQ, 0, hq, tp);
                tma_load_3d(sm + S4_PKQ + 16384, &tm_k, bars + B_PKQ, 64, hq, tp);
                tma_load_3d(sm + S4_PKQ + 8192, &tm_q, bars + B_PKQ, 0, hq, tp);
                tma_load_3d(sm + S4_PKQ + 24576, &tm_q, bars + B_PKQ, 64, hq, tp);
                mbar_arrive_expect_tx(bars + B_PV, 16384);
                tma_load_3d(sm + S4_PV, &tm_v, bars + B_PV, 0, h, tp);
                tma_load_3d(sm + S4_PV + 8192, &tm_v, bars + B_PV, 64, h, tp);
            };
            // the bulk stores of a production complete while the next one starts: its P1 is
            // issued first, then the stores are waited for, the staging released and the
            // chunk signalled to every CTA
            int pend = -1;                          // chunk whose stores are in flight
            auto finish_stores = [&]() {
                bulk_wait_read_all();
                mbar_arrive_local(bars + B_SFREE);
                bulk_wait_all();
                // the writes are complete: one release, then a signal to every CTA
                fence_proxy_async_global();
                fence_release_cluster();
#pragma unroll 1
                for (uint32_t d = 0; d < 4; ++d) mbar_arrive_remote_relaxed(map_to_rank(bars + B_READY + (pend & 7), d));
                pend = -1;
            };
            if ((int)r < nch) load_inputs((int)r);
#pragma unroll 1
            for (int k = 0;; ++k) {
                const int p = (int)r + 4 * k;
                if (p >= nch) break;
                if (!wait_bar(B_PIN, k & 1, false)) { fail(40); break; }
                tc_fence_after();
                {   // P1: [K;Q] K^T
                    const uint32_t kq = smem_u32(sm + S4_PKQ);
#pragma unroll 1
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t a = kq + (ks >> 2) * 16384 + (ks & 3) * 32;
                        umma_bf16(tmem + T4_KQ, sdesc_kmajor(a), sdesc_kmajor(a), id_p1, ks > 0);
                    }
                    umma_commit(bars + B_P1);
                    ++p1_req;
                }
                if (pend >= 0) finish_stores();
                if (!wait_bar(B_TT, k & 1, false)) { fail(41); break; }
                tc_fence_after();
                {   // W = T' K ; U~ = T'' V   (M = 64, N = 128)
                    const uint32_t kq = smem_u32(sm + S4_PKQ), pv = smem_u32(sm + S4_PV);
                    const uint32_t tpa = smem_u32(sm + S4_TP), tppa = smem_u32(sm + S4_TPP);
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + T4_W, sdesc_kmajor(tpa + ks * 32), sdesc_mnmajor(kq + ks * 2048, 16384), id_wu, ks > 0);
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + T4_U, sdesc_kmajor(tppa + ks * 32), sdesc_mnmajor(pv + ks * 2048, 8192), id_wu, ks > 0);
                    umma_commit(bars + B_WU);
                    ++wu_req;
                }
                if (!wait_bar(B_WU, k & 1, false)) { fail(42); break; }
                if (p + 4 < nch) load_inputs(p + 4);   // the prep buffers are free again
                // staging -> this production's global chunk slot (p mod 8), last used two
                // productions ago: every CTA must have loaded that one first
                if (!wait_bar(B_STG, k & 1, false)) { fail(43); break; }
                if (k >= 2 && !wait_bar(B_GFREE0 + (k & 1), ((k - 2) >> 1) & 1, true)) { fail(44); break; }
                unsigned char *gchunk = gring + (size_t)(p & 7) * K4_GCHUNK;
                bulk_store_global(gchunk, sm + S4_WSTG, 16384);
                bulk_store_global(gchunk + 16384, sm + S4_PSTG, 8192);
                bulk_store_global(gchunk + 24576, sm + S4_USTG, 16384);
                bulk_commit();
                pend = p;
            }
            if (pend >= 0 && !*abort_flag) finish_stores();
            bulk_wait_all();
            if (*abort_flag) {
                drain_bar(bars + B_PKQ, in_req, false);
                drain_bar(bars + B_PV, in_req, false);
                drain_bar(bars + B_P1, p1_req, false);
                drain_bar(bars + B_WU, wu_req, false);
            }
        }
        __syncwarp();
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 8) tmem_dealloc(tmem, 512);
    if (r == 0 && tid == 256 && ring_slot >= 0) {
        __threadfence();
        atomicExch(&g4_pool[ring_slot], 0);
    }
}

// ------------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encoder4() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_map4(CUtensorMap *map, const void *base, long long T_total, int H) {
    auto enc = encoder4();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T_total};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct ClusterDeviceState {
    bool ready = false;
};
constexpr int kMaxDev4 = 128;
std::mutex g_dev4_mutex;
ClusterDeviceState g_dev4[kMaxDev4];

// the 226 KB shared-memory opt-in of both instantiations, once per device
cudaError_t cluster_device_setup() {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev4) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev4_mutex);
    if (!g_dev4[dev].ready) {
        e = cudaFuncSetAttribute(prefill_tc_cluster_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, K4_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_tc_cluster_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, K4_SMEM);
        if (e != cudaSuccess) return e;
        g_dev4[dev].ready = true;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_prefill_tc_cluster(const void *q, const void *k, const void *v, const float *g,
                                      const float *beta, const float *S0, void *out, float *S_final,
                                      const int32_t *cu, int N, long long T_dense, long long T_total,
                                      int H_qk, int H_v, float scale, int opts, DeviceError *err,
                                      uint32_t budget, cudaStream_t stream)
{
    if (T_total >= (1LL << 31) || (long long)N * 4 > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    if (!make_map4(&mq, q, T_total, H_qk) || !make_map4(&mk, k, T_total, H_qk) ||
        !make_map4(&mv, v, T_total, H_v))
        return cudaErrorInvalidValue;
    const cudaError_t se = cluster_device_setup();
    if (se != cudaSuccess) return se;
    dim3 grid((unsigned)(4 * N), (unsigned)H_v);
    auto kern = (opts & kOptL2Norm) ? prefill_tc_cluster_kernel<true> : prefill_tc_cluster_kernel<false>;
    kern<<<grid, K4_THREADS, K4_SMEM, stream>>>(
        mq, mk, mv, g, beta, S0, (__nv_bfloat16 *)out, S_final, cu, T_dense, H_qk, H_v, scale,
        opts, err, budget);
    return cudaGetLastError();
}

}  // namespace gdn
