// Chunked prefill of the gated delta rule, dk = dv = 128, bf16 I/O, one sm_100a CTA per
// (unit, value head), where a unit is a whole sequence or one segment of it.
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
// The state chain runs transposed: S^T (value column v in TMEM lane v, key index d in
// column d) stays in TMEM for the whole unit, and every chain product has the 128 value
// columns as its M dimension, so one CTA carries a whole head at full MMA width:
//   C1  (Q~ S)^T = S^T Q~^T, and (W S)^T - U~^T = S^T W^T + (-U~^T), accumulated onto
//       the -U~^T that P3 left in one of two buffers (A = S^T bf16 in TMEM, N = 64 each)
//   E3  U^T = -((W S)^T - U~^T)  -> shared memory (bf16)
//   C2  S^T += U^T K~                               (S^T pre-scaled by gamma_end)
//   C3  O^T = (Q~ S)^T + U^T P^T                     (off the chain, second issuer)
//   E4  S^T -> bf16 copy for the next C1, then S^T *= gamma_end(next)
// The per-chunk quantities that do not depend on S (A, P, the inverse T, W, U~^T, Q~ =
// diag(gamma) Q, K~) are prepared ahead by other warps of the same CTA, three chunks deep:
// a chunk's K, Q and V land in one of three regions as soon as the chain has finished
// with the chunk three back.
//
// Segments.  Within a segment everything is affine in the state S_in entering it: the
// outputs are O = O_local + Psi S_in and the end state S_end = M S_in + B, where O_local
// and B come from the chain started at S_in = 0, and Psi and M from the chain started at
// S_in = I with U~ = 0 (its "outputs" are exactly Psi_c = (diag(gamma) Q_c - P_c W_c)
// Phi_c, Phi_c the transfer from the segment start to chunk c).  So a long sequence runs
// as (see launch_prefill_chain):
//   1. one pass of chains: for every segment the local chain (grid slice z = 1; the first
//      segment starts from S0 and is then exact) and, past the first segment, the
//      transfer chain (slice 0), in parallel;
//   2. scan: S_in(p + 1) = M_p S_in(p) + B_p over the segments, and S_final;
//   3. correction: out += Psi S_in(p) for the tokens of every segment p >= 1, a streamed
//      tensor-core product.
//
// Roles (448 threads):
//   warps 0-3    chain group: E3 and E4; thread 0 issues C1 and C2, thread 32 issues C3
//   warps 4-7    prep group: A/P epilogue, triangular inverse (in place), T' and -T''
//   warps 8-11   output group: W rows from W^T and Q~ in place (the chunk is then ready for
//                C1), O^T -> out for the chunk before, then K~ in place (for C2)
//   warp 12      prep issuer: MMAs P1 ([K;Q] K^T) of the next chunk and P2 (W^T = K^T T'^T),
//                P3 (-U~^T = V^T (-T'')^T, into the -U buffer of the chunk's parity) of this
//                one, in whichever order their inputs arrive
//   warp 13      loader: TMA of K, Q, V; per-chunk vectors (g, beta -> G, gamma, ...)
// Every wait is bounded: a role whose wait runs out records GDN_ERR_TIMEOUT, raises the
// CTA's abort flag so the other roles stop at their next wait, and the CTA drains its
// own copies and MMAs before it frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "tri_inverse.cuh"

namespace gdn {
using namespace sm100;

namespace {

constexpr int CC = 64;                   // chunk
constexpr int DD = 128;                  // dk = dv
constexpr int CH_THREADS = 448;
constexpr int NREG = 3;                  // chunks in flight (regions)
constexpr uint32_t kDrainBudget = GDN_DEFAULT_WAIT_BUDGET;   // waits after an abort
constexpr uint32_t kPollNs = 2000;      // longest hardware suspension of one poll

// TMEM columns (512 allocated)
constexpr uint32_t TM_S = 0;        // 128: S^T fp32 (lane v, column d), pre-scaled by gamma_end
constexpr uint32_t TM_QW = 128;     // 64:  O^T = (Q~ S + P U)^T, lane v, column token
constexpr uint32_t TM_WU0 = 192;    // 2 x 64: -U^T = (W S)^T - U~^T of chunks of parity 0, 1
constexpr uint32_t TM_WU1 = 256;    //   (P3 writes -U~^T, C1 adds (W S)^T; lane v, column token)
constexpr uint32_t TM_SB = 320;     // 64:  S^T bf16 pairs (A operand of C1)
constexpr uint32_t TM_KQ = 384;     // 64:  [K;Q] K^T (lanes 0-63 K K^T, 64-127 Q K^T)
constexpr uint32_t TM_WT = 448;     // 64:  W^T fp32 (lane d, column token)

// shared memory (offsets from a 1024-aligned base); every MMA tile is 1024-aligned.
// A chunk region holds, per 64-wide K block kb (at kb * SR_KB): K rows (8 KB), Q rows
// (8 KB), and V rows that W rows replace once P3 has read them (8 KB), each 64 rows of
// 128 B in the 128-byte swizzle.  So [K;Q] and [Q~;W] are contiguous 128-row K-major
// operands, and K, K~ and V are MN-major operands (their 64-element blocks SR_KB apart).
constexpr uint32_t SR_KB = 24576;
constexpr uint32_t SR_Q = 8192, SR_W = 16384;
constexpr uint32_t SR_BYTES = 2 * SR_KB;
constexpr uint32_t S_REG = 0;                        // NREG regions of 48 KB
constexpr uint32_t S_P = S_REG + NREG * SR_BYTES;    // NREG x 8 KB P (K-major rows i)
constexpr uint32_t S_U = S_P + NREG * 8192;          // 16 KB U^T bf16 (K-major rows v, 64 tokens)
constexpr uint32_t S_TT = S_U + 16384;               // 16 KB T' | T'' (bf16, K-major rows i)
constexpr uint32_t S_M = S_TT + 16384;               // fp32 A, then T, 64 rows of TP floats
constexpr int TP = 72;                               // fp32 row pitch (conflict-free fragments)
constexpr uint32_t S_VEC = S_M + 64 * TP * 4;        // NREG buffers x 6 vectors x 64 fp32
constexpr int VEC_FLOATS = 6 * 64;
constexpr uint32_t S_BAR = S_VEC + NREG * VEC_FLOATS * 4;
constexpr uint32_t S_MISC = S_BAR + 48 * 8;          // tmem base, abort flag
constexpr uint32_t S_END = S_MISC + 16;
constexpr uint32_t CH_SMEM = S_END + 1024;
static_assert(CH_SMEM <= 232448, "shared memory");
// vector slots inside one buffer (64 floats each)
constexpr int V_BETA = 0, V_G = 64, V_GAM = 128, V_INV = 192, V_DTE = 256, V_BG = 320;

enum Bar {
    B_LD0 = 0, B_LD1, B_LD2,           // loader: K (Q, V) of the region's chunk landed
    B_VEC0, B_VEC1, B_VEC2,            // loader: vectors of the buffer's chunk
    B_IN,                              // prep: inputs normalised (q/k L2 norm only)
    B_P1, B_KQF, B_TT, B_P2, B_WTF,
    B_P30, B_P31,                      // P3 of chunks of parity 0, 1
    B_UF0, B_UF1,                      // chain: -U^T buffer of parity 0, 1 read
    B_RDY0, B_RDY1, B_RDY2,            // output group: chunk ready for the chain
    B_C1, B_C2, B_C3, B_OF,
    B_RF0, B_RF1, B_RF2,               // commit: region free (after C2)
    B_PF0, B_PF1, B_PF2,               // commit: P tile free (after C3)
    B_VF0, B_VF1, B_VF2,               // chain: vector buffer free
    B_KS0, B_KS1, B_KS2,               // output group: K~ of the region's chunk scaled (C2 may read)
    B_DRAIN0, B_DRAIN1, B_DRAIN2,
    B_COUNT
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
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// parity of the k-th completion (k = 0, 1, ...) of a barrier
__device__ __forceinline__ uint32_t par(int k) { return (uint32_t)(k & 1); }
// every element of a 128-byte row of bf16 scaled by f, in place; the 16-byte pieces are
// taken in swizzled order, so the rows of a warp's threads touch different banks
__device__ __noinline__ void scale_row128(unsigned char *row, int r, float f) {
#pragma unroll 2
    for (int cc = 0; cc < 8; ++cc) {
        unsigned char *pp = row + (((cc ^ r) & 7) << 4);
        uint4 w = *reinterpret_cast<const uint4 *>(pp);
        uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) { const float2 x = unpack2(wv[e]); wv[e] = pack2(x.x * f, x.y * f); }
        *reinterpret_cast<uint4 *>(pp) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

// The gate prologue of one loader lane's two tokens: (log-decay g0, g1, strength b0, b1);
// a token past the unit contributes nothing.  Out of line: one copy of the gate code.
__device__ __noinline__ float4 gate_pair(float g0, float g1, float b0, float b1, bool in0, bool in1,
                                         int opts) {
    return make_float4(in0 ? gate_log_decay(g0, opts) : 0.f, in1 ? gate_log_decay(g1, opts) : 0.f,
                       in0 ? gate_strength(b0, opts) : 0.f, in1 ? gate_strength(b1, opts) : 0.f);
}

}  // namespace

// Launch parameters (one copy per launch, in the constant bank).
struct ChainParams {
    const float *g, *beta;
    const float *S0;            // initial states [N, H_v, dk, dv] (null: zero)
    float *S_final;             // final states [N, H_v, dk, dv] (null: not written)
    __nv_bfloat16 *out;
    const int32_t *cu_seqlens;  // null: dense [N, T_dense]
    const int4 *units;          // null: computed (see unit_of)
    float *ws_M, *ws_B, *ws_S;  // per unit: transfer M, local end state B, start state S_in
    __nv_bfloat16 *ws_Psi;      // transfer-chain outputs Psi, [T_total, H_v, dk]
    long long T_dense;
    int N, H_qk, H_v;
    int seg_tokens;             // 0: one unit per sequence; else tokens per segment
    int units_per_seq;          // dense, segmented: segments per sequence
    float scale;
    int opts;
    DeviceError *err;
    uint32_t budget;
};

// The unit of CTA column x: sequence n, tokens [tb, te), segment p of P.
struct Unit {
    int n, p, P;
    long long tb, te;
};
__device__ __forceinline__ bool unit_of(const ChainParams &prm, int x, Unit &u)
{
    if (prm.units) {
        const int4 e = prm.units[x];
        if (e.x < 0) return false;
        u.n = e.x; u.tb = e.y; u.te = e.z; u.p = e.w & 0xffff; u.P = e.w >> 16;
        return true;
    }
    if (prm.seg_tokens == 0) {
        if (x >= prm.N) return false;
        u.n = x; u.p = 0; u.P = 1;
        if (prm.cu_seqlens) { u.tb = prm.cu_seqlens[x]; u.te = prm.cu_seqlens[x + 1]; }
        else { u.tb = (long long)x * prm.T_dense; u.te = u.tb + prm.T_dense; }
        return true;
    }
    // dense, segmented
    const int P = prm.units_per_seq;
    if (x >= prm.N * P) return false;
    u.n = x / P; u.p = x % P; u.P = P;
    const long long s0 = (long long)u.n * prm.T_dense;
    u.tb = s0 + (long long)u.p * prm.seg_tokens;
    u.te = min(u.tb + (long long)prm.seg_tokens, s0 + prm.T_dense);
    return true;
}

// Bounded wait on barrier b of `bars` for the given phase parity: at most `budget` polls
// of up to kPollNs each; gives up early once another role of this CTA has aborted.  Out
// of line: it is called from some thirty places, and the kernel's roles run different code
// at once, so every copy of the loop would compete for the instruction cache.
__device__ __noinline__ bool bounded_wait(uint64_t *bars, int b, uint32_t parity, uint32_t budget,
                                          const volatile int *abort_flag)
{
    uint64_t *bar = bars + b;
    for (uint32_t i = 0; i < budget; ++i) {
        if (mbar_try_wait_sleep(bar, parity, kPollNs)) return true;
        if (*abort_flag) return false;
    }
    return false;
}

__device__ __noinline__ void chain_abort(volatile int *abort_flag, DeviceError *err, int where)
{
    if (!*abort_flag) {
        *abort_flag = 1;
        record_error(err, GDN_ERR_TIMEOUT, where);
    }
}

template <bool L2N, bool SEG>
__global__ void __launch_bounds__(CH_THREADS, 1)
prefill_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ ChainParams prm)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // segmented: slice z = 0 runs the transfer chain (S_in = I, U~ = 0, no V; its outputs
    // are Psi, its final state M), slice 1 the local chain (S_in = S0 for the first
    // segment, else 0; final state B)
    constexpr bool seg = SEG;
    const bool xa = SEG && blockIdx.z == 0;
    const int h = blockIdx.y;
    Unit un;
    if (!unit_of(prm, blockIdx.x, un)) return;
    if (xa && un.p == 0) return;                   // the first segment starts from S0: no transfer
    const int hq = h / (prm.H_v / prm.H_qk);
    const int nch = (int)((un.te - un.tb + CC - 1) / CC);
    const size_t st_n = ((size_t)un.n * prm.H_v + h) * DD * DD;          // [N, H_v] slot
    const size_t st_u = ((size_t)blockIdx.x * prm.H_v + h) * DD * DD;    // [unit, H_v] slot

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + S_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + S_MISC + 4);

    if (warp == 12) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
    if (tid == 0) {
        for (int b = 0; b < B_COUNT; ++b) mbar_init(bars + b, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t budget = prm.budget;

    auto wait_bar = [&](int b, uint32_t parity) -> bool {
        return bounded_wait(bars, b, parity, budget, abort_flag);
    };
    auto fail = [&](int where) { chain_abort(abort_flag, prm.err, where); };
    auto region = [&](int c) -> unsigned char * { return sm + S_REG + (c % NREG) * SR_BYTES; };
    auto vecbuf = [&](int c) -> float * { return reinterpret_cast<float *>(sm + S_VEC) + (c % NREG) * VEC_FLOATS; };
    auto rbar = [&](int base, int c) -> int { return base + c % NREG; };   // per-region barrier
    auto rpar = [&](int c) -> uint32_t { return par(c / NREG); };        // its parity for chunk c

    if (warp < 4) {
        // =============================================================== chain group
        const int t = tid, v = tid, q = warp;
        const uint32_t loff = (uint32_t)(32 * q) << 16;
        const uint32_t id_c1 = idesc_bf16(128, 64, false, false);
        const uint32_t id_c2 = idesc_bf16(128, 128, false, true);
        const uint32_t id_c3 = idesc_bf16(128, 64, false, false);
        const uint32_t su = smem_u32(sm + S_U);
        bool ok = true;
        int mma_issued = 0;

        auto issue_c1 = [&](int c) {           // thread 0
            const uint32_t rq = smem_u32(region(c)) + SR_Q, rw = smem_u32(region(c)) + SR_W;
            const uint32_t wu = tmem + ((c & 1) ? TM_WU1 : TM_WU0);
#pragma unroll 1
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ko = (ks >> 2) * SR_KB + (ks & 3) * 32;
                // (W S)^T onto P3's -U~^T (the transfer chain has U~ = 0: a fresh sum)
                umma_bf16_ta(wu, tmem + TM_SB + 8 * ks, sdesc_kmajor(rw + ko), id_c1, !xa || ks > 0);
                umma_bf16_ta(tmem + TM_QW, tmem + TM_SB + 8 * ks, sdesc_kmajor(rq + ko), id_c1, ks > 0);
            }
            umma_commit(bars + B_C1);
            ++mma_issued;
        };

        // ---- initial state: S^T (fp32, scaled by gamma_end(0)) and its bf16 copy
        const float *src = nullptr;
        if (!xa && un.p == 0 && prm.S0) src = prm.S0 + st_n;
        float *dst = seg ? (xa ? prm.ws_M : prm.ws_B) + st_u : (prm.S_final ? prm.S_final + st_n : nullptr);
        if (nch == 0) {
            // no token: the final state is the initial one
            if (dst)
                for (int d = 0; d < DD; ++d)
                    dst[(size_t)d * DD + v] = src ? src[(size_t)d * DD + v] : (xa && d == v ? 1.f : 0.f);
            ok = false;
        } else if (!group_all<1>(t != 0 || wait_bar(B_VEC0, 0))) {
            fail(1);
            ok = false;
        } else {
            const float ge0 = vecbuf(0)[V_GAM + 63];
#pragma unroll 1
            for (int db = 0; db < 4; ++db) {
                uint32_t xs[32], xb[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const int d = 32 * db + j;
                    const float x0 = src ? src[(size_t)d * DD + v] : (xa && d == v ? 1.f : 0.f);
                    const float x1 = src ? src[(size_t)(d + 1) * DD + v] : (xa && d + 1 == v ? 1.f : 0.f);
                    xs[j] = __float_as_uint(ge0 * x0);
                    xs[j + 1] = __float_as_uint(ge0 * x1);
                    xb[j >> 1] = pack2(x0, x1);       // the bf16 copy holds the unscaled state
                }
                tmem_st32(tmem + loff + TM_S + 32 * db, xs);
                tmem_st16(tmem + loff + TM_SB + 16 * db, xb);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync<1>();
            bool okw = true;
            if (t == 0) {
                okw = wait_bar(B_RDY0, 0);
                if (okw) { tc_fence_after(); issue_c1(0); }
            }
            if (!group_all<1>(okw)) { fail(2); ok = false; }
        }

#pragma unroll 1
        for (int c = 0; ok && c < nch; ++c) {
            // ---- E3: U^T = -((W S)^T - U~^T)  ->  U^T (bf16, K-major rows v).  C1 was
            // issued after RDY(c), which the output group raised only once P3(c) was done.
            if (!group_all<1>(t != 0 || wait_bar(B_C1, par(c)))) {
                fail(3);
                break;
            }
            tc_fence_after();
            const uint32_t wu = (c & 1) ? TM_WU1 : TM_WU0;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t nu[32];
                tmem_ld32(tmem + loff + wu + 32 * h2, nu);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t pu[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * k + 2 * e;
                        pu[e] = pack2(-__uint_as_float(nu[j]), -__uint_as_float(nu[j + 1]));
                    }
                    *reinterpret_cast<uint4 *>(sm + S_U + sw128(v, 4 * h2 + k)) = make_uint4(pu[0], pu[1], pu[2], pu[3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<1>();
            if (t == 0) {
                if (!xa) mbar_arrive_local(bars + B_UF0 + (c & 1));
                mbar_arrive_local(bars + rbar(B_VF0, c));
                // ---- C2: S^T += U^T K~, once the output group has scaled K~
                if (!wait_bar(rbar(B_KS0, c), rpar(c))) {
                    fail(7);
                } else {
                    tc_fence_after();
                    const uint32_t kreg = smem_u32(region(c));
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + TM_S, sdesc_kmajor(su + ks * 32),
                                  sdesc_mnmajor(kreg + ks * 2048, SR_KB), id_c2, 1);
                    umma_commit(bars + B_C2);
                    umma_commit(bars + rbar(B_RF0, c));
                    ++mma_issued;
                }
            } else if (t == 32) {
                // ---- C3: O^T += U^T P^T, issued beside C2 (off the chain)
                tc_fence_after();
                const uint32_t pt = smem_u32(sm + S_P + (c % NREG) * 8192);
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + TM_QW, sdesc_kmajor(su + ks * 32), sdesc_kmajor(pt + ks * 32), id_c3, 1);
                umma_commit(bars + B_C3);
                umma_commit(bars + rbar(B_PF0, c));
                ++mma_issued;
            }
            // ---- E4: the updated state
            const bool last = c + 1 == nch;
            if (!group_all<1>(t != 0 || (wait_bar(B_C2, par(c)) &&
                                         (last || wait_bar(rbar(B_VEC0, c + 1), rpar(c + 1)))))) {
                fail(4);
                break;
            }
            tc_fence_after();
            if (last) {
                if (dst) {
#pragma unroll 1
                    for (int db = 0; db < 4; ++db) {
                        uint32_t xs[32];
                        tmem_ld32(tmem + loff + TM_S + 32 * db, xs);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) dst[(size_t)(32 * db + j) * DD + v] = __uint_as_float(xs[j]);
                    }
                }
                break;
            }
            // bf16 copy first (the next C1 waits for it), then the pre-scaling
#pragma unroll 1
            for (int db = 0; db < 4; ++db) {
                uint32_t xs[32], xb[16];
                tmem_ld32(tmem + loff + TM_S + 32 * db, xs);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) xb[j] = pack2(__uint_as_float(xs[2 * j]), __uint_as_float(xs[2 * j + 1]));
                tmem_st16(tmem + loff + TM_SB + 16 * db, xb);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync<1>();
            bool okw = true;
            if (t == 0) {
                okw = wait_bar(rbar(B_RDY0, c + 1), rpar(c + 1)) && wait_bar(B_OF, par(c));
                if (okw) { tc_fence_after(); issue_c1(c + 1); }
            }
            const float ge = vecbuf(c + 1)[V_GAM + 63];
#pragma unroll 1
            for (int db = 0; db < 4; ++db) {
                uint32_t xs[32];
                tmem_ld32(tmem + loff + TM_S + 32 * db, xs);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) xs[j] = __float_as_uint(ge * __uint_as_float(xs[j]));
                tmem_st32(tmem + loff + TM_S + 32 * db, xs);
            }
            tmem_wait_st();
            tc_fence_before();
            if (!group_all<1>(okw)) { fail(5); break; }
        }
        if (*abort_flag && (t == 0 || t == 32) && mma_issued > 0) {
            uint64_t *db = bars + (t == 0 ? B_DRAIN0 : B_DRAIN2);
            umma_commit(db);
            mbar_wait(db, 0, kDrainBudget);
        }
    } else if (warp < 8) {
        // ================================================================ prep group
        const int t = tid - 128, q = warp - 4, l = lane;
        const int row = 32 * q + l;                       // TMEM lane
        const uint32_t loff = (uint32_t)(32 * q) << 16;
        float *Mf = reinterpret_cast<float *>(sm + S_M);
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            unsigned char *rg = region(c);
            const float *vb = vecbuf(c);
            if constexpr (L2N) {
                // q/k normalisation before P1 reads the tiles; thread t: row t & 63 of K
                // (t < 64) or Q
                if (!group_all<2>(t != 0 || wait_bar(rbar(B_LD0, c), rpar(c)))) { fail(10); break; }
                {
                    const int r = t & 63;
                    unsigned char *r0 = rg + (t >= 64 ? SR_Q : 0) + r * 128;
                    float ss = 0.f;
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) {
                            const uint4 w = *reinterpret_cast<const uint4 *>(r0 + kb * SR_KB + (((cc ^ r) & 7) << 4));
                            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) { const float2 f = unpack2(wv[e]); ss += f.x * f.x + f.y * f.y; }
                        }
                    const float rn = rsqrtf(ss + 1e-6f);
                    scale_row128(r0, r, rn);
                    scale_row128(r0 + SR_KB, r, rn);
                }
                fence_proxy_async();
                group_sync<2>();
                if (t == 0) mbar_arrive_local(bars + B_IN);
            }

            // ---- A (fp32, rows 0..63) and P (bf16, rows 64..127) from [K;Q] K^T.  The P
            // tile of this region was last read by C3(c - NREG).
            if (!group_all<2>(t != 0 || (wait_bar(rbar(B_VEC0, c), rpar(c)) && wait_bar(B_P1, par(c)) &&
                                         (c < NREG || wait_bar(rbar(B_PF0, c), rpar(c - NREG)))))) {
                fail(11);
                break;
            }
            tc_fence_after();
            {
                const bool is_a = q < 2;
                const int i = is_a ? row : row - 64;
                const float Gi = vb[V_G + i], wi = is_a ? vb[V_BETA + i] : 1.f;
                // exp(G_i - G_j) = gamma_i exp(-G_j) is exact enough and in range while the
                // chunk's total log-decay stays above -80 (uniform across the CTA); otherwise
                // each factor comes from the clamped difference
                const bool factored = vb[V_G + 63] > -80.f;
                const float wi_e = wi * vb[V_GAM + i];
                const float we = factored ? wi_e : wi;        // row factor
                const int iend = is_a ? i : i + 1;            // kept columns j < iend
                const int jend = 32 * ((q & 1) + 1);      // columns from here on are masked for the warp
                unsigned char *pt = sm + S_P + (c % NREG) * 8192;
                const float *fsrc = vb + (factored ? V_INV : V_G);
                {
#pragma unroll 1
                    for (int jh = 0; jh < 64; jh += 16) {
                        if (is_a && jh >= jend) break;    // the inverse never reads A above the diagonal
                        float xv[16];
                        if (jh >= jend) {
#pragma unroll
                            for (int u = 0; u < 16; ++u) xv[u] = 0.f;
                        } else {
                            uint32_t kr[16];
                            tmem_ld16(tmem + loff + TM_KQ + jh, kr);
                            tmem_wait_ld();
#pragma unroll
                            for (int u = 0; u < 16; u += 4) {
                                const float4 f4 = *reinterpret_cast<const float4 *>(fsrc + jh + u);
                                const float fj[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const int j = jh + u + e2;
                                    const float keep = (j < iend) ? 1.f : 0.f;
                                    const float e = factored ? fj[e2] : __expf(fminf(Gi - fj[e2], 0.f));
                                    xv[u + e2] = (we * keep) * e * __uint_as_float(kr[u + e2]);
                                }
                            }
                        }
                        if (is_a) {
#pragma unroll
                            for (int u = 0; u < 16; u += 4)
                                *reinterpret_cast<float4 *>(Mf + i * TP + jh + u) = make_float4(xv[u], xv[u + 1], xv[u + 2], xv[u + 3]);
                        } else {
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2)
                                *reinterpret_cast<uint4 *>(pt + sw128(i, (jh >> 3) + h2)) = make_uint4(
                                    pack2(xv[8 * h2 + 0], xv[8 * h2 + 1]), pack2(xv[8 * h2 + 2], xv[8 * h2 + 3]),
                                    pack2(xv[8 * h2 + 4], xv[8 * h2 + 5]), pack2(xv[8 * h2 + 6], xv[8 * h2 + 7]));
                        }
                    }
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<2>();
            if (t == 0) mbar_arrive_local(bars + B_KQF);
            // ---- T = (I + A)^-1, in place
            invert_unit_lower_64_inplace_wg<TP>(Mf, t, [] { group_sync<2>(); });
            // ---- T' = T diag(beta gamma), -T'' = -T diag(beta) (bf16, K-major rows i), once
            // the previous chunk's P2 and P3 have read the last ones
            if (!group_all<2>(t != 0 || c == 0 || (wait_bar(B_P2, par(c - 1)) && (xa || wait_bar(B_P30 + ((c - 1) & 1), par((c - 1) >> 1)))))) {
                fail(12);
                break;
            }
            {
                const int i = t >> 1, half = t & 1;           // row i, columns [32 half, +32)
                const float *trow = Mf + i * TP + 32 * half;
                unsigned char *tp1 = sm + S_TT, *tp2 = sm + S_TT + 8192;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    const int j0 = 32 * half + 8 * cc;
                    uint4 o1 = make_uint4(0u, 0u, 0u, 0u), o2 = o1;
                    if (j0 <= i) {                            // T is lower triangular
                        const float4 t0 = *reinterpret_cast<const float4 *>(trow + 8 * cc);
                        const float4 t1 = *reinterpret_cast<const float4 *>(trow + 8 * cc + 4);
                        const float4 b0 = *reinterpret_cast<const float4 *>(vb + V_BETA + j0);
                        const float4 b1 = *reinterpret_cast<const float4 *>(vb + V_BETA + j0 + 4);
                        const float4 g0 = *reinterpret_cast<const float4 *>(vb + V_BG + j0);
                        const float4 g1 = *reinterpret_cast<const float4 *>(vb + V_BG + j0 + 4);
                        const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                        float w1[8], w2[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float tt = (j0 + e <= i) ? tv[e] : 0.f;
                            w1[e] = tt * gv[e];
                            w2[e] = -tt * bv[e];
                        }
                        o1 = make_uint4(pack2(w1[0], w1[1]), pack2(w1[2], w1[3]), pack2(w1[4], w1[5]), pack2(w1[6], w1[7]));
                        o2 = make_uint4(pack2(w2[0], w2[1]), pack2(w2[2], w2[3]), pack2(w2[4], w2[5]), pack2(w2[6], w2[7]));
                    }
                    *reinterpret_cast<uint4 *>(tp1 + sw128(i, 4 * half + cc)) = o1;
                    *reinterpret_cast<uint4 *>(tp2 + sw128(i, 4 * half + cc)) = o2;
                }
            }
            fence_proxy_async();
            tc_fence_before();
            group_sync<2>();
            if (t == 0) mbar_arrive_local(bars + B_TT);
        }
    } else if (warp < 12) {
        // ============================================================== output group
        // Iteration c finishes chunk c's preparation (W rows from W^T, Q~ = diag(gamma) Q
        // and K~ = diag(dte) K in place) and then writes the outputs of chunk c - 1.
        const int t = tid - 256, v = t, q = warp - 8, l = lane;
        const uint32_t loff = (uint32_t)(32 * q) << 16;
        const bool odd = l & 1;
        const float scale = prm.scale;
        // outputs of chunk c: O^T (lane v) is read out of TMEM and the accumulator handed
        // back to the chain first; the rows are written after that
        auto outputs = [&](int c) -> bool {
            if (!group_all<3>(t != 0 || wait_bar(B_C3, par(c)))) return false;
            tc_fence_after();
            // o_i[v] for the 64 tokens, rounded to bf16 in pairs of tokens (low half = even i)
            uint32_t pk[32];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t x[32];
                tmem_ld32(tmem + loff + TM_QW + 32 * h2, x);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    pk[16 * h2 + m] = pack2(scale * __uint_as_float(x[2 * m]), scale * __uint_as_float(x[2 * m + 1]));
            }
            tc_fence_before();
            group_sync<3>();
            if (t == 0) mbar_arrive_local(bars + B_OF);
            const long long t0 = un.tb + (long long)c * CC;
            const int L = (int)min((long long)CC, un.te - t0);
            // lanes (v, v ^ 1) pair up: the even lane writes token 2m's two values, the odd
            // lane token 2m + 1's
            __nv_bfloat16 *obase = (xa ? prm.ws_Psi : prm.out) + ((size_t)t0 * prm.H_v + h) * DD + (v & ~1);
            const size_t rstride = (size_t)prm.H_v * DD;
#pragma unroll
            for (int m = 0; m < 32; ++m) {
                const uint32_t w = pk[m];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, odd ? (w & 0xffffu) : (w >> 16), 1);
                const int r = 2 * m + (odd ? 1 : 0);
                const uint32_t val = odd ? ((recv & 0xffffu) | (w & 0xffff0000u)) : ((w & 0xffffu) | (recv << 16));
                if (r < L) *reinterpret_cast<uint32_t *>(obase + (size_t)r * rstride) = val;
            }
            return true;
        };
#pragma unroll 1
        for (int c = 0; c <= nch; ++c) {
            if (c < nch) {
                unsigned char *rg = region(c);
                const float *vb = vecbuf(c);
                // ---- W^T (lane d) -> W rows (K-major, token i) over V in the region's W slots
                // (P3 has read V); P2 and P3 follow P1, so Q and K are free to scale
                if (!group_all<3>(t != 0 || (wait_bar(B_P2, par(c)) && (xa || wait_bar(B_P30 + (c & 1), par(c >> 1)))))) { fail(20); break; }
                tc_fence_after();
                {
                    const int d = v, kb = d >> 6, dc = d & 63;
                    const uint32_t wbase = smem_u32(rg + kb * SR_KB + SR_W);
                    const uint32_t bofs = (uint32_t)((dc & 7) * 2) - (odd ? 2u : 0u);
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t x[32];
                        tmem_ld32(tmem + loff + TM_WT + 32 * h2, x);
                        tmem_wait_ld();
#pragma unroll
                        for (int ii = 0; ii < 32; ii += 2) {
                            const float send = __uint_as_float(odd ? x[ii] : x[ii + 1]);
                            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                            const int r = 32 * h2 + ii + (odd ? 1 : 0);
                            const uint32_t val = odd ? pack2(recv, __uint_as_float(x[ii + 1]))
                                                     : pack2(__uint_as_float(x[ii]), recv);
                            st_shared_u32(wbase + sw128(r, dc >> 3) + bofs, val);
                        }
                    }
                }
                tc_fence_before();
                // ---- Q~ = diag(gamma) Q, rows in place: with W, what C1 reads
                const int r = t & 63, kb = t >> 6;
                scale_row128(rg + kb * SR_KB + SR_Q + r * 128, r, vb[V_GAM + r]);
                fence_proxy_async();
                group_sync<3>();
                if (t == 0) {
                    mbar_arrive_local(bars + B_WTF);
                    mbar_arrive_local(bars + rbar(B_RDY0, c));
                }
            }
            // the outputs of chunk c - 1 (the chain's next C1 waits for their read-out) ...
            if (c >= 1 && !outputs(c - 1)) { fail(21); break; }
            // ... then K~ = diag(dte) K in place, which only C2(c) reads, after C1 and E3
            if (c < nch) {
                const int r = t & 63, kb = t >> 6;
                scale_row128(region(c) + kb * SR_KB + r * 128, r, vecbuf(c)[V_DTE + r]);
                fence_proxy_async();
                group_sync<3>();
                if (t == 0) mbar_arrive_local(bars + rbar(B_KS0, c));
            }
        }
    } else if (warp == 12) {
        // =============================================================== prep issuer
        if (lane == 0) {
            const uint32_t id_p1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_p23 = idesc_bf16(128, 64, true, false);
            const uint32_t tpa = smem_u32(sm + S_TT);
            int issued = 0;
            // P1 of chunk c: [K;Q] K^T once the tiles have landed (and been normalised) and
            // the accumulator has been read for chunk c - 1
            auto issue_p1 = [&](int c) -> bool {
                if (!(L2N ? wait_bar(B_IN, par(c)) : wait_bar(rbar(B_LD0, c), rpar(c))) ||
                    (c > 0 && !wait_bar(B_KQF, par(c - 1))))
                    return false;
                tc_fence_after();
                const uint32_t rg = smem_u32(region(c));
#pragma unroll 1
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t a = rg + (ks >> 2) * SR_KB + (ks & 3) * 32;
                    umma_bf16(tmem + TM_KQ, sdesc_kmajor(a), sdesc_kmajor(a), id_p1, ks > 0);
                }
                umma_commit(bars + B_P1);
                ++issued;
                return true;
            };
            // P2 (W^T = K^T T'^T) and P3 (-U~^T = V^T (-T'')^T, V in the W slots, into the
            // -U^T buffer of the chunk's parity once C2 and C3 of chunk c - 2 have read the
            // U^T left there; the transfer chain has U~ = 0 and no P3)
            auto issue_p23 = [&](int c) -> bool {
                const uint32_t rg = smem_u32(region(c));
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + TM_WT, sdesc_mnmajor(rg + ks * 2048, SR_KB), sdesc_kmajor(tpa + ks * 32),
                              id_p23, ks > 0);
                umma_commit(bars + B_P2);
                if (!xa) {
                    if (c > 1 && !wait_bar(B_UF0 + (c & 1), par((c >> 1) - 1))) return false;
                    tc_fence_after();
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + ((c & 1) ? TM_WU1 : TM_WU0), sdesc_mnmajor(rg + SR_W + ks * 2048, SR_KB),
                                  sdesc_kmajor(tpa + 8192 + ks * 32), id_p23, ks > 0);
                    umma_commit(bars + B_P30 + (c & 1));
                }
                return true;
            };
            if (nch > 0 && !issue_p1(0)) fail(30);
            // Chunk c: P1 of chunk c + 1 (its tiles landed, the accumulator read for chunk c)
            // and P2, P3 of chunk c (T' of chunk c formed, W^T of chunk c - 1 read), in
            // whichever order their inputs arrive: a region that the chain frees late then
            // holds back P1 only, not this chunk's W and U~.  Polled with short naps, at most
            // `budget` polls per chunk.
#pragma unroll 1
            for (int c = 0; c < nch && !*abort_flag; ++c) {
                bool need_p1 = c + 1 < nch, need_p23 = true;
                uint32_t polls = 0;
                while (need_p1 || need_p23) {
                    if (*abort_flag) break;
                    if (need_p1 &&
                        (L2N ? mbar_try_wait(bars + B_IN, par(c + 1))
                             : mbar_try_wait(bars + rbar(B_LD0, c + 1), rpar(c + 1))) &&
                        mbar_try_wait(bars + B_KQF, par(c))) {
                        need_p1 = false;
                        if (!issue_p1(c + 1)) { fail(30); break; }
                        continue;
                    }
                    if (need_p23 && mbar_try_wait(bars + B_TT, par(c)) &&
                        (c == 0 || mbar_try_wait(bars + B_WTF, par(c - 1)))) {
                        need_p23 = false;
                        if (!issue_p23(c)) { fail(32); break; }
                        continue;
                    }
                    if (++polls > budget) { fail(need_p23 ? 31 : 30); break; }
                    __nanosleep(200);
                }
            }
            if (*abort_flag && issued > 0) {
                umma_commit(bars + B_DRAIN1);
                mbar_wait(bars + B_DRAIN1, 0, kDrainBudget);
            }
        }
        __syncwarp();
    } else {
        // ==================================================================== loader
        const int l = lane;
        int ld_issued[NREG] = {};
        // g, beta of tokens 2l, 2l+1 as stored (loaded a chunk ahead), and whether the
        // tokens lie inside the unit
        float rg0 = 0.f, rg1 = 0.f, rb0 = 0.f, rb1 = 0.f;
        bool in0 = false, in1 = false;
        auto fetch = [&](int c) {
            const long long t0 = un.tb + (long long)c * CC;
            const long long i0 = t0 + 2 * l, i1 = i0 + 1;
            in0 = i0 < un.te;
            in1 = i1 < un.te;
            rg0 = in0 ? prm.g[(size_t)i0 * prm.H_v + h] : 0.f;
            rg1 = in1 ? prm.g[(size_t)i1 * prm.H_v + h] : 0.f;
            rb0 = in0 ? prm.beta[(size_t)i0 * prm.H_v + h] : 0.f;
            rb1 = in1 ? prm.beta[(size_t)i1 * prm.H_v + h] : 0.f;
        };
        if (nch > 0) fetch(0);
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const int tc = (int)(un.tb + (long long)c * CC);
            bool okc = true;
            if (l == 0) {
                // ---- K, Q, V into this chunk's region once chunk c - NREG has left it
                unsigned char *rg = region(c);
                okc = c < NREG || wait_bar(rbar(B_RF0, c), rpar(c - NREG));
                if (okc) {
                    uint64_t *bar = bars + rbar(B_LD0, c);
                    mbar_arrive_expect_tx(bar, 16384 * (xa ? 2 : 3));
                    tma_load_3d(rg, &tm_k, bar, 0, hq, tc);
                    tma_load_3d(rg + SR_KB, &tm_k, bar, 64, hq, tc);
                    tma_load_3d(rg + SR_Q, &tm_q, bar, 0, hq, tc);
                    tma_load_3d(rg + SR_KB + SR_Q, &tm_q, bar, 64, hq, tc);
                    if (!xa) {
                        tma_load_3d(rg + SR_W, &tm_v, bar, 0, h, tc);
                        tma_load_3d(rg + SR_KB + SR_W, &tm_v, bar, 64, h, tc);
                    }
                    ++ld_issued[c % NREG];
                }
                if (okc && c >= NREG) okc = wait_bar(rbar(B_VF0, c), rpar(c - NREG));
            }
            okc = __shfl_sync(0xffffffffu, okc ? 1 : 0, 0) != 0;
            if (!okc) { if (l == 0) fail(40); break; }
            // ---- vectors of chunk c: G (in-chunk cumsum), gamma, exp(-G), decay to chunk
            // end, beta gamma
            float *vb = vecbuf(c);
            const float4 gt = gate_pair(rg0, rg1, rb0, rb1, in0, in1, prm.opts);
            const float pg0 = gt.x, pg1 = gt.y, pb0 = gt.z, pb1 = gt.w;
            float sc = pg0 + pg1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, sc, o);
                if (l >= o) sc += y;
            }
            const float G0 = sc - pg1, G1 = sc, Ge = __shfl_sync(0xffffffffu, sc, 31);
            const float gam0 = expf(G0), gam1 = expf(G1);
            vb[V_BETA + 2 * l] = pb0; vb[V_BETA + 2 * l + 1] = pb1;
            vb[V_G + 2 * l] = G0; vb[V_G + 2 * l + 1] = G1;
            vb[V_GAM + 2 * l] = gam0; vb[V_GAM + 2 * l + 1] = gam1;
            vb[V_INV + 2 * l] = expf(-G0); vb[V_INV + 2 * l + 1] = expf(-G1);
            vb[V_DTE + 2 * l] = expf(Ge - G0); vb[V_DTE + 2 * l + 1] = expf(Ge - G1);
            vb[V_BG + 2 * l] = pb0 * gam0; vb[V_BG + 2 * l + 1] = pb1 * gam1;
            __syncwarp();
            if (l == 0) mbar_arrive_local(bars + rbar(B_VEC0, c));
            if (c + 1 < nch) fetch(c + 1);
        }
        if (*abort_flag && l == 0) {
            // let this CTA's copies land before its shared memory is released
            for (int b = 0; b < NREG; ++b)
                if (ld_issued[b]) mbar_wait(bars + B_LD0 + b, par(ld_issued[b] - 1), kDrainBudget);
        }
        __syncwarp();
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 12) tmem_dealloc(tmem, 512);
}

// Segment start states and the final state: S_in(1) = B_0 (the first segment's chain
// started from S0), S_in(p + 1) = M_p S_in(p) + B_p, and S_final = S_in(P).  One CTA
// per (sequence, value head, 16 value columns); 256 threads, thread t owns row t / 2 and 8
// columns.  Exact fp32 on the CUDA cores.
__global__ void __launch_bounds__(256)
segment_scan_kernel(const float *ws_M, const float *ws_B, float *ws_S, float *S_final,
                    const int2 *seqs, int N, int H_v, int units_per_seq)
{
    __shared__ float S[DD][16];
    const int n = blockIdx.x, h = blockIdx.y, c0 = 16 * blockIdx.z, t = threadIdx.x;
    int u0, P;
    if (seqs) { const int2 e = seqs[n]; u0 = e.x; P = e.y; }
    else { u0 = n * units_per_seq; P = units_per_seq; }
    if (P < 1) return;
    const int d = t >> 1, cs = 8 * (t & 1);
    for (int e = t; e < DD * 16; e += 256) {
        const int dd = e >> 4, cc = e & 15;
        S[dd][cc] = ws_B[(((size_t)u0 * H_v + h) * DD + dd) * DD + c0 + cc];
    }
    __syncthreads();
#pragma unroll 1
    for (int p = 1; p < P; ++p) {
        const size_t su = ((size_t)(u0 + p) * H_v + h) * DD * DD;
        // S_in(p) for the correction pass
        float *dsts = ws_S + su + (size_t)d * DD + c0 + cs;
        *reinterpret_cast<float4 *>(dsts) = make_float4(S[d][cs], S[d][cs + 1], S[d][cs + 2], S[d][cs + 3]);
        *reinterpret_cast<float4 *>(dsts + 4) = make_float4(S[d][cs + 4], S[d][cs + 5], S[d][cs + 6], S[d][cs + 7]);
        const float *Mr = ws_M + su + (size_t)d * DD;
        float acc[8];
        const float4 b0 = *reinterpret_cast<const float4 *>(ws_B + su + (size_t)d * DD + c0 + cs);
        const float4 b1 = *reinterpret_cast<const float4 *>(ws_B + su + (size_t)d * DD + c0 + cs + 4);
        acc[0] = b0.x; acc[1] = b0.y; acc[2] = b0.z; acc[3] = b0.w;
        acc[4] = b1.x; acc[5] = b1.y; acc[6] = b1.z; acc[7] = b1.w;
#pragma unroll 4
        for (int e = 0; e < DD; e += 4) {
            const float4 m = *reinterpret_cast<const float4 *>(Mr + e);
            const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(mv[k], S[e + k][cs + j], acc[j]);
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) S[d][cs + j] = acc[j];
        __syncthreads();
    }
    if (S_final) {
        float *dst = S_final + (((size_t)n * H_v + h) * DD + d) * DD + c0 + cs;
        *reinterpret_cast<float4 *>(dst) = make_float4(S[d][cs], S[d][cs + 1], S[d][cs + 2], S[d][cs + 3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(S[d][cs + 4], S[d][cs + 5], S[d][cs + 6], S[d][cs + 7]);
    }
}

// Output correction of a segmented call: the local chain of segment p >= 1 started from
// zero, so its outputs miss Psi S_in(p), where Psi (the transfer chain's outputs) maps the
// segment's start state to every token's output.  out[t] += Psi[t] S_in(p) for the
// segment's tokens, on the tensor cores: (Psi S_in)^T = S_in^T Psi^T, A = S_in^T (bf16 in
// TMEM, lane = value column), B = a 64-token tile of Psi (K-major rows, by TMA), D in TMEM.
// The pass streams Psi and out (read and written once), so every chunk's Psi and out tiles
// come in by TMA a few chunks ahead; two warpgroups add D to the out tile, 32 tokens each,
// and write the sums back as pairs of values.
// One CTA per (unit, value head), two per SM; 288 threads: warps 0-7 convert S_in and run
// the epilogue (thread 0 issues the MMAs), warp 8 loads.
namespace {
constexpr int CR_THREADS = 288, CR_NBUF = 3;
constexpr uint32_t CR_TM_A = 0, CR_TM_D = 64;          // TMEM: S_in^T bf16, two 64-column D
constexpr uint32_t CR_BUF = 32768;                     // Psi tile (16 KB) | out tile (16 KB)
constexpr uint32_t CR_OUT = 16384;
constexpr uint32_t CR_BAR = CR_NBUF * CR_BUF;
constexpr uint32_t CR_SMEM = CR_BAR + 16 * 8 + 16 + 1024;
enum CrBar { CR_LD0 = 0, CR_FREE0 = CR_NBUF, CR_DONE0 = 2 * CR_NBUF, CR_DRAIN = CR_DONE0 + 2,
             CR_COUNT };
static_assert(CR_COUNT <= 16, "correction barriers");
static_assert(2 * (CR_SMEM + 1024) <= 233472, "two correction CTAs per SM");
}  // namespace

__global__ void __launch_bounds__(CR_THREADS)
segment_correct_kernel(const __grid_constant__ CUtensorMap tm_psi,
                       const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ ChainParams prm)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    Unit un;
    if (!unit_of(prm, blockIdx.x, un) || un.p == 0) return;
    const int nch = (int)((un.te - un.tb + CC - 1) / CC);
    if (nch == 0) return;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + CR_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + CR_BAR + 16 * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + CR_BAR + 16 * 8 + 4);
    if (warp == 0) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
    if (tid == 0) {
        for (int b = 0; b < CR_COUNT; ++b) mbar_init(bars + b, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t budget = prm.budget;
    auto wait_bar = [&](int b, uint32_t parity) -> bool {
        return bounded_wait(bars, b, parity, budget, abort_flag);
    };
    auto fail = [&](int where) { chain_abort(abort_flag, prm.err, where); };

    if (warp < 8) {
        const int t = tid, half = warp >> 2, v = 32 * (warp & 3) + lane;
        const uint32_t loff = (uint32_t)(32 * (warp & 3)) << 16;
        const bool odd = lane & 1;
        const uint32_t id_c = idesc_bf16(128, 64, false, false);
        int issued = 0;
        // S_in^T (bf16 pairs, lane v, column d / 2); warpgroup `half` converts d in
        // [64 half, 64 half + 64)
        const float *src = prm.ws_S + ((size_t)blockIdx.x * prm.H_v + h) * DD * DD;
#pragma unroll 1
        for (int db = 2 * half; db < 2 * half + 2; ++db) {
            uint32_t xb[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int d = 32 * db + 2 * j;
                xb[j] = pack2(src[(size_t)d * DD + v], src[(size_t)(d + 1) * DD + v]);
            }
            tmem_st16(tmem + loff + CR_TM_A + 16 * db, xb);
        }
        tmem_wait_st();
        tc_fence_before();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        auto issue = [&](int c) -> bool {        // thread 0; D(c & 1) was read at c - 2
            const int b = c % CR_NBUF;
            if (!wait_bar(CR_LD0 + b, par(c / CR_NBUF))) return false;
            tc_fence_after();
            const uint32_t base = smem_u32(sm + b * CR_BUF);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16_ta(tmem + CR_TM_D + 64 * (c & 1), tmem + CR_TM_A + 8 * ks,
                             sdesc_kmajor(base + (ks >> 2) * 8192 + (ks & 3) * 32), id_c, ks > 0);
            umma_commit(bars + CR_DONE0 + (c & 1));
            ++issued;
            return true;
        };
        if (t == 0 && !issue(0)) fail(50);
        // element (token r, value v) of a 64-token out tile: two 64-value boxes of 128-byte
        // rows in the 128-byte swizzle
        const uint32_t vcol = (uint32_t)(v >> 6) * 8192u, vb2 = (uint32_t)(v & 63) * 2u;
        const size_t rstride = (size_t)prm.H_v * DD;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const int b = c % CR_NBUF;
            // the next chunk's MMA (into the D buffer read at c - 1) runs beside this epilogue
            if (t == 0 && c + 1 < nch && !*abort_flag && !issue(c + 1)) fail(51);
            uint32_t ok2;
            {
                const bool w = t != 0 || (!*abort_flag && wait_bar(CR_DONE0 + (c & 1), par(c >> 1)));
                asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 256, p;\n\t"
                             "selp.u32 %0, 1, 0, q;\n\t}" : "=r"(ok2) : "r"(w ? 1u : 0u) : "memory");
            }
            if (!ok2) { fail(52); break; }
            tc_fence_after();
            uint32_t x[32];                          // tokens 32 half + j
            tmem_ld32(tmem + loff + CR_TM_D + 64 * (c & 1) + 32 * half, x);
            tmem_wait_ld();
            tc_fence_before();
            const long long t0 = un.tb + (long long)c * CC;
            const int L = (int)min((long long)CC, un.te - t0);
            const unsigned char *ot = sm + b * CR_BUF + CR_OUT + vcol;
            // lanes (v, v ^ 1) pair up: the even lane writes token 2m's two values, the odd
            // lane token 2m + 1's
            __nv_bfloat16 *obase = prm.out + ((size_t)t0 * prm.H_v + h) * DD + (v & ~1);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                float o[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = 32 * half + 2 * m + e;
                    const uint32_t off = (uint32_t)r * 128u + ((((vb2 >> 4) ^ (uint32_t)(r & 7)) << 4) | (vb2 & 15u));
                    o[e] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ot + off)) +
                           __uint_as_float(x[2 * m + e]);
                }
                const float recv = __shfl_xor_sync(0xffffffffu, odd ? o[0] : o[1], 1);
                const int r = 32 * half + 2 * m + (odd ? 1 : 0);
                const uint32_t val = odd ? pack2(recv, o[1]) : pack2(o[0], recv);
                if (r < L) *reinterpret_cast<uint32_t *>(obase + (size_t)r * rstride) = val;
            }
            // every thread has read D(c) and both tiles: the buffer goes back to the loader
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (t == 0) mbar_arrive_local(bars + CR_FREE0 + b);
        }
        if (t == 0 && *abort_flag && issued > 0) {
            umma_commit(bars + CR_DRAIN);
            mbar_wait(bars + CR_DRAIN, 0, kDrainBudget);
        }
    } else if (lane == 0) {
        // loader: Psi and out tiles of the unit's chunks
        int ld = 0;
        const int tbi = (int)un.tb;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const int b = c % CR_NBUF;
            if (c >= CR_NBUF && !wait_bar(CR_FREE0 + b, par((c - CR_NBUF) / CR_NBUF))) { fail(53); break; }
            unsigned char *buf = sm + b * CR_BUF;
            mbar_arrive_expect_tx(bars + CR_LD0 + b, CR_BUF);
            tma_load_3d(buf, &tm_psi, bars + CR_LD0 + b, 0, h, tbi + c * CC);
            tma_load_3d(buf + 8192, &tm_psi, bars + CR_LD0 + b, 64, h, tbi + c * CC);
            tma_load_3d(buf + CR_OUT, &tm_out, bars + CR_LD0 + b, 0, h, tbi + c * CC);
            tma_load_3d(buf + CR_OUT + 8192, &tm_out, bars + CR_LD0 + b, 64, h, tbi + c * CC);
            ++ld;
        }
        if (*abort_flag)
            for (int c = max(0, ld - CR_NBUF); c < ld; ++c)
                mbar_wait(bars + CR_LD0 + c % CR_NBUF, par(c / CR_NBUF), kDrainBudget);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// Unit table of a segmented varlen call: sequence n is split into ceil(len / seg) units
// (one for an empty sequence).  units[u] = {n, tb, te, p | P << 16}; seqs[n] = {u0, P};
// entries past the last unit get n = -1.  One thread (segmentation is chosen only when
// sequences are few).
__global__ void segment_plan_kernel(const int32_t *cu, int N, int seg, int U_max, int4 *units,
                                    int2 *seqs)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int u = 0;
    for (int n = 0; n < N; ++n) {
        const int tb = cu[n], te = cu[n + 1];
        const int len = te > tb ? te - tb : 0;
        int P = (len + seg - 1) / seg;
        if (P < 1) P = 1;
        if (u + P > U_max) P = max(U_max - u, 0);       // cannot happen for valid offsets
        seqs[n] = make_int2(u, P);
        for (int p = 0; p < P; ++p) {
            const int a = tb + p * seg, e = min(a + seg, te);
            units[u++] = make_int4(n, a, max(e, a), p | (P << 16));
        }
    }
    for (; u < U_max; ++u) units[u] = make_int4(-1, 0, 0, 0);
}

// ------------------------------------------------------------------------ host side
cudaError_t launch_prefill_tc_cluster(const void *q, const void *k, const void *v, const float *g,
                                      const float *beta, const float *S0, void *out, float *S_final,
                                      const int32_t *cu, int N, long long T_dense, long long T_total,
                                      int H_qk, int H_v, float scale, int opts, DeviceError *err,
                                      uint32_t budget, cudaStream_t stream);

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

bool make_map(CUtensorMap *map, const void *base, long long T_total, int H) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T_total};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device launch state: the shared-memory opt-in of each kernel instantiation and the
// SM count, set up once per device under a lock.
struct DeviceState {
    bool ready = false;
    int sms = 0;
};
constexpr int kMaxDev = 128;
std::mutex g_dev_mutex;
DeviceState g_dev[kMaxDev];

cudaError_t device_state(int *sms) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceState &s = g_dev[dev];
    if (!s.ready) {
        e = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(prefill_chain_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(prefill_chain_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(prefill_chain_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(prefill_chain_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(segment_correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CR_SMEM);
        if (e != cudaSuccess) return e;
        s.ready = true;
    }
    *sms = s.sms;
    return cudaSuccess;
}

constexpr size_t kStateBytes = (size_t)DD * DD * sizeof(float);


constexpr size_t kHead = 256;                 // error word (and padding)

}  // namespace

struct PrefillPlan {
    enum Kind { kChain, kCluster } kind;
    int seg_tokens;             // kChain: 0 = one unit per sequence
};

// Measured cost of one 64-token chunk step on one B200 (SM cycles, steady state):
// the single-CTA kernel here, and the four-CTA cluster kernel (prefill_tc_cluster.cu),
// whose chain per value-column quarter is shorter but takes four SMs per head.
constexpr double kChainStep = 8400.0, kClusterStep = 4700.0;
constexpr double kFill = 3.0;           // chunk steps to fill a pipeline at a unit's start
constexpr double kScanStep = 1.5;       // chunk steps per segment of the (sequential) scan
// The output correction streams Psi and out in and out once; measured, each of its CTAs
// moves about kCorrectCtaBps and the whole pass about kCorrectBps at most.  kStepSeconds
// (kChainStep at the full clock) converts its time into chunk steps.
constexpr double kCorrectCtaBps = 21e9, kCorrectBps = 6e12, kStepSeconds = 4.3e-6;

// Schedule for a call: the cluster kernel (one wave of four-CTA clusters per (sequence,
// value head)), or this kernel with one unit per sequence, or this kernel with segments of
// L chunks.  The model counts time on the critical path, assuming equal sequence lengths:
// unsegmented, ceil(units / slots) waves of C chunks; segmented, one pass of (2 P - 1)
// N H_v units (a local and, past the first segment, a transfer chain per segment) in
// ceil(units / SMs) waves of L chunks, the scan (about 4 steps) and the output correction
// (reads Psi, reads and writes out: HBM-bound, kCorrectBytesPerStep bytes per chunk step).
// override_tokens: 0 automatic, -1 one unit per sequence, -2 the cluster kernel, > 0 that
// segment length.
PrefillPlan plan_prefill(int N, long long T_total, int H_v, int sms, int override_tokens)
{
    PrefillPlan pl{PrefillPlan::kChain, 0};
    if (N <= 0 || T_total <= 0 || sms <= 0 || override_tokens == -1) return pl;
    if (override_tokens == -2) { pl.kind = PrefillPlan::kCluster; return pl; }
    if (override_tokens > 0) { pl.seg_tokens = override_tokens; return pl; }
    const long long C = (T_total / N + CC - 1) / CC;       // chunks per sequence (mean)
    const long long units0 = (long long)N * H_v;
    auto waves = [&](long long units, long long slots) { return (double)((units + slots - 1) / slots); };
    double best = waves(units0, sms) * ((double)C + kFill) * kChainStep;
    const double cluster = waves(units0, sms / 4) * ((double)C + kFill) * kClusterStep;
    if (cluster < best) { best = cluster; pl.kind = PrefillPlan::kCluster; }
    // bytes of out (read and written) and Psi (read), bf16, of the segments past the first
    const double corr_bytes = (double)T_total * H_v * DD * 2 * 3;
    // segment counts from the fewest up, each with segments of equal length L = ceil(C / P)
    // chunks (so the last one is not left short while the others set the time); more
    // segments (more transfer chains, scan steps and correction) must be 3 % better
    for (long long P = 2; P <= C / 8; ++P) {
        const long long L = (C + P - 1) / P;
        if ((C + L - 1) / L != P) continue;              // that length is P' < P segments
        const double ctas = (double)(P - 1) * units0;
        const double corr = corr_bytes * (double)(P - 1) / (double)P /
                            std::min(kCorrectBps, ctas * kCorrectCtaBps) / kStepSeconds;
        const double t = (waves((2 * P - 1) * units0, sms) * ((double)L + kFill) + kScanStep * (double)P + corr) *
                         kChainStep;
        if (t < 0.97 * best) { best = t; pl.kind = PrefillPlan::kChain; pl.seg_tokens = (int)(L * CC); }
    }
    return pl;
}

// What launch_prefill_chain will launch for these sizes: kind 0 = this kernel, 1 = the
// cluster kernel; seg_tokens 0 = one unit per sequence; launches = kernels per call.
void describe_prefill(int N, long long T_total, int H_v, int sms, int override_tokens,
                      size_t workspace_bytes, bool varlen, int *kind, int *seg_tokens, int *launches);

size_t chain_workspace_bytes(int N, long long T_total, int H_v, int sms, int override_tokens)
{
    const PrefillPlan pl = plan_prefill(N, T_total, H_v, sms, override_tokens);
    const int seg = pl.kind == PrefillPlan::kChain ? pl.seg_tokens : 0;
    if (seg == 0) return kHead;
    const long long U = N + T_total / seg;
    return kHead + (size_t)U * 16 + (size_t)N * 8 + 1024 + 3 * (size_t)U * H_v * kStateBytes +
           (size_t)T_total * H_v * DD * 2;
}

void describe_prefill(int N, long long T_total, int H_v, int sms, int override_tokens,
                      size_t workspace_bytes, bool varlen, int *kind, int *seg_tokens, int *launches)
{
    const PrefillPlan pl = plan_prefill(N, T_total, H_v, sms, override_tokens);
    int seg = pl.kind == PrefillPlan::kChain ? pl.seg_tokens : 0;
    if (seg && workspace_bytes < chain_workspace_bytes(N, T_total, H_v, sms, override_tokens)) seg = 0;
    *kind = pl.kind == PrefillPlan::kCluster ? 1 : 0;
    *seg_tokens = seg;
    *launches = seg ? (varlen ? 4 : 3) : 1;       // plan (varlen), transfers, scan, outputs
}

bool prefill_chain_supported(int dk, int dv, gdn_dtype dtype)
{
    return dk == DD && dv == DD && dtype == GDN_BF16;
}

int device_sm_count()
{
    int sms = 0;
    return device_state(&sms) == cudaSuccess ? sms : 0;
}

cudaError_t launch_prefill_chain(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *S0, void *out, float *S_final,
                                 const int32_t *cu, int N, long long T_dense, long long T_total,
                                 int H_qk, int H_v, float scale, int opts, void *workspace,
                                 size_t workspace_bytes, uint32_t budget, int seg_override,
                                 cudaStream_t stream)
{
    if (T_total >= (1LL << 31) || N <= 0) return cudaErrorInvalidValue;
    int sms = 0;
    cudaError_t e = device_state(&sms);
    if (e != cudaSuccess) return e;
    ChainParams prm;
    memset(&prm, 0, sizeof(prm));
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, T_total, H_qk) || !make_map(&mk, k, T_total, H_qk) ||
        !make_map(&mv, v, T_total, H_v))
        return cudaErrorInvalidValue;
    prm.g = g; prm.beta = beta; prm.S0 = S0; prm.S_final = S_final;
    prm.out = (__nv_bfloat16 *)out; prm.cu_seqlens = cu; prm.T_dense = T_dense;
    prm.N = N; prm.H_qk = H_qk; prm.H_v = H_v; prm.scale = scale; prm.opts = opts;
    prm.err = reinterpret_cast<DeviceError *>(workspace);
    prm.budget = budget;
    const bool l2n = opts & kOptL2Norm;

    const PrefillPlan pl = plan_prefill(N, T_total, H_v, sms, seg_override);
    if (pl.kind == PrefillPlan::kCluster)
        return launch_prefill_tc_cluster(q, k, v, g, beta, S0, out, S_final, cu, N, T_dense, T_total,
                                         H_qk, H_v, scale, opts, prm.err, budget, stream);
    int seg = pl.seg_tokens;
    if (seg && workspace_bytes < chain_workspace_bytes(N, T_total, H_v, sms, seg_override)) seg = 0;
    int U = N;
    int2 *seqs = nullptr;
    if (seg) {
        U = (int)(N + T_total / seg);
        unsigned char *p = reinterpret_cast<unsigned char *>(workspace) + kHead;
        int4 *units = reinterpret_cast<int4 *>(p);
        p += (size_t)U * 16;
        seqs = reinterpret_cast<int2 *>(p);
        p += (size_t)N * 8;
        p = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
        prm.ws_M = reinterpret_cast<float *>(p);
        prm.ws_B = prm.ws_M + (size_t)U * H_v * DD * DD;
        prm.ws_S = prm.ws_B + (size_t)U * H_v * DD * DD;
        prm.ws_Psi = reinterpret_cast<__nv_bfloat16 *>(prm.ws_S + (size_t)U * H_v * DD * DD);
        prm.seg_tokens = seg;
        if (cu) {
            segment_plan_kernel<<<1, 32, 0, stream>>>(cu, N, seg, U, units, seqs);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            prm.units = units;
        } else {
            prm.units_per_seq = (int)((T_dense + seg - 1) / seg);
            U = N * prm.units_per_seq;
            seqs = nullptr;
        }
    }
    // the chains: per unit, the local chain (slice 1, or the only slice) and, for segments
    // past the first, the transfer chain (slice 0)
    auto kc = seg ? (l2n ? prefill_chain_kernel<true, true> : prefill_chain_kernel<false, true>)
                  : (l2n ? prefill_chain_kernel<true, false> : prefill_chain_kernel<false, false>);
    kc<<<dim3((unsigned)U, (unsigned)H_v, seg ? 2 : 1), CH_THREADS, CH_SMEM, stream>>>(mq, mk, mv, prm);
    if ((e = cudaGetLastError()) != cudaSuccess || !seg) return e;
    // segment start states and final states, then the output corrections
    segment_scan_kernel<<<dim3((unsigned)N, (unsigned)H_v, DD / 16), 256, 0, stream>>>(
        prm.ws_M, prm.ws_B, prm.ws_S, S_final, seqs, N, H_v, prm.units_per_seq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap mpsi, mout;
    if (!make_map(&mpsi, prm.ws_Psi, T_total, H_v) || !make_map(&mout, prm.out, T_total, H_v))
        return cudaErrorInvalidValue;
    segment_correct_kernel<<<dim3((unsigned)U, (unsigned)H_v), CR_THREADS, CR_SMEM, stream>>>(mpsi, mout, prm);
    return cudaGetLastError();
}

}  // namespace gdn
