// QSA compressed indexer on sm_100a: the block cache (mean-pooled, rotary-encoded keys)
// and the decode-time indexer (multi-query block scores, budgeted selection, expansion
// to tokens).  Operation and contract: include/qsa.h ("論文解説: Qwen3.8-Next の設計",
// section "部品②: QSA").
//
//   qsa_compress_kernel   stream of 4 token keys in, one encoded block key out (HBM-bound).
//   qsa_score_kernel      stream over the block cache, each row read once for the T <= 4
//                         queries of its sequence: one fp32 score per (query, eligible
//                         block) and a 4096-bin histogram of the scores' top 12 order
//                         bits per query (HBM-bound; the dominant kernel of the indexer).
//                         The CTA that finishes a sequence's last work item derives each
//                         query's threshold bin (the bin that holds the budget-th score).
//   qsa_collect_kernel    pass over the scores (L2-resident): blocks above the threshold
//                         bin are kept, blocks inside it become candidates.
//   qsa_finish_kernel     per query: exact selection among the candidates (two radix
//                         passes over the low score bits, then the block index for ties),
//                         blocks written in block order, with scores and tokens; the
//                         query's workspace record is zeroed again.
//
// "Query units": query j of sequence n is unit n T + j; it sits at position q_pos[n] + j
// and has its own causal cut.  Scores are reduced to one vector per query: its four heads
// share the key and the logits are summed, so sum_h q_h . k = (sum_h q_h) . k.  Ranking
// compares 32-bit order keys of the fp32 scores (a monotone map of the float's bits), and
// ties fall to the smaller block index, which makes the kept set unique.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "device_once.h"
#include "../../include/qsa.h"

namespace gdn {
namespace {

constexpr int QR = GDN_QSA_R, QD = GDN_QSA_DIM, QROPE = GDN_QSA_ROPE_DIMS;
constexpr int QHALF = QROPE / 2, QHEADS = GDN_QSA_HEADS;
constexpr int HBITS = 12, HBINS = 1 << HBITS;        // first radix digit (score kernel)
constexpr int SURE_CAP = GDN_QSA_MAX_BUDGET;          // blocks kept above the threshold bin
constexpr int CAND_CAP = 8192;                        // candidates listed from that bin
constexpr int SCORE_TILE = 512;                       // cache rows per scoring work item
constexpr int COLLECT_TILE = 4096;                    // score entries per collect work item
constexpr int kScoreThreads = 256, kFinishThreads = 1024;

// One query unit's record in the indexer workspace (zero between calls except thr/rank;
// the score kernel counts a sequence's finished work items in its first unit's record).
struct SeqWork {
    uint32_t hist[HBINS];     // scores per top-12-bit bin, filled by the score kernel
    uint32_t n_sure, n_cand;  // list lengths (n_cand counts past CAND_CAP too)
    int32_t thr_bin, rank;    // threshold bin (-1: keep every eligible block), rank inside it
    uint32_t items_done;      // score work items finished (the last one sets thr_bin, rank)
    uint32_t pad[3];
    uint2 sure[SURE_CAP];     // (order key, block) kept outright
    uint2 cand[CAND_CAP];     // (order key, block) inside the threshold bin
};
static_assert(sizeof(SeqWork) % 16 == 0, "workspace records stay 16-byte aligned");

constexpr double kTwoPiHi = 6.283185307179586;        // 2 pi rounded to double
constexpr double kTwoPiLo = 2.4492935982947064e-16;   // 2 pi - kTwoPiHi
constexpr double kInvTwoPi = 0.15915494309189535;

// Rotation angle p * w, reduced into [-pi, pi] in double precision by subtracting the
// nearest multiple of a two-part 2 pi (Cody and Waite's additive reduction).  Positions
// reach 2^31, where a float angle would be off by whole hundredths of a radian.
__device__ __forceinline__ float reduced_angle(double p, double w) {
    const double x = p * w;
    const double n = rint(x * kInvTwoPi);
    return (float)fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, x));
}

__device__ __forceinline__ double rotary_freq(double base, int i) {   // base^(-i / 32)
    return pow(base, -(double)i / (double)QHALF);
}

__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Programmatic dependent launch: the next kernel of the call may start its prologue while
// this one drains; it waits for this grid's completion (and its memory) before it reads
// anything this grid wrote.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_primary() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Monotone map float -> uint32 (larger score, larger key); -0 is taken as +0 so that equal
// scores always get equal keys.
__device__ __forceinline__ uint32_t order_key(float x) {
    if (x == 0.f) x = 0.f;
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Rows of sequence n in the cache (inside its total_blocks rows, whatever the offsets say).
__device__ __forceinline__ int cached_rows(const int32_t *cu_blocks, int n, int total_blocks) {
    const int end = cu_blocks[n + 1] < total_blocks ? cu_blocks[n + 1] : total_blocks;
    return end > cu_blocks[n] ? end - cu_blocks[n] : 0;
}

// Blocks of sequence n that its query j (at position q_pos[n] + j) may score: whole blocks
// at or before that position, inside the cache.
__device__ __forceinline__ int eligible(const int32_t *cu_blocks, const int32_t *q_pos, int n,
                                        int total_blocks, int j = 0) {
    const long long cached = cached_rows(cu_blocks, n, total_blocks);
    const long long seen = ((long long)q_pos[n] + j + 1) / QR;
    const long long e = cached < seen ? cached : seen;
    return e > 0 ? (int)e : 0;
}

// Exclusive prefix sum of one int per thread over the CTA (blockDim.x multiple of 32,
// at most 1024); `total` gets the sum.  Uses 33 ints of shared scratch.
__device__ int block_exclusive_scan(int v, int *scratch, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) scratch[lane] = w;          // inclusive warp totals
        if (lane == 31) scratch[32] = w;
    }
    __syncthreads();
    const int before = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
    total = scratch[32];
    __syncthreads();                                // scratch may be reused at once
    return before;
}

// item0[m] = first work item of unit m, item0[M] = item count; a unit gets
// ceil(eligible / tile) items.  Units are sequences (M = N, eligibility of their last query
// T - 1, which sees the most blocks) or queries (M = N T, unit m = query m mod T of
// sequence m / T).  M <= GDN_QSA_MAX_SEQS.
__device__ __forceinline__ int unit_eligible(const int32_t *cu_blocks, const int32_t *q_pos,
                                             int total_blocks, int m, int T, bool per_query) {
    return per_query ? eligible(cu_blocks, q_pos, m / T, total_blocks, m % T)
                     : eligible(cu_blocks, q_pos, m, total_blocks, T - 1);
}

__device__ void build_items(int *item0, int *scratch, int M, const int32_t *cu_blocks,
                            const int32_t *q_pos, int total_blocks, int tile, int T,
                            bool per_query) {
    const int per = (M + blockDim.x - 1) / blockDim.x;
    const int m0 = threadIdx.x * per;
    int local = 0;
    for (int m = m0; m < m0 + per && m < M; ++m)
        local += (unit_eligible(cu_blocks, q_pos, total_blocks, m, T, per_query) + tile - 1) / tile;
    int total;
    int acc = block_exclusive_scan(local, scratch, total);
    for (int m = m0; m < m0 + per && m < M; ++m) {
        item0[m] = acc;
        acc += (unit_eligible(cu_blocks, q_pos, total_blocks, m, T, per_query) + tile - 1) / tile;
    }
    if (threadIdx.x == 0) item0[M] = total;
    __syncthreads();
}

// TP values per lane -> lane l holds the sum over its aligned group of W lanes of value
// (l mod TP): halving exchanges, then the remaining lane halves inside the group.
template <int TP, int W>
__device__ __forceinline__ float transpose_sum(float (&x)[TP], int lane) {
#pragma unroll
    for (int m = TP / 2; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = upper ? x[i] : x[i + m];
            const float keep = upper ? x[i + m] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
#pragma unroll
    for (int m = TP; m < W; m <<= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], m);
    return x[0];
}


// Largest n < N with item0[n] <= it (sequences without items are skipped).
__device__ __forceinline__ int seq_of_item(const int *item0, int N, int it) {
    int lo = 0, hi = N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (item0[mid] <= it) lo = mid; else hi = mid;
    }
    return lo;
}

// Among nbins counts in h (shared), the highest bin b with
//   count(bins above b) < r <= count(bins at or above b)       (1 <= r <= total)
// -> out[0] = b, out[1] = count(bins above b), out[2] = h[b].  nbins is a multiple of
// blockDim.x; every thread of the CTA calls this.
__device__ void find_from_top(const uint32_t *h, int nbins, int r, int *scratch, int *out) {
    const int per = nbins / blockDim.x;
    const int top = nbins - per * threadIdx.x;      // this thread owns bins [top - per, top)
    if (threadIdx.x == 0) { out[0] = 0; out[1] = 0; out[2] = 0; }   // (r outside 1..total)
    int local = 0;
    for (int b = top - 1; b >= top - per; --b) local += (int)h[b];
    int total;
    const int above = block_exclusive_scan(local, scratch, total);
    if (above < r && r <= above + local) {
        int acc = above;
        for (int b = top - 1; b >= top - per; --b) {
            if (acc + (int)h[b] >= r) { out[0] = b; out[1] = acc; out[2] = (int)h[b]; break; }
            acc += (int)h[b];
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------ compress
// A half-warp per cache row: lane l (0..15) owns dims 8 l .. 8 l + 7 of the row.  Lanes
// 0-3 hold the first rotary halves (dims 0..31), lanes 4-7 their partners (32..63), lanes
// 8-15 the pass-through dims.
__global__ void __launch_bounds__(256) qsa_compress_kernel(
    const __nv_bfloat16 *__restrict__ k, const int32_t *__restrict__ cu_seqlens,
    const int32_t *__restrict__ cu_blocks, const int32_t *__restrict__ pos0,
    __nv_bfloat16 *__restrict__ k_hat, int N, int total_blocks, double base)
{
    __shared__ double w_s[QHALF];
    if (threadIdx.x < QHALF) w_s[threadIdx.x] = rotary_freq(base, threadIdx.x);
    __syncthreads();
    const int lane = threadIdx.x & 31, hl = lane & 15;
    const unsigned hmask = 0xffffu << (lane & 16);
    const int half_id = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 4);
    const int n_halves = (int)((gridDim.x * blockDim.x) >> 4);
    for (int row = half_id; row < total_blocks; row += n_halves) {
        int lo = 0, hi = N;                          // largest n with cu_blocks[n] <= row
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(cu_blocks + mid) <= row) lo = mid; else hi = mid;
        }
        const int n = lo;
        const int b = row - __ldg(cu_blocks + n);
        const int t0 = __ldg(cu_seqlens + n), len = __ldg(cu_seqlens + n + 1) - t0;
        const int nb = __ldg(cu_blocks + n + 1) - __ldg(cu_blocks + n);
        if (b < 0 || b >= nb || b >= len / QR) continue;    // uniform over the half-warp
        const __nv_bfloat16 *src = k + (size_t)(t0 + QR * b) * QD + 8 * hl;
        uint4 tok[QR];
#pragma unroll
        for (int j = 0; j < QR; ++j) tok[j] = ld_stream(src + (size_t)j * QD);
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
#pragma unroll
        for (int j = 0; j < QR; ++j) {
            const uint32_t wv[4] = {tok[j].x, tok[j].y, tok[j].z, tok[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) { x[2 * e] += bf_lo(wv[e]); x[2 * e + 1] += bf_hi(wv[e]); }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= 1.f / QR;
        float y[8];                                  // the rotation partner's pooled value
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = __shfl_xor_sync(hmask, x[e], 4, 16);
        if (hl < 8) {
            const double p = (double)(pos0 ? __ldg(pos0 + n) : 0) + (double)QR * b;
            const bool first = hl < 4;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float s, c;
                __sincosf(reduced_angle(p, w_s[8 * (hl & 3) + e]), &s, &c);
                x[e] = first ? fmaf(x[e], c, -y[e] * s) : fmaf(x[e], c, y[e] * s);
            }
        }
        uint4 o;
        o.x = pack_bf2(x[0], x[1]); o.y = pack_bf2(x[2], x[3]);
        o.z = pack_bf2(x[4], x[5]); o.w = pack_bf2(x[6], x[7]);
        *reinterpret_cast<uint4 *>(k_hat + (size_t)row * QD + 8 * hl) = o;
    }
}

// The threshold of sequence n from its finished histogram (h: HBINS counts in shared
// memory, loaded by the caller): the bin holding the budget-th best score and that
// score's rank inside the bin; bin -1 when every eligible block is kept.
__device__ void threshold_of(const uint32_t *h, int elig, int budget, int *scratch, int *res,
                             int &bin, int &rank) {
    if (elig <= budget) { bin = -1; rank = elig; return; }
    find_from_top(h, HBINS, budget, scratch, res);
    bin = res[0];
    rank = budget - res[1];
    __syncthreads();
}

// --------------------------------------------------------------------- score
// Persistent CTAs; CTA c takes the contiguous run of work items [c per, (c + 1) per) over
// the sequences, so it stays on one sequence for long stretches (one set of summed queries
// and one histogram hand-off per sequence it touches).  Each cache row is read once for all
// T queries of its sequence (query j at position q_pos + j scores only the rows it may see).
// A group of 8 lanes owns a row (lane g owns dims 16 g .. 16 g + 15, 32 bytes), a warp 4
// rows per step, 4 steps deep (4 KB per warp in flight).  With T > 1 queries each lane
// holds its 16 dims of all T summed queries; the T partial dots are summed over the group
// transposed, so lane j of the group ends with query j's score.
constexpr int kScoreUnroll = 4;
constexpr int kMmaTiles = 2;            // 16-row tiles per warp and pass (T > 1 path)

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
// D += A (16 x 16, bf16, row-major fragment) * B (16 x 8, bf16, column fragment), fp32 D
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int T>
__global__ void __launch_bounds__(kScoreThreads, T == 1 ? 4 : 2) qsa_score_kernel(
    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ q_pos,
    const __nv_bfloat16 *__restrict__ k_hat, const int32_t *__restrict__ cu_blocks, int N,
    int total_blocks, int budget, double base, SeqWork *__restrict__ ws,
    float *__restrict__ scores)
{
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem);               // [T][HBINS]
    float *qbar = reinterpret_cast<float *>(hist + T * HBINS);          // [T][QD]
    int *scratch = reinterpret_cast<int *>(qbar + T * QD);
    int *item0 = scratch + 36;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < T * HBINS; i += blockDim.x) hist[i] = 0;
    build_items(item0, scratch, N, cu_blocks, q_pos, total_blocks, SCORE_TILE, T, false);
    const int n_items = item0[N];
    const int per = (n_items + gridDim.x - 1) / gridDim.x;
    int it = blockIdx.x * per;
    const int it_end = min(n_items, it + per);
    while (it < it_end) {
        const int n = seq_of_item(item0, N, it);
        const int seg_end = min(it_end, item0[n + 1]);
        const int r0 = (it - item0[n]) * SCORE_TILE;
        const int r1 = min(eligible(cu_blocks, q_pos, n, total_blocks, T - 1),
                           (seg_end - item0[n]) * SCORE_TILE);
        const long long row0 = cu_blocks[n];
        const int cached = cached_rows(cu_blocks, n, total_blocks);
        int elig[T];
#pragma unroll
        for (int j = 0; j < T; ++j) elig[j] = eligible(cu_blocks, q_pos, n, total_blocks, j);
        for (int e = tid; e < T * QD; e += blockDim.x) {   // sum over heads of RoPE(q_h, pos)
            const int j = e / QD, d = e - j * QD;
            const __nv_bfloat16 *qn = q + ((size_t)n * T + j) * QHEADS * QD;
            float acc = 0.f;
            if (d < QROPE) {
                float sn, cs;
                sincosf(reduced_angle((double)q_pos[n] + j, rotary_freq(base, d & (QHALF - 1))),
                        &sn, &cs);
                const int pd = d ^ QHALF;           // rotation partner
                const float sg = d < QHALF ? -sn : sn;
#pragma unroll
                for (int h = 0; h < QHEADS; ++h)
                    acc += fmaf(__bfloat162float(qn[h * QD + d]), cs,
                                sg * __bfloat162float(qn[h * QD + pd]));
            } else {
#pragma unroll
                for (int h = 0; h < QHEADS; ++h) acc += __bfloat162float(qn[h * QD + d]);
            }
            qbar[e] = acc;
        }
        __syncthreads();
        float *sc = scores + (size_t)T * row0;     // query j's scores at sc + j * cached
        if constexpr (T > 1) {
            // Several queries: the rows against the T summed queries as a skinny contraction
            // on the tensor cores, 16 rows per m16n8k16 tile.  Column n of B holds the high
            // (n < 4) or low (n >= 4) bf16 part of summed query n & 3, so a score keeps about
            // 16 significant bits of the query (the keys are bf16 already) and is the sum of
            // columns j and j + 4.  The 128 dims are permuted consistently in A and B so that
            // lane (g, t) reads dims [32 t, 32 t + 32) of rows g and g + 8 as four 16-byte
            // loads each: in k step s its fragment pairs are dims 32 t + 4 s + {0, 1} and
            // + {2, 3}.
            const int g = lane >> 2, t4 = lane & 3;
            uint32_t bq[8][2];
            {
                const int j = g & 3;
                const bool lo = g >= 4;
#pragma unroll
                for (int st = 0; st < 8; ++st)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int d = 32 * t4 + 4 * st + 2 * hh;
                        const float x0 = j < T ? qbar[j * QD + d] : 0.f;
                        const float x1 = j < T ? qbar[j * QD + d + 1] : 0.f;
                        const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
                        const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
                        bq[st][hh] = lo ? pack_bf16x2(x0 - h0, x1 - h1) : pack_bf16x2(x0, x1);
                    }
            }
            // after the exchange lane t4 reports queries jq, jq + 1 of row g (t4 < 2) or
            // row g + 8 (t4 >= 2)
            const int jq = 2 * (t4 & 1);
            const bool upper = t4 >= 2;
            const int eqa = jq < T ? eligible(cu_blocks, q_pos, n, total_blocks, jq) : 0;
            const int eqb = jq + 1 < T ? eligible(cu_blocks, q_pos, n, total_blocks, jq + 1) : 0;
            const __nv_bfloat16 *kb = k_hat + (size_t)row0 * QD + 32 * t4;
            constexpr int kWarps = kScoreThreads / 32;
            for (int tb = r0 + 16 * warp; tb < r1; tb += 16 * kWarps * kMmaTiles) {
                uint4 ra[kMmaTiles][2][4];
#pragma unroll
                for (int u = 0; u < kMmaTiles; ++u)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int row = tb + 16 * kWarps * u + g + 8 * hh;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            ra[u][hh][i] = row < r1 ? ld_stream(kb + (size_t)row * QD + 8 * i)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                for (int u = 0; u < kMmaTiles; ++u) {
                    const uint32_t *wa = reinterpret_cast<const uint32_t *>(ra[u][0]);
                    const uint32_t *wb = reinterpret_cast<const uint32_t *>(ra[u][1]);
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int st = 0; st < 8; ++st)
                        mma_bf16_16816(d, wa[2 * st], wb[2 * st], wa[2 * st + 1], wb[2 * st + 1],
                                       bq[st][0], bq[st][1]);
                    // lane t4 holds columns 2 t4, 2 t4 + 1 of rows g (d0, d1) and g + 8 (d2,
                    // d3); its partner t4 ^ 2 holds the other part of the same two queries
                    const float x0 = __shfl_xor_sync(0xffffffffu, upper ? d[0] : d[2], 2);
                    const float x1 = __shfl_xor_sync(0xffffffffu, upper ? d[1] : d[3], 2);
                    const float sa = (upper ? d[2] : d[0]) + x0, sb = (upper ? d[3] : d[1]) + x1;
                    const int row = tb + 16 * kWarps * u + g + (upper ? 8 : 0);
                    if (row < eqa) {
                        sc[(size_t)jq * cached + row] = sa;
                        atomicAdd(&hist[jq * HBINS + (order_key(sa) >> (32 - HBITS))], 1u);
                    }
                    if (row < eqb) {
                        sc[(size_t)(jq + 1) * cached + row] = sb;
                        atomicAdd(&hist[(jq + 1) * HBINS + (order_key(sb) >> (32 - HBITS))], 1u);
                    }
                }
            }
        } else {
            constexpr int TP = T == 1 ? 1 : (T == 2 ? 2 : 4);
            const int g = lane >> 3, gl = lane & 7;
            float qv[T][16];
#pragma unroll
            for (int j = 0; j < T; ++j)
#pragma unroll
                for (int e = 0; e < 16; ++e) qv[j][e] = qbar[j * QD + 16 * gl + e];
            const int jq = gl < T ? gl : 0;         // the query this lane reports
            float *scq = sc + (size_t)jq * cached;
            uint32_t *hq = hist + jq * HBINS;
            const int eq = gl < T ? eligible(cu_blocks, q_pos, n, total_blocks, jq) : 0;
            const __nv_bfloat16 *kb = k_hat + (size_t)row0 * QD + 16 * gl;
            for (int base_row = r0 + 4 * warp; base_row < r1; base_row += 32 * kScoreUnroll) {
                uint4 a[kScoreUnroll][2];
#pragma unroll
                for (int u = 0; u < kScoreUnroll; ++u) {
                    const int row = base_row + g + 32 * u;
                    if (row < r1) {
                        a[u][0] = ld_stream(kb + (size_t)row * QD);
                        a[u][1] = ld_stream(kb + (size_t)row * QD + 8);
                    } else {
                        a[u][0] = make_uint4(0, 0, 0, 0);
                        a[u][1] = make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int u = 0; u < kScoreUnroll; ++u) {
                    const uint32_t wv[8] = {a[u][0].x, a[u][0].y, a[u][0].z, a[u][0].w,
                                            a[u][1].x, a[u][1].y, a[u][1].z, a[u][1].w};
                    float kf[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) { kf[2 * e] = bf_lo(wv[e]); kf[2 * e + 1] = bf_hi(wv[e]); }
                    float p[TP > 1 ? TP : 1];
#pragma unroll
                    for (int j = 0; j < (TP > 1 ? TP : 1); ++j) p[j] = 0.f;
#pragma unroll
                    for (int j = 0; j < T; ++j) {
                        float s0 = 0.f, s1 = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            s0 = fmaf(qv[j][2 * e], kf[2 * e], s0);
                            s1 = fmaf(qv[j][2 * e + 1], kf[2 * e + 1], s1);
                        }
                        p[j] = s0 + s1;
                    }
                    float sum;
                    if constexpr (T == 1) {
                        sum = p[0];
                        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                    } else {
                        sum = transpose_sum<TP, 8>(p, lane);
                    }
                    const int row = base_row + g + 32 * u;
                    if (gl < T && row < eq) {
                        scq[row] = sum;
                        atomicAdd(&hq[order_key(sum) >> (32 - HBITS)], 1u);
                    }
                }
            }
        }
        __syncthreads();                            // hand this sequence's counts on
        for (int i = tid; i < T * HBINS; i += blockDim.x) {
            const uint32_t v = hist[i];
            if (v) { atomicAdd(&ws[(size_t)n * T + i / HBINS].hist[i % HBINS], v); hist[i] = 0; }
        }
        // the CTA that completes the sequence's last work item derives the thresholds of
        // its T queries (every thread fences its own counts before the one arrival on the
        // item counter)
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const uint32_t mine = (uint32_t)(seg_end - it);
            const uint32_t all = (uint32_t)(item0[n + 1] - item0[n]);
            scratch[35] = (atomicAdd(&ws[(size_t)n * T].items_done, mine) + mine == all) ? 1 : 0;
            __threadfence();
        }
        __syncthreads();
        if (scratch[35]) {
#pragma unroll 1
            for (int j = 0; j < T; ++j) {
                SeqWork &wj = ws[(size_t)n * T + j];
                for (int i = tid; i < HBINS; i += blockDim.x) hist[i] = __ldcg(&wj.hist[i]);
                __syncthreads();
                int thr, rank;
                threshold_of(hist, elig[j], budget, scratch, scratch + 32, thr, rank);
                if (tid == 0) { wj.thr_bin = thr; wj.rank = rank; }
                __syncthreads();
            }
            for (int i = tid; i < HBINS; i += blockDim.x) hist[i] = 0;
            __syncthreads();
        }
        it = seg_end;
    }
    pdl_launch_dependents();
}

// ------------------------------------------------------------------- collect
// Same contiguous work split as the score kernel (COLLECT_TILE scores per item); each
// CTA derives the threshold of every sequence it touches from that sequence's histogram.
constexpr int kCollectPer = COLLECT_TILE / kScoreThreads;      // scores per thread per item

__global__ void __launch_bounds__(kScoreThreads) qsa_collect_kernel(
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ cu_blocks, int N, int T,
    int total_blocks, const float *__restrict__ scores, SeqWork *__restrict__ ws)
{
    extern __shared__ __align__(16) unsigned char smem[];
    int *scratch = reinterpret_cast<int *>(smem);
    int *item0 = scratch + 36;
    __shared__ uint32_t s_base[2];
    const int U = N * T;                            // query units: query u % T of sequence u / T
    build_items(item0, scratch, U, cu_blocks, q_pos, total_blocks, COLLECT_TILE, T, true);
    const int n_items = item0[U];
    const int per = (n_items + gridDim.x - 1) / gridDim.x;
    int it = blockIdx.x * per;
    const int it_end = min(n_items, it + per);
    pdl_wait_primary();                             // scores and thresholds are complete
    while (it < it_end) {
        const int u = seq_of_item(item0, U, it);
        const int n = u / T, j = u - n * T;
        const int seg_end = min(it_end, item0[u + 1]);
        const int elig = eligible(cu_blocks, q_pos, n, total_blocks, j);
        const int r0 = (it - item0[u]) * COLLECT_TILE;
        const int r1 = min(elig, (seg_end - item0[u]) * COLLECT_TILE);
        SeqWork &w = ws[u];
        const int thr = w.thr_bin;
        const float *sc = scores + (size_t)T * cu_blocks[n] +
                          (size_t)j * cached_rows(cu_blocks, n, total_blocks);
        // rows r0 + threadIdx.x + 256 e, all loads of a step issued before any is used;
        // the loop bound is uniform over the CTA, as the block scan below needs
        for (int b = r0; b < r1; b += COLLECT_TILE) {
            float v[kCollectPer];
#pragma unroll
            for (int e = 0; e < kCollectPer; ++e) {
                const int row = b + threadIdx.x + kScoreThreads * e;
                v[e] = row < r1 ? __ldcg(sc + row) : 0.f;
            }
            // one reservation per list for the whole CTA: per-thread counts packed in one
            // int (kept blocks in the low 16 bits, candidates in the high 16), one scan
            uint32_t keys[kCollectPer];
            unsigned sure_m = 0, cand_m = 0;
#pragma unroll
            for (int e = 0; e < kCollectPer; ++e) {
                const int row = b + threadIdx.x + kScoreThreads * e;
                keys[e] = order_key(v[e]);
                const int bin = (int)(keys[e] >> (32 - HBITS));
                if (row < r1) {
                    if (thr < 0 || bin > thr) sure_m |= 1u << e;
                    else if (bin == thr) cand_m |= 1u << e;
                }
            }
            int total;
            const int before = block_exclusive_scan(__popc(sure_m) | (__popc(cand_m) << 16), scratch,
                                                    total);
            if (threadIdx.x == 0) {
                s_base[0] = (total & 0xffff) ? atomicAdd(&w.n_sure, (uint32_t)(total & 0xffff)) : 0u;
                s_base[1] = (total >> 16) ? atomicAdd(&w.n_cand, (uint32_t)(total >> 16)) : 0u;
            }
            __syncthreads();
            uint32_t slot_s = s_base[0] + (uint32_t)(before & 0xffff);
            uint32_t slot_c = s_base[1] + (uint32_t)(before >> 16);
#pragma unroll
            for (int e = 0; e < kCollectPer; ++e) {
                const uint32_t row = (uint32_t)(b + threadIdx.x + kScoreThreads * e);
                if (sure_m & (1u << e)) {
                    if (slot_s < SURE_CAP) w.sure[slot_s] = make_uint2(keys[e], row);
                    ++slot_s;
                } else if (cand_m & (1u << e)) {
                    if (slot_c < CAND_CAP) w.cand[slot_c] = make_uint2(keys[e], row);
                    ++slot_c;
                }
            }
        }
        it = seg_end;
    }
    pdl_launch_dependents();
}

// -------------------------------------------------------------------- finish
// One CTA per query unit.  Dynamic shared memory: the radix-pass histogram (2048 words), the
// kept list (SURE_CAP pairs), the candidates (CAND_CAP pairs) and a bitmap of kept blocks
// (kBitmapBlocks bits).  With at most kBitmapBlocks eligible blocks the kept set is marked
// in the bitmap and written out in block order by one ordered compaction; longer caches
// sort the kept list instead.
constexpr int kPassBins = 2048;
constexpr int kBitmapBlocks = 1 << 18;
constexpr int kBitmapWords = kBitmapBlocks / 32;
constexpr size_t kFinishSmem = kPassBins * 4 + SURE_CAP * 8 + CAND_CAP * 8 + kBitmapWords * 4;

__global__ void __launch_bounds__(kFinishThreads) qsa_finish_kernel(
    const int32_t *__restrict__ q_pos, const int32_t *__restrict__ cu_blocks, int T,
    int total_blocks, int budget, const float *__restrict__ scores, SeqWork *__restrict__ ws,
    int32_t *__restrict__ block_idx, float *__restrict__ block_score,
    int32_t *__restrict__ token_idx)
{
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t *h = reinterpret_cast<uint32_t *>(smem);
    uint2 *sel = reinterpret_cast<uint2 *>(h + kPassBins);
    uint2 *cand = sel + SURE_CAP;
    uint32_t *bm = reinterpret_cast<uint32_t *>(cand + CAND_CAP);
    __shared__ int scratch[36], res[3], s_count;
    const int u = blockIdx.x, tid = threadIdx.x;   // query unit: query u % T of sequence u / T
    const int n = u / T, jq = u - n * T;
    SeqWork &w = ws[u];
    const int elig = eligible(cu_blocks, q_pos, n, total_blocks, jq);
    const bool use_bitmap = elig <= kBitmapBlocks;
    const int n_words = (elig + 31) / 32;
    if (use_bitmap)
        for (int i = tid; i < n_words; i += blockDim.x) bm[i] = 0u;
    pdl_wait_primary();                             // the lists are complete
    const int n_sure = elig > 0 ? min((int)w.n_sure, SURE_CAP) : 0;
    const uint32_t n_cand = elig > 0 ? w.n_cand : 0u;
    const bool listed = n_cand <= (uint32_t)CAND_CAP;
    const int thr = elig > 0 ? w.thr_bin : -1;
    int r = w.rank;
    if (tid == 0) s_count = 0;
    // all list loads of a thread issued before any is stored
#pragma unroll
    for (int j = 0; j < SURE_CAP / kFinishThreads; ++j) {
        const int i = tid + j * kFinishThreads;
        if (i < n_sure) sel[i] = __ldcg(&w.sure[i]);
    }
    if (listed) {
#pragma unroll
        for (int j = 0; j < CAND_CAP / kFinishThreads; ++j) {
            const uint32_t i = tid + j * kFinishThreads;
            if (i < n_cand) cand[i] = __ldcg(&w.cand[i]);
        }
    }
    __syncthreads();

    if (thr >= 0) {
        const float *sc = scores + (size_t)T * cu_blocks[n] +
                          (size_t)jq * cached_rows(cu_blocks, n, total_blocks);
        // every candidate (order key, block) of the threshold bin: from shared memory, or,
        // when the bin overflowed the list, from the scores themselves
        auto for_cand = [&](auto &&f) {
            if (listed) {
                for (uint32_t i = tid; i < n_cand; i += blockDim.x) {
                    const uint2 c = cand[i];
                    f(c.x, c.y);
                }
            } else {
                for (int i = tid; i < elig; i += blockDim.x) {
                    const uint32_t key = order_key(sc[i]);
                    if ((int)(key >> (32 - HBITS)) == thr) f(key, (uint32_t)i);
                }
            }
        };
        uint32_t kmask = 0xffffffffu << (32 - HBITS), kval = (uint32_t)thr << (32 - HBITS);
        int eq = 0;
        for (int shift = 32 - HBITS - 10; shift >= 0; shift -= 10) {   // bits 19..10, 9..0
            for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0;
            __syncthreads();
            for_cand([&](uint32_t key, uint32_t) {
                if ((key & kmask) == kval) atomicAdd(&h[(key >> shift) & 1023u], 1u);
            });
            __syncthreads();
            find_from_top(h, 1024, r, scratch, res);
            kval |= (uint32_t)res[0] << shift;
            kmask |= 1023u << shift;
            r -= res[1];
            eq = res[2];
            __syncthreads();
        }
        const uint32_t tau = kval;                  // order key of the budget-th best block
        uint32_t iota = 0xffffffffu;                // blocks of key tau kept up to this index
        if (eq > r) {
            // the r smallest block indices among key == tau: radix over the index bits,
            // smallest first (bin nb - 1 - digit, so that "from the top" means smallest)
            uint32_t imask = 0, ival = 0;
            const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
            for (int p = 0; p < 3; ++p) {
                const int nb = 1 << widths[p], sh = shifts[p];
                for (int i = tid; i < nb; i += blockDim.x) h[i] = 0;
                __syncthreads();
                for_cand([&](uint32_t key, uint32_t idx) {
                    if (key == tau && (idx & imask) == ival)
                        atomicAdd(&h[nb - 1 - ((idx >> sh) & (uint32_t)(nb - 1))], 1u);
                });
                __syncthreads();
                find_from_top(h, nb, r, scratch, res);
                ival |= (uint32_t)(nb - 1 - res[0]) << sh;
                imask |= (uint32_t)(nb - 1) << sh;
                r -= res[1];
                __syncthreads();
            }
            iota = ival;
        }
        for_cand([&](uint32_t key, uint32_t idx) {
            if (key > tau || (key == tau && idx <= iota)) {
                if (use_bitmap) {
                    if (idx < (uint32_t)elig) atomicOr(&bm[idx >> 5], 1u << (idx & 31));
                } else {
                    const int slot = n_sure + atomicAdd(&s_count, 1);
                    if (slot < SURE_CAP) sel[slot] = make_uint2(key, idx);
                }
            }
        });
    }
    if (use_bitmap)                                 // (entries are < elig; the test keeps the
        for (int i = tid; i < n_sure; i += blockDim.x) {   //  bitmap in bounds whatever the lists hold)
            const uint32_t idx = sel[i].y;
            if (idx < (uint32_t)elig) atomicOr(&bm[idx >> 5], 1u << (idx & 31));
        }
    __syncthreads();
    int count = min(thr >= 0 ? n_sure + s_count : n_sure, min(budget, SURE_CAP));

    int32_t *bi = block_idx + (size_t)u * budget;
    float *bs = block_score ? block_score + (size_t)u * budget : nullptr;
    int32_t *ti = token_idx ? token_idx + (size_t)u * budget * QR : nullptr;
    auto put = [&](int pos, uint2 e) {             // kept block e at output position pos
        bi[pos] = (int32_t)e.y;
        if (bs) bs[pos] = key_value(e.x);
        if (ti) {
#pragma unroll
            for (int j = 0; j < QR; ++j) ti[pos * QR + j] = (int32_t)(QR * e.y + (uint32_t)j);
        }
    };
    if (use_bitmap) {
        // ordered compaction: thread t owns bitmap words [t per, (t + 1) per)
        const float *sc = scores + (size_t)T * cu_blocks[n] +
                          (size_t)jq * cached_rows(cu_blocks, n, total_blocks);
        const int per = (n_words + blockDim.x - 1) / blockDim.x;
        const int w0 = tid * per, w1 = min(n_words, w0 + per);
        int local = 0;
        for (int i = w0; i < w1; ++i) local += __popc(bm[i]);
        int total;
        int pos = block_exclusive_scan(local, scratch, total);
        count = min(total, min(budget, SURE_CAP));   // the bitmap holds the kept set
        uint32_t *ord = reinterpret_cast<uint32_t *>(sel);   // kept blocks in block order
        for (int i = w0; i < w1; ++i) {
            uint32_t m = bm[i];
            while (m) {
                const int b = __ffs(m) - 1;
                m &= m - 1;
                if (pos < count) ord[pos] = 32u * (uint32_t)i + (uint32_t)b;
                ++pos;
            }
        }
        __syncthreads();
        // one output entry per thread: all score loads in flight at once
        for (int i = tid; i < count; i += blockDim.x) {
            const uint32_t idx = ord[i];
            put(i, make_uint2(order_key(__ldcg(sc + idx)), idx));
        }
    } else {
        int P = 1;
        while (P < count) P <<= 1;
        for (int i = count + tid; i < P; i += blockDim.x) sel[i] = make_uint2(0u, 0xffffffffu);
        __syncthreads();
        for (int kk = 2; kk <= P; kk <<= 1) {
            for (int j = kk >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < P; i += blockDim.x) {
                    const int ij = i ^ j;
                    if (ij > i) {
                        const uint2 a = sel[i], b = sel[ij];
                        const bool up = (i & kk) == 0;
                        if ((a.y > b.y) == up) { sel[i] = b; sel[ij] = a; }
                    }
                }
                __syncthreads();
            }
        }
        for (int i = tid; i < count; i += blockDim.x) put(i, sel[i]);
    }
    for (int i = count + tid; i < budget; i += blockDim.x) {
        bi[i] = -1;
        if (bs) bs[i] = -INFINITY;
        if (ti) {
#pragma unroll
            for (int j = 0; j < QR; ++j) ti[i * QR + j] = -1;
        }
    }
    // leave the record zeroed for the next call
    for (int i = tid; i < HBINS; i += blockDim.x) w.hist[i] = 0;
    if (tid == 0) { w.n_sure = 0; w.n_cand = 0; w.items_done = 0; }
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

}  // namespace

size_t qsa_index_workspace_bytes(int N, long long total_blocks, int T) {
    const size_t rec = (size_t)N * T * sizeof(SeqWork);
    return rec + (((size_t)total_blocks * T * sizeof(float) + 255) / 256) * 256;
}

cudaError_t launch_qsa_compress(const void *k, const int32_t *cu_seqlens, const int32_t *cu_blocks,
                                const int32_t *pos0, void *k_hat, int N, long long total_blocks,
                                float rope_base, cudaStream_t stream) {
    const int rows_per_cta = 256 / 16;
    long long want = (total_blocks + rows_per_cta - 1) / rows_per_cta;
    const long long cap = (long long)sm_count() * 8;
    const int grid = (int)(want < cap ? want : cap);
    qsa_compress_kernel<<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(k), cu_seqlens, cu_blocks, pos0,
        static_cast<__nv_bfloat16 *>(k_hat), N, (int)total_blocks, (double)rope_base);
    return cudaGetLastError();
}

namespace {

// Opt a kernel in to more than 48 KB of dynamic shared memory, once per device.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, PerDevice &once) {
    return once.ensure([&] {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)bytes);
    });
}

template <int T>
PerDevice g_score_setup;
PerDevice g_finish_setup;

template <int T>
cudaError_t launch_score(const void *q, const int32_t *q_pos, const void *k_hat,
                         const int32_t *cu_blocks, int N, long long total_blocks, int budget,
                         float rope_base, SeqWork *ws, float *scores, cudaStream_t stream) {
    const size_t fixed = (size_t)T * (HBINS * sizeof(uint32_t) + QD * sizeof(float));
    const size_t smem = fixed + (size_t)(36 + N + 1) * sizeof(int);
    // the limit is set once per device, so for the largest call (GDN_QSA_MAX_SEQS sequences)
    cudaError_t e = allow_smem(qsa_score_kernel<T>,
                               fixed + (size_t)(36 + GDN_QSA_MAX_SEQS + 1) * sizeof(int),
                               g_score_setup<T>);
    if (e != cudaSuccess) return e;
    qsa_score_kernel<T><<<sm_count() * (T == 1 ? 4 : 2), kScoreThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), q_pos, static_cast<const __nv_bfloat16 *>(k_hat),
        cu_blocks, N, (int)total_blocks, budget, (double)rope_base, ws, scores);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qsa_index(const void *q, const int32_t *q_pos, const void *k_hat,
                             const int32_t *cu_blocks, int N, long long total_blocks, int T,
                             int budget, float rope_base, int32_t *block_idx,
                             float *block_score, int32_t *token_idx, void *workspace,
                             cudaStream_t stream) {
    SeqWork *ws = static_cast<SeqWork *>(workspace);
    float *scores = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) +
                                              (size_t)N * T * sizeof(SeqWork));
    cudaError_t e;
    switch (T) {
    case 1: e = launch_score<1>(q, q_pos, k_hat, cu_blocks, N, total_blocks, budget, rope_base, ws, scores, stream); break;
    case 2: e = launch_score<2>(q, q_pos, k_hat, cu_blocks, N, total_blocks, budget, rope_base, ws, scores, stream); break;
    case 3: e = launch_score<3>(q, q_pos, k_hat, cu_blocks, N, total_blocks, budget, rope_base, ws, scores, stream); break;
    case 4: e = launch_score<4>(q, q_pos, k_hat, cu_blocks, N, total_blocks, budget, rope_base, ws, scores, stream); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count() * 4);
    cfg.blockDim = dim3(kScoreThreads);
    cfg.dynamicSmemBytes = (size_t)(36 + N * T + 1) * sizeof(int);
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, qsa_collect_kernel, q_pos, cu_blocks, N, T, (int)total_blocks,
                           (const float *)scores, ws);
    if (e != cudaSuccess) return e;
    if ((e = allow_smem(qsa_finish_kernel, kFinishSmem, g_finish_setup)) != cudaSuccess) return e;
    cfg.gridDim = dim3(N * T);
    cfg.blockDim = dim3(kFinishThreads);
    cfg.dynamicSmemBytes = kFinishSmem;
    return cudaLaunchKernelEx(&cfg, qsa_finish_kernel, q_pos, cu_blocks, T, (int)total_blocks,
                              budget, (const float *)scores, ws, block_idx, block_score,
                              token_idx);
}

}  // namespace gdn
