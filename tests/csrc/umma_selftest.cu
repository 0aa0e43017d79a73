// Unit checks of the sm_100a primitives the tensor-core prefill is built from
// (test infrastructure; built by tests/selftest_lib.py, used by tests only).
//
//  selftest_umma: one 128 x N x K product D = A B^T through tcgen05.mma with
//    operands placed in 128-byte-swizzled shared memory as K-major or MN-major
//    tiles (the placements the prefill kernel uses), read back from TMEM.
//  selftest_tma:  one 64-token x 128-element tile of a [T, H, 128] bf16 tensor
//    loaded by TMA (two 128-byte boxes, 128-byte swizzle) and un-swizzled with
//    the same formula the prefill kernel uses for its own shared-memory writes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../linear_attention_token_b200/csrc/sm100.cuh"

using namespace gdn::sm100;

namespace {

constexpr int ST_THREADS = 128;

// variant bits: 1 = A MN-major, 2 = B MN-major, 4 = negate B, 8 = N=128 (else 64),
//               16 = K=128 (else 64), 32 = M=64, 64 = N=32,
//               128 = B MN-major with 64-byte swizzle (with N=32: one 64-byte row per k)
__global__ void __launch_bounds__(ST_THREADS, 1)
umma_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int variant, int *status)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const bool a_mn = variant & 1, b_sw64 = variant & 128, b_mn = (variant & 2) || b_sw64, neg = variant & 4;
    const int M = (variant & 32) ? 64 : 128;
    const int N = (variant & 64) ? 32 : ((variant & 8) ? 128 : 64);
    const int K = (variant & 16) ? 128 : 64;
    unsigned char *As = base;                  // up to 32 KB
    unsigned char *Bs = base + 32768;          // up to 32 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (warp == 0) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }
    if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }

    // place A (logical M x K, row-major in global)
    for (int e = tid; e < M * K / 8; e += ST_THREADS) {
        uint4 val;
        __nv_bfloat16 *pv = reinterpret_cast<__nv_bfloat16 *>(&val);
        if (!a_mn) {                       // rows m, 16-B chunk c of k-block cg
            const int m = e / (K / 8), kc = e % (K / 8), cg = kc / 8, c = kc % 8;
            for (int i = 0; i < 8; ++i) pv[i] = A[m * K + cg * 64 + c * 8 + i];
            *reinterpret_cast<uint4 *>(As + cg * (M * 128) + sw128(m, c)) = val;
        } else {                           // rows k, 16-B chunk c of m-block blk
            const int k = e / (M / 8), mc = e % (M / 8), blk = mc / 8, c = mc % 8;
            for (int i = 0; i < 8; ++i) pv[i] = A[(blk * 64 + c * 8 + i) * K + k];
            *reinterpret_cast<uint4 *>(As + blk * (K * 128) + sw128(k, c)) = val;
        }
    }
    // place B (logical N x K, row-major in global)
    for (int e = tid; e < N * K / 8; e += ST_THREADS) {
        uint4 val;
        __nv_bfloat16 *pv = reinterpret_cast<__nv_bfloat16 *>(&val);
        if (b_sw64) {                      // rows k of 32 elements, 16-B chunk c
            const int k = e / 4, c = e % 4;
            for (int i = 0; i < 8; ++i) pv[i] = B[(c * 8 + i) * K + k];
            *reinterpret_cast<uint4 *>(Bs + sw64(k, c)) = val;
        } else if (!b_mn) {
            const int n = e / (K / 8), kc = e % (K / 8), cg = kc / 8, c = kc % 8;
            for (int i = 0; i < 8; ++i) pv[i] = B[n * K + cg * 64 + c * 8 + i];
            *reinterpret_cast<uint4 *>(Bs + cg * (N * 128) + sw128(n, c)) = val;
        } else {
            const int k = e / (N / 8), nc = e % (N / 8), blk = nc / 8, c = nc % 8;
            for (int i = 0; i < 8; ++i) pv[i] = B[(blk * 64 + c * 8 + i) * K + k];
            *reinterpret_cast<uint4 *>(Bs + blk * (K * 128) + sw128(k, c)) = val;
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_base;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_mn, b_mn, neg);
        for (int s = 0; s < K / 16; ++s) {
            const uint32_t a_addr = a_mn ? smem_u32(As) + s * 2048
                                         : smem_u32(As) + (s / 4) * (M * 128) + (s % 4) * 32;
            const uint32_t b_addr = b_sw64 ? smem_u32(Bs) + s * 1024
                                  : b_mn ? smem_u32(Bs) + s * 2048
                                         : smem_u32(Bs) + (s / 4) * (N * 128) + (s % 4) * 32;
            const uint64_t ad = a_mn ? sdesc_mnmajor(a_addr, K * 128) : sdesc_kmajor(a_addr);
            const uint64_t bd = b_sw64 ? sdesc_mn_sw64(b_addr)
                              : b_mn ? sdesc_mnmajor(b_addr, K * 128) : sdesc_kmajor(b_addr);
            umma_bf16(tm, ad, bd, id, s > 0);
        }
        umma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0, 1u << 20);
    if (!ok && tid == 0) atomicExch(status, 4);
    tc_fence_after();
    // warp w reads lanes 32w..32w+31.  M = 128: lane = row.  M = 64: rows 16w..16w+15
    // sit in lanes 32w..32w+15 (the other 16 lanes of each quadrant are not written).
    const int l = tid & 31;
    const int m = (M == 128) ? warp * 32 + l : warp * 16 + l;
    const bool has_row = (M == 128) || l < 16;
    for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tm + ((uint32_t)(warp * 32) << 16) + c0, r);
        tmem_wait_ld();
        if (has_row)
            for (int j = 0; j < 32; ++j) D[m * N + c0 + j] = __uint_as_float(r[j]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 128);
}

__global__ void tma_kernel(const __grid_constant__ CUtensorMap map, int h, int t0,
                           __nv_bfloat16 *out, int *status)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar, 2 * 8192);
        tma_load_3d(base, &map, &bar, 0, h, t0);
        tma_load_3d(base + 8192, &map, &bar, 64, h, t0);
    }
    __syncthreads();
    if (!mbar_wait(&bar, 0, 1u << 20)) { if (tid == 0) atomicExch(status, 4); return; }
    for (int e = tid; e < 64 * 16; e += blockDim.x) {
        const int r = e / 16, kc = e % 16, cg = kc / 8, c = kc % 8;
        const uint4 val = *reinterpret_cast<const uint4 *>(base + cg * 8192 + sw128(r, c));
        *reinterpret_cast<uint4 *>(out + r * 128 + cg * 64 + c * 8) = val;
    }
}

// Four CTAs of one cluster: each fills 16 KB with a pattern, copies it into the next
// CTA's shared memory with a bulk copy that completes on that CTA's mbarrier, pings the
// next CTA's second mbarrier with a remote arrive, and checks what it received.
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(128, 1)
cluster_kernel(int *out)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t recv_bar, ping_bar;
    uint32_t *sendbuf = reinterpret_cast<uint32_t *>(base);
    uint32_t *recvbuf = reinterpret_cast<uint32_t *>(base + 16384);
    const int tid = threadIdx.x;
    const uint32_t rank = cluster_rank();
    const uint32_t next = (rank + 1) & 3, prev = (rank + 3) & 3;
    for (int i = tid; i < 4096; i += blockDim.x) { sendbuf[i] = rank * 100000u + i; recvbuf[i] = 0xdeadbeefu; }
    if (tid == 0) {
        mbar_init(&recv_bar, 1);
        mbar_init(&ping_bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&recv_bar, 16384);          // expect one 16 KB copy
    }
    fence_proxy_async();
    cluster_sync();                                        // barriers and buffers ready everywhere
    if (tid == 0) {
        bulk_copy_to_cluster(map_to_rank(recvbuf, next), sendbuf, 16384, map_to_rank(&recv_bar, next));
        mbar_arrive_remote(map_to_rank(&ping_bar, next));
    }
    const bool ok1 = mbar_wait_cluster(&recv_bar, 0, 1u << 20);
    const bool ok2 = mbar_wait_cluster(&ping_bar, 0, 1u << 20);
    int bad = (!ok1 || !ok2) ? 1 : 0;
    if (ok1)
        for (int i = tid; i < 4096; i += blockDim.x)
            if (recvbuf[i] != prev * 100000u + i) bad = 2;
    bad = __syncthreads_or(bad);
    if (tid == 0) out[blockIdx.x] = bad ? (ok1 && ok2 ? 2 : 1) : 0;
    cluster_sync();                                        // nobody leaves while others may copy
}

// Timing probe: `reps` rounds of `nmma` MMAs of one placement, each round committed and
// waited for; records clock64 per round (issue of the first MMA to completion seen).
__global__ void __launch_bounds__(128, 1)
umma_timing_kernel(int variant, int nmma, int reps, long long *cycles, int streams)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const bool a_mn = variant & 1, b_mn = variant & 2;
    const int M = (variant & 32) ? 64 : 128;
    const int N = (variant & 64) ? 32 : ((variant & 8) ? 128 : 64);
    unsigned char *As = base, *Bs = base + 65536;
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < 32768; i += 128) reinterpret_cast<uint32_t *>(base)[i] = 0x3c003c00u;
    if (warp == 0) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
    if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_mn, b_mn, false);
        for (int rep = 0; rep < reps; ++rep) {
            const long long t0 = clock64();
            for (int s = 0; s < nmma; ++s) {
                const uint32_t ks = s & 7;
                const uint32_t a_addr = a_mn ? smem_u32(As) + ks * 2048 : smem_u32(As) + (ks / 4) * (M * 128) + (ks % 4) * 32;
                const uint32_t b_addr = b_mn ? smem_u32(Bs) + ks * 2048 : smem_u32(Bs) + (ks / 4) * (N * 128) + (ks % 4) * 32;
                const uint64_t ad = a_mn ? sdesc_mnmajor(a_addr, 16384) : sdesc_kmajor(a_addr);
                const uint64_t bd = b_mn ? sdesc_mnmajor(b_addr, 16384) : sdesc_kmajor(b_addr);
                // `streams` independent accumulators, used round-robin
                const int st = s % streams;
                umma_bf16(tmem_base + st * N, ad, bd, id, s >= streams);
            }
            umma_commit(&bar);
            mbar_wait(&bar, rep & 1, 1u << 22);
            cycles[rep] = clock64() - t0;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

// Timing probe with compile-time shape: NMMA MMAs (M x N x 16, both operands K-major),
// descriptors precomputed, fully unrolled; D accumulates in place.
template <int M, int N, int NMMA>
__global__ void __launch_bounds__(128, 1) umma_timing2_kernel(int reps, long long *cycles)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *As = base, *Bs = base + 65536;
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < 32768; i += 128) reinterpret_cast<uint32_t *>(base)[i] = 0x3c003c00u;
    if (warp == 0) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
    if (tid == 0) { mbar_init(&bar, 1); fence_mbar_init(); }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        constexpr uint32_t id = idesc_bf16(M, N, false, false, false);
        uint64_t ad[8], bd[8];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            ad[ks] = sdesc_kmajor(smem_u32(As) + (ks / 4) * (M * 128) + (ks % 4) * 32);
            bd[ks] = sdesc_kmajor(smem_u32(Bs) + (ks / 4) * (N * 128) + (ks % 4) * 32);
        }
        const uint32_t d = tmem_base;
        for (int rep = 0; rep < reps; ++rep) {
            const long long t0 = clock64();
#pragma unroll
            for (int s2 = 0; s2 < NMMA; ++s2) umma_bf16(d, ad[s2 & 7], bd[s2 & 7], id, s2 > 0);
            umma_commit(&bar);
            mbar_wait(&bar, rep & 1, 1u << 22);
            cycles[rep] = clock64() - t0;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

// Timing probe: one TMA tile load of `boxes` boxes (64 tokens x 128 B each) of a
// [T, H, 128] bf16 tensor, issue to completion seen, repeated `reps` times.
__global__ void tma_timing_kernel(const __grid_constant__ CUtensorMap map, int boxes, int reps,
                                  int stride_tokens, long long *cycles)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        for (int rep = 0; rep < reps; ++rep) {
            const long long t0 = clock64();
            mbar_arrive_expect_tx(&bar, boxes * 8192);
            for (int b = 0; b < boxes; ++b)
                tma_load_3d(base + b * 8192, &map, &bar, (b & 1) * 64, (b >> 1), rep * stride_tokens);
            mbar_wait(&bar, rep & 1, 1u << 22);
            cycles[rep] = clock64() - t0;
        }
    }
}


// Contention probe: warp 0's first lane issues 8 MMAs (M=64, N=32, K=128; A K-major,
// B in 64-byte rows) and waits for them, `reps` times, recording each round's cycles
// and the cycles of one try_wait on an already-completed barrier.  Meanwhile warps 1..15
// run bounded background loops: mode 0 none, 1 FMA chains, 2 shared-memory load/store,
// 3 both.  The background stops after a fixed iteration count (no flag waits).
__global__ void __launch_bounds__(512, 1)
contention_kernel(int mode, int reps, int bg_iters, long long *cycles)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *As = base, *Bs = base + 16384, *scratch = base + 32768;   // scratch 64 KB
    __shared__ uint64_t bar, done_bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < (32768 + 65536) / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(base)[i] = 0x3c003c00u;
    if (warp == 0) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }
    if (tid == 0) { mbar_init(&bar, 1); mbar_init(&done_bar, 1); fence_mbar_init(); mbar_arrive_local(&done_bar); }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(64, 32, false, true);
            const uint64_t da = sdesc_kmajor(smem_u32(As)), db = sdesc_mn_sw64(smem_u32(Bs));
            for (int rep = 0; rep < reps; ++rep) {
                const long long t0 = clock64();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_bf16(tmem_base, da + (ks >> 2) * 512 + (ks & 3) * 2, db + ks * 64, id, ks > 0);
                const long long t1 = clock64();
                umma_commit(&bar);
                mbar_wait(&bar, rep & 1, 1u << 22);
                const long long t2 = clock64();
                const bool okw = mbar_try_wait(&done_bar, 0);       // phase 0 completed at setup
                const long long t3 = clock64();
                cycles[3 * rep] = t1 - t0;
                cycles[3 * rep + 1] = t2 - t0;
                cycles[3 * rep + 2] = okw ? t3 - t2 : -1;
                // spread the rounds over the background's run
                for (int w = 0; w < 200; ++w) __nanosleep(20);
            }
        }
    } else if (mode != 0) {
        float a = lane * 0.001f, b = 1.0001f, c2 = 0.9999f, d = 0.5f;
        uint4 *sp = reinterpret_cast<uint4 *>(scratch) + ((warp * 32 + lane) & 4095);
        uint4 acc = make_uint4(0, 0, 0, 0);
        for (int it = 0; it < bg_iters; ++it) {
            if (mode & 1) {
#pragma unroll
                for (int u = 0; u < 16; ++u) { a = fmaf(a, b, c2); d = fmaf(d, c2, b); }
            }
            if (mode & 2) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 v = sp[(u * 512) & 4095];
                    acc.x ^= v.x; acc.y += v.y;
                    sp[((u * 512) + 64) & 4095] = acc;
                }
            }
        }
        if (a == 12345.f && d == 1.f && acc.x == 7) cycles[0] = 0;    // keep the work
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 128);
}

// DSMEM bandwidth probe: in a cluster of 4, CTA 0 copies `bytes` (a multiple of 4096,
// at most 57344) from its shared memory into the same offset of each destination CTA
// (mask bit d = CTA d) with 4 KB bulk copies completing on the destination's barrier;
// each destination then arrives on CTA 0's ack barrier.  Records the cycles from the
// first copy to the last ack, `reps` times.
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(128, 1)
dsmem_bw_kernel(int bytes, int mask, int reps, long long *cycles)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t recv_bar, ack_bar;
    const int tid = threadIdx.x;
    const uint32_t rank = cluster_rank();
    int ndst = 0;
    for (int d = 0; d < 4; ++d) ndst += (mask >> d) & 1;
    for (int i = tid; i < 57344 / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(base)[i] = rank + i;
    if (tid == 0) {
        mbar_init(&recv_bar, 1);
        mbar_init(&ack_bar, ndst);
        fence_mbar_init();
    }
    fence_proxy_async();
    cluster_sync();
    for (int rep = 0; rep < reps; ++rep) {
        const bool is_dst = (mask >> rank) & 1;
        if (tid == 0 && is_dst) mbar_arrive_expect_tx(&recv_bar, (uint32_t)bytes);
        cluster_sync();                            // every destination armed
        long long t0 = 0;
        if (rank == 0 && tid == 0) {
            t0 = clock64();
            for (int d = 0; d < 4; ++d) {
                if (!((mask >> d) & 1)) continue;
                const uint32_t bar = map_to_rank(&recv_bar, (uint32_t)d);
                for (int off = 0; off < bytes; off += 4096)
                    bulk_copy_to_cluster(map_to_rank(base + 65536 + off, (uint32_t)d), base + off, 4096, bar);
            }
        }
        if (tid == 0 && is_dst) {
            mbar_wait_cluster(&recv_bar, rep & 1, 1u << 22);
            mbar_arrive_remote(map_to_rank(&ack_bar, 0));
        }
        if (rank == 0 && tid == 0) {
            mbar_wait_cluster(&ack_bar, rep & 1, 1u << 22);
            cycles[rep] = clock64() - t0;
        }
        cluster_sync();
    }
}

// Data-movement probe, one cluster of 4 CTAs; CTA 0's thread 0 records cycles for:
//  [0] bulk store of `bytes` smem -> global: issue to wait_group.read
//  [1]   ... to wait_group (writes complete)
//  [2] bulk load of `bytes` global -> smem (the data just stored, L2-resident)
//  [3] 4 remote mbarrier arrives (release.cluster), one to each CTA
//  [4] 4 remote mbarrier arrives (relaxed.cluster)
//  [5] bulk load of `bytes` from a cold region (likely HBM)
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(128, 1)
movement_kernel(unsigned char *gbuf, int bytes, int reps, long long *cycles)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t ld_bar, ping_bar;
    const int tid = threadIdx.x;
    const uint32_t rank = cluster_rank();
    for (int i = tid; i < 2 * 65536 / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(base)[i] = i;
    if (tid == 0) { mbar_init(&ld_bar, 1); mbar_init(&ping_bar, 1); fence_mbar_init(); }
    fence_proxy_async();
    cluster_sync();
    if (rank == 0 && tid == 0) {
        for (int rep = 0; rep < reps; ++rep) {
            long long *cy = cycles + 6 * rep;
            unsigned char *g = gbuf + (size_t)(rep & 1) * 65536;
            long long t0 = clock64();
            bulk_store_global(g, base, (uint32_t)bytes);
            bulk_commit();
            bulk_wait_read_all();
            long long t1 = clock64();
            bulk_wait_all();
            long long t2 = clock64();
            cy[0] = t1 - t0; cy[1] = t2 - t0;
            fence_proxy_async_global();
            t0 = clock64();
            mbar_arrive_expect_tx(&ld_bar, (uint32_t)bytes);
            bulk_load_global(base + 65536, g, (uint32_t)bytes, &ld_bar);
            mbar_wait(&ld_bar, (uint32_t)(2 * rep) & 1, 1u << 22);
            cy[2] = clock64() - t0;
            t0 = clock64();
            for (uint32_t d = 0; d < 4; ++d) mbar_arrive_remote(map_to_rank(&ping_bar, d));
            cy[3] = clock64() - t0;
            t0 = clock64();
            for (uint32_t d = 0; d < 4; ++d) mbar_arrive_remote_relaxed(map_to_rank(&ping_bar, d));
            cy[4] = clock64() - t0;
            unsigned char *cold = gbuf + 131072 + (size_t)rep * 65536;
            t0 = clock64();
            mbar_arrive_expect_tx(&ld_bar, (uint32_t)bytes);
            bulk_load_global(base + 65536, cold, (uint32_t)bytes, &ld_bar);
            mbar_wait(&ld_bar, (uint32_t)(2 * rep + 1) & 1, 1u << 22);
            cy[5] = clock64() - t0;
        }
    }
    cluster_sync();
}
}  // namespace

extern "C" __attribute__((visibility("default")))
int selftest_umma_timing(int variant, int nmma, int reps, long long *cycles, int streams)
{
    const int smem = 131072 + 1024;
    cudaFuncSetAttribute(umma_timing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    umma_timing_kernel<<<1, 128, smem>>>(variant, nmma, reps, cycles, streams);
    return (int)cudaDeviceSynchronize();
}

#define GDN_T2(Mv, Nv, Kn)                                                                   \
    if (M == Mv && N == Nv && nmma == Kn) {                                                  \
        cudaFuncSetAttribute(umma_timing2_kernel<Mv, Nv, Kn>,                                \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);              \
        umma_timing2_kernel<Mv, Nv, Kn><<<1, 128, smem>>>(reps, cycles);                      \
        return (int)cudaDeviceSynchronize();                                                 \
    }
extern "C" __attribute__((visibility("default")))
int selftest_umma_timing2(int M, int N, int nmma, int reps, long long *cycles)
{
    const int smem = 131072 + 1024;
    GDN_T2(128, 256, 8) GDN_T2(128, 256, 32) GDN_T2(128, 128, 8) GDN_T2(128, 128, 32)
    GDN_T2(128, 64, 8) GDN_T2(128, 64, 32) GDN_T2(128, 32, 8) GDN_T2(128, 32, 32)
    GDN_T2(64, 32, 8) GDN_T2(64, 32, 32) GDN_T2(64, 128, 32) GDN_T2(128, 256, 1) GDN_T2(128, 32, 1)
    return -1;
}

extern "C" __attribute__((visibility("default")))
int selftest_tma_timing(const void *src, int T, int H, int boxes, int reps, int stride_tokens,
                        long long *cycles)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", (void **)&encode, cudaEnableDefault, &q)
            != cudaSuccess || !encode)
        return -1;
    CUtensorMap map;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(src), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return -2;
    const int smem = 65536 + 1024;
    cudaFuncSetAttribute(tma_timing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    tma_timing_kernel<<<1, 32, smem>>>(map, boxes, reps, stride_tokens, cycles);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default")))
int selftest_cluster(int *out)
{
    const int smem = 32768 + 1024;
    cudaFuncSetAttribute(cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cluster_kernel<<<8, 128, smem>>>(out);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default")))
int selftest_umma(const void *A, const void *B, float *D, int variant, int *status)
{
    const int smem = 64 * 1024 + 1024;
    cudaFuncSetAttribute(umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    umma_kernel<<<1, ST_THREADS, smem>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, D,
                                          variant, status);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default")))
int selftest_tma(const void *src, int T, int H, int h, int t0, void *out, int *status)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", (void **)&encode, cudaEnableDefault, &q)
            != cudaSuccess || !encode)
        return -1;
    CUtensorMap map;
    cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)H * 128 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(src), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return -2;
    const int smem = 16384 + 1024;
    cudaFuncSetAttribute(tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    tma_kernel<<<1, 128, smem>>>(map, h, t0, (__nv_bfloat16 *)out, status);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default")))
int selftest_contention(int mode, int reps, int bg_iters, long long *cycles)
{
    const int smem = 32768 + 65536 + 1024;
    cudaFuncSetAttribute(contention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    contention_kernel<<<1, 512, smem>>>(mode, reps, bg_iters, cycles);
    return (int)cudaDeviceSynchronize();
}

extern "C" __attribute__((visibility("default")))
int selftest_dsmem_bw(int bytes, int mask, int reps, long long *cycles)
{
    if (bytes <= 0 || bytes > 57344 || bytes % 4096 != 0 || (mask & 15) == 0) return -1;
    const int smem = 65536 + 57344 + 1024;
    cudaFuncSetAttribute(dsmem_bw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dsmem_bw_kernel<<<4, 128, smem>>>(bytes, mask & 15, reps, cycles);
    return (int)cudaDeviceSynchronize();
}

// gbuf: at least 131072 + reps * 65536 bytes of device memory
extern "C" __attribute__((visibility("default")))
int selftest_movement(void *gbuf, int bytes, int reps, long long *cycles)
{
    if (bytes <= 0 || bytes > 65536 || bytes % 16 != 0) return -1;
    const int smem = 2 * 65536 + 1024;
    cudaFuncSetAttribute(movement_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    movement_kernel<<<4, 128, smem>>>((unsigned char *)gbuf, bytes, reps, cycles);
    return (int)cudaDeviceSynchronize();
}
