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
//               128 = B MN-major with 64-byte swizzle (with N=32: one 64-byte row per k),
//               256 = A read from TMEM (M = 128, K-major) instead of shared memory
__global__ void __launch_bounds__(ST_THREADS, 1)
umma_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int variant, int *status)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const bool a_mn = variant & 1, b_sw64 = variant & 128, b_mn = (variant & 2) || b_sw64, neg = variant & 4;
    const bool a_tm = variant & 256;
    const int M = (variant & 32) ? 64 : 128;
    const int N = (variant & 64) ? 32 : ((variant & 8) ? 128 : 64);
    const int K = (variant & 16) ? 128 : 64;
    unsigned char *As = base;                  // up to 32 KB
    unsigned char *Bs = base + 32768;          // up to 32 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (warp == 0) { tmem_alloc(&tmem_base, 256); tmem_relinquish(); }
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
    if (a_tm) {                            // row tid of A into lane tid, columns 128..
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
            for (int j = 0; j < 16; ++j) {
                const __nv_bfloat162 pr = __halves2bfloat162(A[tid * K + 2 * (c0 + j)],
                                                             A[tid * K + 2 * (c0 + j) + 1]);
                r[j] = *reinterpret_cast<const uint32_t *>(&pr);
            }
            tmem_st16(tm + ((uint32_t)(warp * 32) << 16) + 128 + c0, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
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
            if (a_tm) umma_bf16_ta(tm, tm + 128 + s * 8, bd, id, s > 0);
            else umma_bf16(tm, ad, bd, id, s > 0);
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
    if (warp == 0) tmem_dealloc(tm, 256);
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

}  // namespace




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



