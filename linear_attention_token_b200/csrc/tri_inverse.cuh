// T = (I + A)^-1 for a 64 x 64 strictly lower triangular A, in fp32 on the CUDA
// cores, by 256 threads of one CTA.  This is the per-chunk triangular solve of the
// chunked gated delta rule: with A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i), the
// chunk's write vectors satisfy (I + A) U = diag(beta) V - diag(beta gamma) K S.
//
// Block algorithm (16 x 16 blocks, B_ij of A, D_i of T):
//   1. D_i = (I + A_ii)^-1 for the four diagonal blocks, one thread per column,
//      by forward substitution in registers;
//   2. 16 -> 32:  T_10 = -D_1 (A_10 D_0),  T_32 = -D_3 (A_32 D_2);
//   3. 32 -> 64:  T_HL = -D_H (A_HL D_L)  with the 32 x 32 blocks L = [0,32), H = [32,64).
// This is the 2 x 2 block inverse [[X, 0], [Y, Z]]^-1 = [[X^-1, 0], [-Z^-1 Y X^-1, Z^-1]]
// applied twice.  Layout: row-major with pitch TP (65 floats).  On entry T holds the
// identity (its strict upper triangle must be zero and stays zero); the strict upper
// triangle of A is used as scratch and is overwritten.  The caller synchronises the
// CTA before (A and T written) and after (T read).
#pragma once

namespace gdn {

template <int TP>
__device__ __forceinline__ void invert_unit_lower_64(float *A, float *T, int tid)
{
    // 1. diagonal blocks: thread (b, col) owns column col of D_b
    if (tid < 64) {
        const int b = tid >> 4, col = tid & 15;
        const float *Ab = A + (16 * b) * TP + 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int m = 0; m + 1 < r; m += 2) {
                acc0 = fmaf(Ab[r * TP + m], x[m], acc0);
                acc1 = fmaf(Ab[r * TP + m + 1], x[m + 1], acc1);
            }
            if (r & 1) acc0 = fmaf(Ab[r * TP + r - 1], x[r - 1], acc0);
            x[r] = (r == col) ? 1.f : ((r < col) ? 0.f : -(acc0 + acc1));
        }
        float *Tb = T + (16 * b) * TP + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * TP + col] = x[r];
    }
    __syncthreads();

    // 2. two 16 -> 32 merges; thread: merge p, row r, columns c0, c0 + 1
    {
        const int p = tid >> 7, r = (tid >> 3) & 15, c0 = (tid & 7) * 2;
        const int lo = 32 * p, hi = lo + 16;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float a = A[(hi + r) * TP + lo + m];
            x0 = fmaf(a, T[(lo + m) * TP + lo + c0], x0);
            x1 = fmaf(a, T[(lo + m) * TP + lo + c0 + 1], x1);
        }
        A[(lo + r) * TP + hi + c0] = x0;            // scratch: block (lo, hi) of A's upper part
        A[(lo + r) * TP + hi + c0 + 1] = x1;
        __syncthreads();
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float d = T[(hi + r) * TP + hi + m];
            y0 = fmaf(d, A[(lo + m) * TP + hi + c0], y0);
            y1 = fmaf(d, A[(lo + m) * TP + hi + c0 + 1], y1);
        }
        T[(hi + r) * TP + lo + c0] = -y0;
        T[(hi + r) * TP + lo + c0 + 1] = -y1;
    }
    __syncthreads();

    // 3. the 32 -> 64 merge; thread: rows r0, r0 + 1 and columns c0, c0 + 1 of 32 x 32
    {
        const int r0 = (tid >> 4) * 2, c0 = (tid & 15) * 2;
        float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            const float a0 = A[(32 + r0) * TP + m], a1 = A[(33 + r0) * TP + m];
            const float d0 = T[m * TP + c0], d1 = T[m * TP + c0 + 1];
            x00 = fmaf(a0, d0, x00); x01 = fmaf(a0, d1, x01);
            x10 = fmaf(a1, d0, x10); x11 = fmaf(a1, d1, x11);
        }
        // scratch: rows 0..31, columns 32..63 of A (strictly above the diagonal)
        A[r0 * TP + 32 + c0] = x00; A[r0 * TP + 33 + c0] = x01;
        A[(r0 + 1) * TP + 32 + c0] = x10; A[(r0 + 1) * TP + 33 + c0] = x11;
        __syncthreads();
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            const float d0 = T[(32 + r0) * TP + 32 + m], d1 = T[(33 + r0) * TP + 32 + m];
            const float x0 = A[m * TP + 32 + c0], x1 = A[m * TP + 33 + c0];
            y00 = fmaf(d0, x0, y00); y01 = fmaf(d0, x1, y01);
            y10 = fmaf(d1, x0, y10); y11 = fmaf(d1, x1, y11);
        }
        T[(32 + r0) * TP + c0] = -y00; T[(32 + r0) * TP + c0 + 1] = -y01;
        T[(33 + r0) * TP + c0] = -y10; T[(33 + r0) * TP + c0 + 1] = -y11;
    }
}

// ---------------------------------------------------------------------------------
// Same result with the two merge levels on the warp-level tensor cores (mma.sync
// m16n8k8, tf32 operands, fp32 accumulate).  Used where T is rounded to bf16
// afterwards anyway (tf32 keeps 10 mantissa bits, bf16 7), so the merges cost a few
// dozen MMAs instead of ~65k fp32 FMAs through shared memory.

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One warp: C[16 x 16] = X[16 x K] Y[K x 16]; X, Y, C row-major with pitch TP.
// Writes C * sign.
template <int TP, int K>
__device__ __forceinline__ void warp_gemm_16x16(const float *X, const float *Y, float *C,
                                                float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float acc[2][4] = {};
#pragma unroll
    for (int kk = 0; kk < K; kk += 8) {
        uint32_t a[4];
        a[0] = to_tf32(X[g * TP + kk + t]);
        a[1] = to_tf32(X[(g + 8) * TP + kk + t]);
        a[2] = to_tf32(X[g * TP + kk + t + 4]);
        a[3] = to_tf32(X[(g + 8) * TP + kk + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b[2];
            b[0] = to_tf32(Y[(kk + t) * TP + nt * 8 + g]);
            b[1] = to_tf32(Y[(kk + t + 4) * TP + nt * 8 + g]);
            mma_16x8x8_tf32(acc[nt], a, b);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        C[g * TP + nt * 8 + 2 * t] = sign * acc[nt][0];
        C[g * TP + nt * 8 + 2 * t + 1] = sign * acc[nt][1];
        C[(g + 8) * TP + nt * 8 + 2 * t] = sign * acc[nt][2];
        C[(g + 8) * TP + nt * 8 + 2 * t + 1] = sign * acc[nt][3];
    }
}

// Blocked inverse with tf32 tensor-core merges, run by one warpgroup (t = 0..127) that
// synchronises with `sync()` (a named barrier over exactly those threads):
//   1. the four diagonal 16 x 16 blocks by forward substitution in fp32 (one thread per
//      column of a block);
//   2. 16 -> 32: warp p merges blocks (2p, 2p+1), T_HL = -T_HH A_HL T_LL, with the
//      product A_HL T_LL kept in A's upper block (lo, hi) as scratch;
//   3. 32 -> 64: warp w < 4 owns quadrant (w >> 1, w & 1) of the lower-left 32 x 32 block,
//      with A_HL T_LL kept in rows 0..31, columns 32..63 of A.
template <int TP, typename Sync>
__device__ __forceinline__ void invert_unit_lower_64_tf32_wg(float *A, float *T, int t, Sync sync)
{
    const int warp = t >> 5, lane = t & 31;
    if (t < 64) {
        const int b = t >> 4, col = t & 15;
        const float *Ab = A + (16 * b) * TP + 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int m = 0; m + 1 < r; m += 2) {
                acc0 = fmaf(Ab[r * TP + m], x[m], acc0);
                acc1 = fmaf(Ab[r * TP + m + 1], x[m + 1], acc1);
            }
            if (r & 1) acc0 = fmaf(Ab[r * TP + r - 1], x[r - 1], acc0);
            x[r] = (r == col) ? 1.f : ((r < col) ? 0.f : -(acc0 + acc1));
        }
        float *Tb = T + (16 * b) * TP + 16 * b;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * TP + col] = x[r];
    }
    sync();
    if (warp < 2) {
        const int lo = 32 * warp, hi = lo + 16;
        warp_gemm_16x16<TP, 16>(A + hi * TP + lo, T + lo * TP + lo, A + lo * TP + hi, 1.f, lane);
        __syncwarp();
        warp_gemm_16x16<TP, 16>(T + hi * TP + hi, A + lo * TP + hi, T + hi * TP + lo, -1.f, lane);
    }
    sync();
    {
        const int mb = (warp >> 1) * 16, nb = (warp & 1) * 16;
        warp_gemm_16x16<TP, 32>(A + (32 + mb) * TP, T + nb, A + mb * TP + 32 + nb, 1.f, lane);
        sync();
        warp_gemm_16x16<TP, 32>(T + (32 + mb) * TP + 32, A + 32 + nb, T + (32 + mb) * TP + nb, -1.f, lane);
    }
}

}  // namespace gdn

namespace gdn {

// ---------------------------------------------------------------------------------
// T = (I + A)^-1 for a 64 x 64 strictly lower triangular A, by one warpgroup (t = 0..127)
// with every warp busy at each level and no cross-warp dependency inside a level:
//   1. warp w inverts diagonal block w (16 x 16) in registers, one lane per column,
//      right-looking: once x_m is final, A[r][m] x_m is added to every later row r, so
//      the dependent path is 16 FMAs long;
//   2. 16 -> 32: warp w forms columns [8 (w & 1), +8) of T_HL = -D_H (A_HL D_L) for the
//      block pair p = w >> 1 (H = 2p + 1, L = 2p);
//   3. 32 -> 64: warp w forms columns [8w, 8w + 8) of T_HL = -T_HH (A_HL T_LL) with the
//      32 x 32 halves L = [0, 32), H = [32, 64).
// Levels 2 and 3 run on the warp-level tensor cores (mma.sync m16n8k8, tf32 operands,
// fp32 accumulate): T is rounded to bf16 afterwards, and tf32 keeps 10 mantissa bits.
// The products A_HL D_L / A_HL T_LL pass through A's strict upper triangle, which the
// caller no longer needs.  Layout: row-major, pitch TP floats (TP = 72 keeps the fragment
// loads free of bank conflicts).  On entry T's two blocks T[0:16, 16:32] and
// T[32:48, 48:64] must be zero (they are read as part of T_LL and T_HH and never
// written); everything else of T is written here.  The caller synchronises the group
// before (A written) and after (T read).
template <int TP>
__device__ __forceinline__ void mma_tile_16x8(const float *X, int ldx, const float *Y, int ldy,
                                              int K, float (&acc)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 4
    for (int kk = 0; kk < K; kk += 8) {
        uint32_t a[4], b[2];
        a[0] = to_tf32(X[g * ldx + kk + t]);
        a[1] = to_tf32(X[(g + 8) * ldx + kk + t]);
        a[2] = to_tf32(X[g * ldx + kk + t + 4]);
        a[3] = to_tf32(X[(g + 8) * ldx + kk + t + 4]);
        b[0] = to_tf32(Y[(kk + t) * ldy + g]);
        b[1] = to_tf32(Y[(kk + t + 4) * ldy + g]);
        mma_16x8x8_tf32(acc, a, b);
    }
}
__device__ __forceinline__ void store_tile_16x8(float *C, int ldc, const float (&acc)[4], float sign,
                                                int lane) {
    const int g = lane >> 2, t = lane & 3;
    C[g * ldc + 2 * t] = sign * acc[0];
    C[g * ldc + 2 * t + 1] = sign * acc[1];
    C[(g + 8) * ldc + 2 * t] = sign * acc[2];
    C[(g + 8) * ldc + 2 * t + 1] = sign * acc[3];
}

// In place: M holds A on entry and T on exit (its lower triangle with the diagonal; the
// strict upper triangle is scratch except two blocks, see below).  One warpgroup,
// t = 0..127, synchronised by `sync()` (a named barrier over exactly those threads):
//   1. warp w replaces diagonal block w (16 x 16) of A by its inverse D_w, computed in
//      registers, one lane per column, right-looking (once x_m is final, A[r][m] x_m is
//      added to every later row r, so the dependent path is 16 FMAs long);
//   2. 16 -> 32: for the block pair p = w >> 1 (H = 2p + 1, L = 2p), warp w forms columns
//      [8 (w & 1), +8) of X = A_HL D_L into scratch, and after a barrier replaces those
//      columns of A_HL by T_HL = -D_H X;
//   3. 32 -> 64: with the 32 x 32 halves L = [0, 32), H = [32, 64), warp w forms columns
//      [8w, 8w + 8) of X = A_HL T_LL into scratch and, after a barrier, of T_HL = -T_HH X.
// Levels 2 and 3 run on the warp-level tensor cores (mma.sync m16n8k8, tf32 operands,
// fp32 accumulate): T is rounded to bf16 afterwards, and tf32 keeps 10 mantissa bits.
// Scratch is the upper-right 32 x 32 block (rows 0..31, columns 32..63).  The blocks
// M[0:16, 16:32] and M[32:48, 48:64] are read as the zero upper parts of T_LL and T_HH:
// the caller must have zeroed them (they are never written here).  Row pitch TP floats
// (TP = 72 keeps the fragment loads free of bank conflicts).
template <int TP, typename Sync>
__device__ __forceinline__ void invert_unit_lower_64_inplace_wg(float *M, int t, Sync sync)
{
    const int warp = t >> 5, lane = t & 31;
    // 1. diagonal blocks
    {
        const int c = lane & 15;
        float *Mb = M + (16 * warp) * TP + 16 * warp;
        float acc[16], x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            x[m] = (m < c) ? 0.f : ((m == c) ? 1.f : -acc[m]);
#pragma unroll
            for (int r = m + 1; r < 16; ++r) acc[r] = fmaf(Mb[r * TP + m], x[m], acc[r]);
        }
        __syncwarp();                                  // every lane has read the block
        if (lane < 16) {
#pragma unroll
            for (int r = 0; r < 16; ++r) Mb[r * TP + c] = x[r];
        }
    }
    sync();
    // 2. 16 -> 32 merges
    {
        const int p = warp >> 1, nt = warp & 1;
        const int lo = 32 * p, hi = lo + 16;
        float *X = M + (16 * p) * TP + 32 + 16 * p + 8 * nt;   // scratch rows 16p.., columns 32 + 16p..
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tile_16x8<TP>(M + hi * TP + lo, TP, M + lo * TP + lo + 8 * nt, TP, 16, acc, lane);
        store_tile_16x8(X, TP, acc, 1.f, lane);
        sync();                                        // A_HL read by both warps of the pair
        float acc2[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tile_16x8<TP>(M + hi * TP + hi, TP, X, TP, 16, acc2, lane);
        store_tile_16x8(M + hi * TP + lo + 8 * nt, TP, acc2, -1.f, lane);
    }
    sync();
    // 3. 32 -> 64 merge
    {
        const int nc = 8 * warp;
        float *X = M + 32 + nc;                        // scratch rows 0..31, columns 32 + 8w..
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
            mma_tile_16x8<TP>(M + (32 + 16 * mt) * TP, TP, M + nc, TP, 32, acc[mt], lane);
        sync();                                        // every warp has read A_HL and T_LL
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) store_tile_16x8(X + 16 * mt * TP, TP, acc[mt], 1.f, lane);
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float acc2[4] = {0.f, 0.f, 0.f, 0.f};
            mma_tile_16x8<TP>(M + (32 + 16 * mt) * TP + 32, TP, X, TP, 32, acc2, lane);
            store_tile_16x8(M + (32 + 16 * mt) * TP + nc, TP, acc2, -1.f, lane);
        }
    }
}

}  // namespace gdn
