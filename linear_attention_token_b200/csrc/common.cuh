// Internal helpers shared by the libgdn kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

// Device error word layout (first 16 bytes of the prefill workspace):
//   word[0] = first gdn_status recorded (0 = none), word[1] = where it happened,
//   word[2] = blockIdx.x, word[3] = blockIdx.y of the recording CTA.
struct DeviceError {
    int status;
    int where;
    int bx;
    int by;
};

__device__ __forceinline__ void record_error(DeviceError *err, int status, int where) {
    if (err == nullptr) return;
    if (atomicCAS(&err->status, 0, status) == 0) {
        err->where = where;
        err->bx = blockIdx.x;
        err->by = blockIdx.y;
        __threadfence();
    }
}

// Per-call options the host packs into one int for every kernel.
constexpr int kOptL2Norm = 1;       // L2-normalise q and k per (token, head) in the kernel
constexpr int kOptGateLogits = 2;   // g and beta hold logits: g = -softplus(a), beta = sigmoid(b)

// Gate prologue (GDN_FLAG_GATE_LOGITS): the decay gate alpha = exp(g) must lie in (0, 1)
// and the write strength beta in (0, 1) ("論文解説: Qwen3.8-Next の設計", section "GDNの中身",
// the text under Eq. (1)); from unconstrained logits, g = -softplus(a) and beta = sigmoid(b).
// softplus is evaluated as max(a, 0) + log1p(exp(-|a|)), which neither overflows nor loses
// the small values.
__device__ __forceinline__ float gate_log_decay(float x, int opts) {
    return (opts & kOptGateLogits) ? -(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)))) : x;
}
__device__ __forceinline__ float gate_strength(float x, int opts) {
    return (opts & kOptGateLogits) ? 1.f / (1.f + expf(-x)) : x;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Four consecutive elements as fp32 (16-byte fp32 load or 8-byte bf16 load).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace gdn
