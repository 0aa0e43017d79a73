// Tensor-core (tcgen05) chunked prefill — placeholder until the kernel lands.
#include "common.cuh"

namespace gdn {

bool prefill_tc_supported(int dk, int dv, gdn_dtype dtype)
{
    (void)dk; (void)dv; (void)dtype;
    return false;
}

cudaError_t launch_prefill_tc(const void *, const void *, const void *, const float *,
                              const float *, const float *, void *, float *, const int32_t *, int,
                              long long, long long, int, int, float, int, DeviceError *,
                              cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace gdn
