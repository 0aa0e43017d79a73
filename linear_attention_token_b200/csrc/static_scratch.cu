// Library-held scratch for gdn_prefill_static_scratch (include/gdn.h): callers that
// cannot allocate device memory still need somewhere for the kernel's error word.
// Every GPU that loads the library holds this array until the library is unloaded; all
// calls on a device share it.
#include <cuda_runtime.h>

#include "common.cuh"

namespace gdn {

static __device__ __align__(256) unsigned char g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

size_t static_scratch_capacity() { return GDN_STATIC_SCRATCH_BYTES; }

// Device address of g_static_scratch in the current context.  In host code the array's
// name is only a host-side stand-in, so the address is asked of the runtime on every
// call: once the module is loaded in a context that is a table lookup, and it stays
// right when the device is reset and its primary context (with the module) is made anew,
// which a per-device cache would not.
cudaError_t static_scratch_ptr(void **out)
{
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    *out = p;
    return cudaSuccess;
}

}  // namespace gdn
