// Library-held scratch for gdn_prefill_static_scratch (include/gdn.h): callers that
// cannot allocate device memory still need somewhere for the kernel's error word.
// Every GPU that loads the library holds this array until the library is unloaded; all
// calls on a device share it.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace gdn {

static __device__ __align__(256) unsigned char g_static_scratch[GDN_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};
}  // namespace

size_t static_scratch_capacity() { return GDN_STATIC_SCRATCH_BYTES; }

// Device address of g_static_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device (with
// that device current) with cudaGetSymbolAddress and cached.
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

}  // namespace gdn
