// Host-side, per-device one-time setup for the kernel launchers.
//
// Opting a kernel in to more than 48 KB of dynamic shared memory
// (cudaFuncSetAttribute) and reading the SM count are properties of one device: a
// process that drives several GPUs must do both on each of them, and host threads
// that launch concurrently must not race on the "done" record.  PerDevice keeps that
// record per device index behind a mutex.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace gdn {

class PerDevice {
public:
    static constexpr int kMaxDevices = 128;

    // Runs setup() (returning cudaError_t) once on the current device for the life of
    // the process and writes that device's SM count to *sms (when non-null).  A failed
    // setup is not recorded, so the next call tries again.
    template <class F>
    cudaError_t ensure(F &&setup, int *sms = nullptr) {
        int dev = -1;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mutex_);
        if (!done_[dev]) {
            int n = 0;
            e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (e == cudaSuccess) e = setup();
            if (e != cudaSuccess) return e;
            sms_[dev] = n;
            done_[dev] = true;
        }
        if (sms) *sms = sms_[dev];
        return cudaSuccess;
    }

private:
    std::mutex mutex_;
    bool done_[kMaxDevices] = {};
    int sms_[kMaxDevices] = {};
};

}  // namespace gdn
