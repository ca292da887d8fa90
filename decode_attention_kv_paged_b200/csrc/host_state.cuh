// host_state.cuh -- host-side per-device bookkeeping shared by the entry points.
//
// Per-device records live in fixed arrays indexed by the device ordinal, so
// a pointer to one stays valid for the life of the process (a growing
// container would move its elements when another thread first touches a
// higher-numbered device).  Kernel attributes such as the dynamic
// shared-memory limit are set on the function for the CURRENT device only,
// so "already configured" is tracked per device too.
#pragma once

#include <atomic>

#include <cuda_runtime.h>

namespace attn {

// Devices a process may drive through this library.
constexpr int kMaxDevices = 64;

// Ordinal of the calling thread's current device, or -1 if it cannot be read
// or is beyond kMaxDevices.
inline int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// One bit per device: whether a per-function setting has been applied there.
// Two threads that both see "not done" both apply the setting, which is
// harmless (the settings are idempotent).
class PerDeviceFlag {
  public:
    bool done(int dev) const {
        return dev >= 0 && ((bits_.load(std::memory_order_acquire) >> dev) & 1ull) != 0;
    }
    void mark(int dev) {
        if (dev >= 0) bits_.fetch_or(1ull << dev, std::memory_order_release);
    }

  private:
    std::atomic<unsigned long long> bits_{0};
};

// Applies `set()` (returning cudaError_t) once per device for the function
// whose flag is `flag`; returns the first failure.
template <typename F>
cudaError_t configure_once_per_device(PerDeviceFlag &flag, F &&set) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (flag.done(dev)) return cudaSuccess;
    const cudaError_t e = set();
    if (e == cudaSuccess) flag.mark(dev);
    return e;
}

}  // namespace attn
