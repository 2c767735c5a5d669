// Host-side state that depends only on the device (SM count, device-symbol addresses,
// kernel attributes): computed on a device's first call and reused afterwards, so the
// per-call host work is argument checks, tensor-map encoding and the launch itself.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace puro {

constexpr int kMaxDevices = 64;

// One value of type T per device. get() runs `init(dev, value)` with device `dev` current
// the first time it is asked for the current device and caches the value when init
// returns true; later calls read the cached value without locking. Safe to call from
// several host threads.
template <typename T>
class PerDevice {
 public:
  template <typename F>
  bool get(T &out, F init) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    if (ready_[dev].load(std::memory_order_acquire)) {
      out = value_[dev];
      return true;
    }
    std::lock_guard<std::mutex> lock(mu_);
    if (!ready_[dev].load(std::memory_order_relaxed)) {
      T v{};
      if (!init(dev, v)) return false;
      value_[dev] = v;
      ready_[dev].store(true, std::memory_order_release);
    }
    out = value_[dev];
    return true;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> ready_[kMaxDevices] = {};
  T value_[kMaxDevices] = {};
};

// Number of SMs of the current device (cached).
inline bool sm_count(int &sms) {
  static PerDevice<int> cache;
  return cache.get(sms, [](int dev, int &v) {
    return cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
  });
}

}  // namespace puro
