// Per-device, once-per-device host caches (plain C++, no CUDA dependency).
//
// Kernel attributes (the dynamic shared-memory limit), occupancy queries and device properties
// belong to one device; a process that drives several GPUs must set or query them once per
// device, not once per process.  PerDevice<T> keeps one value per device index, computes it the
// first time that device asks (under a mutex, so concurrent first calls from several host threads
// compute it once), and never caches a failed computation.
#pragma once

#include <mutex>

namespace fs {

constexpr int kMaxDevices = 64;

template <typename T>
class PerDevice {
 public:
  // Returns true and the device's value, computing it with `make(T*) -> bool` on the first
  // successful call for `dev`.  Returns false for a device index outside [0, kMaxDevices) or when
  // `make` fails (the next call tries again).
  template <typename Make>
  bool get(int dev, T* out, Make&& make) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(mu_);
    if (!ready_[dev]) {
      T v{};
      if (!make(&v)) return false;
      val_[dev] = v;
      ready_[dev] = true;
    }
    *out = val_[dev];
    return true;
  }

 private:
  std::mutex mu_;
  bool ready_[kMaxDevices] = {};
  T val_[kMaxDevices] = {};
};

}  // namespace fs
