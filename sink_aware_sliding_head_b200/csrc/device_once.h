// device_once.h - per-device, thread-safe "do this once" flags for host-side
// set-up that must happen on every device a process uses (raising a kernel's
// dynamic shared-memory limit, looking up a device symbol's address).
//
// Plain C++ (no CUDA headers), so the indexing and retry rules can be tested
// on a machine without a GPU.
#pragma once
#include <atomic>
#include <mutex>

namespace flint {

constexpr int kMaxDevices = 64;

// run(dev, f): calls f() the first time it is asked for device `dev` and
// remembers success (f returns 0); a failed call is retried the next time.
// Devices outside [0, kMaxDevices) are not cached: f runs on every call.
// Concurrent callers for the same device wait for the first one, so f runs at
// most once successfully per device.
class PerDeviceOnce {
 public:
  template <class F>
  int run(int dev, F&& f) {
    if (dev < 0 || dev >= kMaxDevices) return static_cast<int>(f());
    if (done_[dev].load(std::memory_order_acquire)) return 0;
    std::lock_guard<std::mutex> g(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return 0;
    const int e = static_cast<int>(f());
    if (e == 0) done_[dev].store(true, std::memory_order_release);
    return e;
  }
  bool done(int dev) const {
    return dev >= 0 && dev < kMaxDevices && done_[dev].load(std::memory_order_acquire);
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

}  // namespace flint
