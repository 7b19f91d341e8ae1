// Per-device one-time set-up (host code only).
//
// A kernel attribute such as its dynamic shared-memory limit belongs to the
// kernel on one device: a process that launches the kernel on several GPUs must
// set it on each of them.  PerDeviceOnce remembers, per device ordinal, whether
// the set-up succeeded; a failed set-up is retried by the next caller.
#pragma once

#include <atomic>
#include <mutex>

namespace attn {

template <int kMaxDevices = 64>
class PerDeviceOnce {
 public:
  // Runs `setup` (returning bool) the first time device `dev` asks, and reports
  // success on every later call for that device without running it again.
  // Devices outside [0, kMaxDevices) are refused.
  template <typename F>
  bool ensure(int dev, F&& setup) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    if (done_[dev].load(std::memory_order_acquire)) return true;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return true;
    const bool ok = setup();
    if (ok) done_[dev].store(true, std::memory_order_release);
    return ok;
  }

  bool done(int dev) const {
    return dev >= 0 && dev < kMaxDevices && done_[dev].load(std::memory_order_acquire);
  }

 private:
  std::atomic<bool> done_[kMaxDevices] = {};
  std::mutex mu_;
};

}  // namespace attn
