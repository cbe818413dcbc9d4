// dlm_per_device.h -- bookkeeping for set-up that must happen once on every CUDA device a
// process uses (host side; no CUDA types, so it is unit-tested on its own).
//
// cudaFuncSetAttribute and cudaGetSymbolAddress act on the calling thread's current
// device: a process that drives two GPUs has to repeat them on each.  PerDeviceOnce keeps
// one "done" bit per device index; run(dev, init) calls init() under a mutex unless the
// bit is already set, sets it only when init() reports success (0), and returns init()'s
// result (or 0 when nothing had to be done).  A failed init is retried by the next call.
// Concurrent first calls from several host threads run init() once per device.
#pragma once
#include <atomic>
#include <cstdint>
#include <mutex>

namespace dlm {

constexpr int kMaxDevices = 64;  // device indices 0 .. 63

class PerDeviceOnce {
 public:
  // Returns kBadDevice for an index outside [0, kMaxDevices), else 0 or init()'s code.
  static constexpr int kBadDevice = -1;

  template <class F>
  int run(int dev, F init) {
    if (dev < 0 || dev >= kMaxDevices) return kBadDevice;
    const uint64_t bit = uint64_t(1) << dev;
    if (done_.load(std::memory_order_acquire) & bit) return 0;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_.load(std::memory_order_relaxed) & bit) return 0;
    const int e = init();
    if (e == 0) done_.fetch_or(bit, std::memory_order_release);
    return e;
  }

  bool done(int dev) const {
    return dev >= 0 && dev < kMaxDevices && (done_.load(std::memory_order_acquire) >> dev) & 1;
  }

 private:
  std::atomic<uint64_t> done_{0};
  std::mutex mu_;
};

}  // namespace dlm
