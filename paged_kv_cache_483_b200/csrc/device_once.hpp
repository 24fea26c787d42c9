// Per-device "do once" bookkeeping for kernel attributes.
//
// A kernel's dynamic shared-memory limit (cudaFuncSetAttribute) belongs to
// each device's context, so a process whose pools live on several devices
// must set it once on every device that launches the kernel.  PerDeviceOnce
// records, in one atomic bit per device id, which devices are done; any host
// thread may call it.  Two threads that reach a new device at the same time
// both run the set-up, which is harmless because it is idempotent; a set-up
// that fails is not recorded and runs again on the next call.
//
// Host-only C++ (no CUDA types), so the bookkeeping is tested on the CPU.
#pragma once

#include <atomic>
#include <cstdint>

namespace pa {

class PerDeviceOnce {
 public:
  static constexpr int kTracked = 64;   // device ids 0 .. 63 are remembered

  // Runs setup() unless it already succeeded on `dev`; returns its result
  // (0 = success) or 0 when nothing had to run.  Devices outside the tracked
  // range run setup() on every call.
  template <class F>
  int run(int dev, F&& setup) {
    const bool tracked = dev >= 0 && dev < kTracked;
    const uint64_t bit = tracked ? (uint64_t(1) << dev) : 0;
    if (tracked && (done_.load(std::memory_order_acquire) & bit)) return 0;
    const int e = setup();
    if (e == 0 && tracked) done_.fetch_or(bit, std::memory_order_acq_rel);
    return e;
  }

  bool done(int dev) const {
    return dev >= 0 && dev < kTracked &&
           (done_.load(std::memory_order_acquire) >> dev) & 1u;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

}  // namespace pa
