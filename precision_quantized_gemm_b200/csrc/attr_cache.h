// attr_cache.h — per-device record of a kernel attribute that only grows
// (the dynamic shared memory a kernel was opened up to).  Plain C++ (no CUDA
// headers) so that the host logic can be tested without a GPU.
//
// cudaFuncSetAttribute acts on the current device only, so the record is
// kept per device: a process that launches on a second GPU configures the
// kernel there on its first launch.  Threads may launch concurrently; the
// fast path is one atomic load, and raising the value is serialised so that
// a smaller request can never overwrite a larger one.
#pragma once
#include <atomic>
#include <mutex>

namespace qg {

constexpr int kAttrMaxDevices = 64;

class GrowOnlyAttr {
 public:
  // Makes sure the attribute on `dev` is at least `value`: calls
  // `set(value)` (which returns 0 on success) when the recorded value is
  // smaller, and records it on success.  Returns set's error, or 0.
  // Devices outside [0, kAttrMaxDevices) are passed straight to `set`.
  template <class Setter>
  int ensure(int dev, int value, Setter&& set) {
    if (dev < 0 || dev >= kAttrMaxDevices) return set(value);
    if (value <= v_[dev].load(std::memory_order_acquire)) return 0;
    std::lock_guard<std::mutex> lk(mu_);
    if (value <= v_[dev].load(std::memory_order_relaxed)) return 0;
    const int e = set(value);
    if (e == 0) v_[dev].store(value, std::memory_order_release);
    return e;
  }
  int recorded(int dev) const {
    return (dev >= 0 && dev < kAttrMaxDevices) ? v_[dev].load(std::memory_order_acquire) : 0;
  }

 private:
  std::atomic<int> v_[kAttrMaxDevices] = {};
  std::mutex mu_;
};

}  // namespace qg
