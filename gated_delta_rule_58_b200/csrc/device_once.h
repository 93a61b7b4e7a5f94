// One-time, per-device set-up steps (kernel attribute opt-ins, cached device
// properties), run under a lock. Plain C++ with no CUDA dependency, so the
// keying logic can be checked on a machine without a GPU.
//
// A CUDA function attribute such as the dynamic shared-memory opt-in applies to
// the device that is current when it is set, so a set-up done once per process
// would leave every other device of the process without it. Each call site keeps
// one PerDeviceOnce and runs its set-up through run_once_per_device with the
// current device index: the set-up runs at most once per device (again after a
// failure), and concurrent host threads see either "not done" (and wait for the
// lock) or the finished result.
#pragma once

#include <mutex>

namespace gdn {

constexpr int kMaxDevicesOnce = 64;

struct PerDeviceOnce {
  std::mutex mu;
  bool done[kMaxDevicesOnce] = {};
  int value[kMaxDevicesOnce] = {};  // an int the set-up may cache (e.g. the SM count)
};

// Runs fn(dev, &value) unless it already succeeded for `dev`; returns true when the
// set-up is (now) done, with *value_out the cached int. fn returns true on success.
// A device index outside [0, kMaxDevicesOnce) is refused (returns false, fn not run).
template <typename F>
bool run_once_per_device(PerDeviceOnce& once, int dev, F&& fn, int* value_out = nullptr) {
  if (dev < 0 || dev >= kMaxDevicesOnce) return false;
  std::lock_guard<std::mutex> lock(once.mu);
  if (!once.done[dev]) {
    int v = 0;
    if (!fn(dev, &v)) return false;
    once.value[dev] = v;
    once.done[dev] = true;
  }
  if (value_out) *value_out = once.value[dev];
  return true;
}

}  // namespace gdn
