// ivc_device_once.h — per-device guards for host-side state that belongs to
// one device's context.
//
// A kernel's dynamic shared-memory opt-in (cudaFuncSetAttribute) and a
// device's SM count are properties of the device current at the call. One
// process may drive several GPUs through the same library instance (a thread
// per GPU, or cudaSetDevice between calls), so a process-wide "done" flag
// would leave every device but the first without the opt-in, and its large
// launches would fail. DeviceTable keeps one value per (key, device ordinal)
// under a mutex, so threads driving different GPUs do not race.
//
// Host-only and free of CUDA calls, so that it can be unit-tested on a
// machine without a GPU.
#pragma once
#include <array>
#include <map>
#include <mutex>

namespace ivc {

constexpr int kMaxDevices = 64;

class DeviceTable {
 public:
  // Raises the value recorded for (key, dev) to `value`: runs `apply()` only
  // when the recorded value is smaller (0 when never set), and records
  // `value` only when apply returns 0. Returns apply's result, 0 when nothing
  // had to be done, or -1 for a device ordinal outside [0, kMaxDevices).
  template <typename F>
  int raise(const void* key, int dev, int value, F&& apply) {
    if (dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> lock(mu_);
    int& cur = table_[key][dev];
    if (cur >= value) return 0;
    const int rc = apply();
    if (rc == 0) cur = value;
    return rc;
  }

  // The value recorded for (key, dev), 0 when never set.
  int get(const void* key, int dev) {
    if (dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu_);
    auto it = table_.find(key);
    return it == table_.end() ? 0 : it->second[dev];
  }

 private:
  std::mutex mu_;
  std::map<const void*, std::array<int, kMaxDevices>> table_;  // value-initialised rows
};

}  // namespace ivc
