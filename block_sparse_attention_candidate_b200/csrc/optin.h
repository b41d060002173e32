// Per-device record of the dynamic shared-memory opt-in of one kernel.
//
// cudaFuncSetAttribute(..., cudaFuncAttributeMaxDynamicSharedMemorySize, ...)
// sets a property of the kernel in the current device's context, so a process
// that launches the same kernel on several GPUs has to set it once on each.
// OptInTable remembers, per device ordinal, the largest size already granted
// and calls the setter (the CUDA call, or a fake in the host tests) only when
// a device has not seen that size yet.  Thread-safe: one mutex per table.
//
// No CUDA types here, so the logic is testable on a machine without a GPU.
#pragma once

#include <mutex>

namespace dynrad {

class OptInTable {
 public:
  static constexpr int kMaxDevices = 64;

  // Returns true when `bytes` is granted on `device`: already recorded, or
  // `set(bytes)` returned true now (then it is recorded).  Returns false for
  // an ordinal outside [0, kMaxDevices) or when the setter fails; a failure is
  // not recorded, so the next call tries again.
  template <class Setter>
  bool ensure(int device, int bytes, Setter&& set) {
    if (device < 0 || device >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(mu_);
    if (granted_[device] >= bytes) return true;
    if (!set(bytes)) return false;
    granted_[device] = bytes;
    return true;
  }

  int granted(int device) const {
    if (device < 0 || device >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(mu_);
    return granted_[device];
  }

 private:
  mutable std::mutex mu_;
  int granted_[kMaxDevices] = {};
};

}  // namespace dynrad
