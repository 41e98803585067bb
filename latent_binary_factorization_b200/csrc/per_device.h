// Per-device caches of host-side launch set-up.
//
// cudaFuncSetAttribute and the occupancy queries act on the device that is
// current when they are called, so a value cached once per process would be
// wrong for the second GPU of a process that drives several.  PerDevice keeps
// one slot per device ordinal.  Plain C++ (no CUDA types), so the keying can
// be checked on a machine without a GPU.
#pragma once

#include <atomic>

namespace lb {

constexpr int kMaxDevices = 64;

// One int per device ordinal; 0 means "not set yet".  Concurrent first calls
// on one device may both run `init` (the CUDA calls it wraps are idempotent);
// the slot then holds one of their equal results.
struct PerDevice {
  std::atomic<int> slot[kMaxDevices] = {};

  // The cached value for `dev`, running init(int& value) -> error code on
  // first use; a non-zero code is returned and nothing is cached.  A device
  // ordinal outside 0..kMaxDevices-1 runs init every time.
  template <class F>
  int get(int dev, int& value, F init) {
    if (dev >= 0 && dev < kMaxDevices) {
      const int v = slot[dev].load(std::memory_order_acquire);
      if (v != 0) {
        value = v;
        return 0;
      }
    }
    int v = 0;
    const int err = init(v);
    if (err != 0) return err;
    if (dev >= 0 && dev < kMaxDevices && v != 0) slot[dev].store(v, std::memory_order_release);
    value = v;
    return 0;
  }
};

}  // namespace lb
