// zha_attr.h -- a per-device "raise once" record for kernel attributes.
//
// cudaFuncSetAttribute (for example the dynamic shared memory a kernel may
// use) acts on the CURRENT device only, so a process that launches the same
// kernel on several devices must set it on each of them.  PerDeviceMax keeps,
// per device ordinal, the largest value already set, and calls the setter
// only when a launch needs more on that device.  Thread-safe: concurrent
// callers may both call the setter (harmless: it is idempotent), and the
// record only ever grows.  Plain C++ (no CUDA types), so the host tests can
// drive it with a fake setter.
#pragma once

#include <atomic>

namespace zha {

template <int DEV_MAX = 64>
struct PerDeviceMax {
    std::atomic<long long> done[DEV_MAX];  // zero-initialised in static storage

    // Make sure device `dev` has been raised to at least `need`: calls
    // set(need) (which returns 0 on success) unless a value >= need was
    // recorded for dev.  Devices outside [0, DEV_MAX) call set every time.
    // Returns the setter's error, or 0.
    template <typename Set>
    int raise(int dev, long long need, Set &&set) {
        if (dev < 0 || dev >= DEV_MAX) return set(need);
        std::atomic<long long> &d = done[dev];
        if (d.load(std::memory_order_acquire) >= need) return 0;
        const int err = set(need);
        if (err != 0) return err;
        long long cur = d.load(std::memory_order_relaxed);
        while (cur < need && !d.compare_exchange_weak(cur, need, std::memory_order_release, std::memory_order_relaxed)) {
        }
        return 0;
    }
};

}  // namespace zha
