// host_once.h -- per-device values computed once, safe across host threads.
//
// Plain C++ (no CUDA): the launchers use it to set kernel attributes and to
// cache occupancy limits the first time a kernel runs on a device.
#pragma once

#include <atomic>
#include <mutex>

namespace lowbit {

// One positive int per device.  get(dev, init) returns the published value;
// the first caller for a device runs init() under a lock and publishes a
// positive result with release order, so later callers read it without
// locking.  A result <= 0 means failure: it is returned, not published, and
// the next call runs init() again.  Devices outside [0, kMaxDevices) get 0.
class PerDevice {
public:
    static constexpr int kMaxDevices = 64;

    template <typename F>
    int get(int dev, F &&init)
    {
        if (dev < 0 || dev >= kMaxDevices) return 0;
        int v = slots_[dev].load(std::memory_order_acquire);
        if (v > 0) return v;
        std::lock_guard<std::mutex> lock(mu_);
        v = slots_[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
        v = init();
        if (v > 0) slots_[dev].store(v, std::memory_order_release);
        return v;
    }

private:
    std::atomic<int> slots_[kMaxDevices] = {};
    std::mutex mu_;
};

}  // namespace lowbit
