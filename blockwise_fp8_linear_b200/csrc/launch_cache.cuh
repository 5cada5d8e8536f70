// launch_cache.cuh -- per-device facts about one kernel configuration that the host
// needs before a launch (the shared-memory opt-in, the register-split check, the
// number of co-resident CTA pairs), worked out once per device and then reused, so
// that a launch costs only its tensor-map encodes and the launch itself.
#pragma once

#include <atomic>

namespace fp8bw {

struct LaunchCache {
    static constexpr int kDevices = 64;
    // 0 = not prepared on this device; otherwise the number of co-resident clusters
    // (1 for single-CTA kernels).  Two threads that prepare at once store the same value.
    std::atomic<int> clusters[kDevices];

    int get(int dev) const
    {
        return (dev >= 0 && dev < kDevices) ? clusters[dev].load(std::memory_order_acquire) : 0;
    }
    void set(int dev, int v)
    {
        if (dev >= 0 && dev < kDevices)
            clusters[dev].store(v, std::memory_order_release);
    }
};

} // namespace fp8bw
