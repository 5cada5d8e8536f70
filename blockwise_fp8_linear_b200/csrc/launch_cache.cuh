// launch_cache.cuh -- per-device facts about one kernel configuration that the host
// needs before a launch (the shared-memory opt-in, the register-split check, the
// number of co-resident CTA pairs), worked out once per device and then reused, so
// that a launch costs only its tensor-map encodes and the launch itself.
#pragma once

#include <atomic>
#include <cuda_runtime.h>

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

#ifndef FP8BW_PDL
#define FP8BW_PDL 1
#endif
// Programmatic stream serialization: the kernel may be launched while the previous
// kernel in the stream is still finishing (every kernel of this library waits for
// its predecessor with griddepcontrol.wait before touching memory), so launch
// latency and prologue (barrier set-up, tensor-memory allocation) overlap that tail.
inline void set_pdl(cudaLaunchAttribute &a)
{
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = FP8BW_PDL;
}

} // namespace fp8bw
