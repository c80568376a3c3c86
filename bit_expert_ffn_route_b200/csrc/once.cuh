// once.cuh — host-side "once per device" guard for launch set-up calls
// (cudaFuncSetAttribute applies to the device current at the call, so a
// process that drives several GPUs needs it once on each).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace moe {

// Runs fn() (returning true on success) the first time this guard is used on
// the current device; later calls on that device return true at once.  A
// failed fn() is retried at the next call.  Devices beyond 63 run fn() every
// time.
template <typename Fn>
bool once_per_device(std::atomic<uint64_t>& done, Fn&& fn) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev < 0 || dev >= 64) return fn();
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (!fn()) return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

// SM count of the current device, looked up once per device (148 if the
// query fails).
inline int device_sm_count() {
    static std::atomic<int> counts[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    auto query = [dev] {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        return n;
    };
    if (dev < 0 || dev >= 64) return query();
    int n = counts[dev].load(std::memory_order_relaxed);
    if (!n) {
        n = query();
        counts[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace moe
