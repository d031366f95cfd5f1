// device.cu -- per-device facts the launch code needs (host only).
#include <cuda_runtime.h>

#include <atomic>

#include "plan_impl.h"

namespace z3 {

namespace {
constexpr int kMaxDevices = 128;
std::atomic<int> g_sm_count[kMaxDevices];  // 0 = not looked up yet
}  // namespace

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    const bool cached = dev >= 0 && dev < kMaxDevices;
    if (cached) {
        const int n = g_sm_count[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (cached) g_sm_count[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace z3
