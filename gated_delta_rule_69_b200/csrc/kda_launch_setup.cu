// Per-device launch set-up shared by the launchers: the dynamic shared-memory
// limit of each kernel (a per-device function attribute) and the SM count.
// Both are cached per (device, kernel) under a mutex, so that one process may
// drive several GPUs and call the library from several host threads.
#include <mutex>
#include <set>
#include <utility>

#include "kda_internal.cuh"

namespace kda {

namespace {

std::mutex g_setup_mutex;
std::set<std::pair<int, const void *>> g_attr_done;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};

}  // namespace

cudaError_t set_max_dynamic_smem(const void *func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const auto key = std::make_pair(dev, func);
    if (g_attr_done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    g_attr_done.insert(key);
    return cudaSuccess;
}

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (dev < kMaxDevices && g_sm_count[dev] > 0) return g_sm_count[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < kMaxDevices) g_sm_count[dev] = n;
    return n;
}

}  // namespace kda
