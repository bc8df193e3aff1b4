// Per-device launch facts, computed once and cached: SM count, the opt-in shared-memory
// attribute of each kernel, and occupancy per (kernel, block size, shared memory). This
// keeps the host cost of a call to a few lookups.
#include <map>
#include <mutex>
#include <set>
#include <tuple>

#include "kernels.h"

namespace moedisp {

namespace {
std::mutex g_mu;

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    return dev;
}
}  // namespace

int current_sm_count() {
    static std::map<int, int> cache;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    cache[dev] = n;
    return n;
}

int64_t current_l2_bytes() {
    static std::map<int, int64_t> cache;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev) != cudaSuccess || n <= 0)
        n = 126 << 20;
    cache[dev] = n;
    return n;
}

cudaError_t allow_dynamic_smem(const void* kernel) {
    static std::set<std::pair<int, const void*>> done;
    const int dev = current_device();
    std::lock_guard<std::mutex> lock(g_mu);
    if (done.count({dev, kernel})) return cudaSuccess;
    int optin = 0;
    cudaError_t err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    cudaFuncAttributes attr;
    err = cudaFuncGetAttributes(&attr, kernel);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               optin - (int)attr.sharedSizeBytes);
    if (err != cudaSuccess) return err;
    done.insert({dev, kernel});
    return cudaSuccess;
}

cudaError_t blocks_per_sm(const void* kernel, int threads, size_t smem, int* out) {
    static std::map<std::tuple<int, const void*, int, size_t>, int> cache;
    cudaError_t err = allow_dynamic_smem(kernel);
    if (err != cudaSuccess) return err;
    const int dev = current_device();
    {
        std::lock_guard<std::mutex> lock(g_mu);
        auto it = cache.find({dev, kernel, threads, smem});
        if (it != cache.end()) {
            *out = it->second;
            return cudaSuccess;
        }
    }
    int n = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (err != cudaSuccess) return err;
    if (n < 1) n = 1;
    std::lock_guard<std::mutex> lock(g_mu);
    cache[{dev, kernel, threads, smem}] = n;
    *out = n;
    return cudaSuccess;
}

}  // namespace moedisp
