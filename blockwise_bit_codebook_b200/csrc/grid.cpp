// Occupancy and SM-count caches for persistent grids.
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "launch.h"

namespace bbc {

// 0 when a query fails: nothing is cached then (a later call asks again), and the launch that
// follows with an empty grid fails, so the entry point reports BBC_ERR_CUDA.
int resident_ctas(const void* kernel, int block, size_t dyn_smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    auto key = std::make_tuple(kernel, dev, block, dyn_smem);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block, dyn_smem) != cudaSuccess)
        return 0;
    if (sms < 1 || per_sm < 1) return 0;
    const int ctas = sms * per_sm;
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = ctas;
    return ctas;
}

// Streaming multiprocessors of the current device (0 when the query fails; not cached then).
int sm_count() {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(dev);
        if (it != cache.end()) return it->second;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) return 0;
    std::lock_guard<std::mutex> lock(mu);
    cache[dev] = sms;
    return sms;
}

}  // namespace bbc
