// Occupancy cache for persistent grids.
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "launch.h"

namespace bbc {

int resident_ctas(const void* kernel, int block, size_t dyn_smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    auto key = std::make_tuple(kernel, dev, block, dyn_smem);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    int sms = 0, per_sm = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, block, dyn_smem);
    if (sms < 1) sms = 1;
    if (per_sm < 1) per_sm = 1;
    int ctas = sms * per_sm;
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = ctas;
    return ctas;
}

}  // namespace bbc
