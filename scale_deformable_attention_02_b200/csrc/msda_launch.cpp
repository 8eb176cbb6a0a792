// msda_launch.cpp -- launch-shape helper shared by the kernels' launchers.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "msda_internal.h"

namespace msda {

int64_t persistent_ctas(const void *kernel, int threads, int64_t items, int round)
{
    static std::mutex mu;
    static std::unordered_map<const void *, int> occ_cache;
    static int sm_cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    int sms = 0, occ = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64) sms = sm_cache[dev];
        auto it = occ_cache.find(kernel);
        if (it != occ_cache.end()) occ = it->second;
    }
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
        std::lock_guard<std::mutex> lock(mu);
        if (dev >= 0 && dev < 64) sm_cache[dev] = sms;
    }
    if (occ <= 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) !=
                cudaSuccess ||
            occ < 1)
            occ = 1;
        std::lock_guard<std::mutex> lock(mu);
        occ_cache[kernel] = occ;
    }
    const int64_t rounds = (items + round - 1) / round;
    int64_t want = (int64_t)sms * occ;
    if (want > rounds) want = rounds;
    return want < 1 ? 1 : want;
}

}  // namespace msda
