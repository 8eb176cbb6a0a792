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

bool one_item_rounds(const void *two_item_kernel, const void *one_item_kernel, int warps,
                     int64_t items)
{
    constexpr int64_t kAll = INT64_C(1) << 40;  // more rounds than any grid holds
    const int64_t w2 = persistent_ctas(two_item_kernel, warps * 32, kAll, 1) * warps;
    const int64_t w1 = persistent_ctas(one_item_kernel, warps * 32, kAll, 1) * warps;
    const int64_t t2 = (items + 2 * w2 - 1) / (2 * w2) * 2;
    const int64_t t1 = (items + w1 - 1) / w1;
    return t1 * 20 <= t2 * 17;
}

}  // namespace msda
