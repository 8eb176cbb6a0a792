// msda_check.cu -- the device word of the bounds-checked build
// (-DMSDA_CHECKED): kernels count the value-map accesses they skipped in it,
// and the host entry points read and clear it after each launch.  Empty in
// the default build.
#include <cuda_runtime.h>

#include <mutex>

#include "msda_internal.h"

namespace msda {

#ifdef MSDA_CHECKED
namespace {
// [0] = accesses skipped, [1] = element index of the first one recorded
__device__ __align__(16) unsigned long long g_check_word[2];
}  // namespace

unsigned long long *check_word()
{
    static std::mutex mu;
    static unsigned long long *cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_check_word) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<unsigned long long *>(ptr);
    }
    return cache[dev];
}
#endif

}  // namespace msda
