// msda_check.cu -- the device word of the bounds-checked build
// (-DMSDA_CHECKED): kernels count the value-map accesses they skipped in it,
// and the host entry points read and clear it after each launch.  Empty in
// the default build.
#include <cuda_runtime.h>

#include "msda_internal.h"

namespace msda {

#ifdef MSDA_CHECKED
namespace {
// [0] = accesses skipped, [1] = element index of the first one recorded
__device__ __align__(16) unsigned long long g_check_word[2];
}  // namespace

unsigned long long *check_word()
{
    // Looked up on every call (this build is for checking, not timing): the
    // address stays valid for the current device's context, including a
    // context created again after cudaDeviceReset.
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_check_word) != cudaSuccess) return nullptr;
    return static_cast<unsigned long long *>(ptr);
}
#endif

}  // namespace msda
