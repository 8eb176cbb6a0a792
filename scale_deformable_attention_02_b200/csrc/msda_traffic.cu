// msda_traffic.cu -- the memory-system floor of the path: replays a list of
// 128-byte value rows as plain gathers, as vector reductions, or as both,
// with no index arithmetic, so the kernels' times can be set against what
// the memory system does with the same rows in the same order.  Test and
// benchmark support (msda_debug_row_traffic), not part of the compute path.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

// Warps sweep contiguous ranges of the row list; eight lanes move one row
// (16 bytes each), so a warp instruction covers four rows, and each lane
// keeps kB rows in flight.
template <int MODE, int kB>  // MODE 0: gather, 1: reduce a row of ones, 2: both; kB rows in flight
__global__ void __launch_bounds__(256) row_traffic_kernel(const __grid_constant__ TrafficParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int slot = lane >> 3, chunk = lane & 7;
    const int64_t r0 = gw * p.per_warp;
    const int64_t r1 = r0 + p.per_warp < p.n_rows ? r0 + p.per_warp : p.n_rows;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; r += 4 * kB) {
        int64_t o[kB];
        float4 v[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            const int64_t i = r + 4 * b + slot;
            o[b] = i < r1 ? (int64_t)__ldg(p.rows + i) : -1;
            // rows outside the buffers or off the 16-byte grid are skipped
            if (o[b] < 0 || o[b] + 32 > p.n_value || (o[b] & 3) != 0) o[b] = -1;
            v[b] = make_float4(1.f, 1.f, 1.f, 1.f);
            if (MODE != 1 && o[b] >= 0)
                v[b] = __ldg(reinterpret_cast<const float4 *>(p.value + o[b]) + chunk);
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (o[b] < 0) continue;
            if (MODE != 0)
                red_add_v4(p.grad + o[b] + 4 * chunk, v[b].x, v[b].y, v[b].z, v[b].w);
            acc += v[b].x + v[b].y + v[b].z + v[b].w;
        }
    }
    if (p.sink_len > 0) p.sink[(gw * 32 + lane) % p.sink_len] = acc;
}

}  // namespace

template <int MODE>
cudaError_t launch_mode(const TrafficParams &p, int depth, int ctas, cudaStream_t stream)
{
    switch (depth) {
    case 2: row_traffic_kernel<MODE, 2><<<ctas, 256, 0, stream>>>(p); break;
    case 4: row_traffic_kernel<MODE, 4><<<ctas, 256, 0, stream>>>(p); break;
    case 8: row_traffic_kernel<MODE, 8><<<ctas, 256, 0, stream>>>(p); break;
    case 16: row_traffic_kernel<MODE, 16><<<ctas, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_row_traffic(TrafficParams p, int mode, int depth, int ctas,
                               cudaStream_t stream)
{
    if (p.n_rows == 0) return cudaSuccess;
    if (depth <= 0) depth = 8;
    if (ctas <= 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
        ctas = 8 * sms;  // 64 warps per SM
    }
    const int64_t warps = (int64_t)ctas * 8;
    p.per_warp = (p.n_rows + warps - 1) / warps;
    p.per_warp = (p.per_warp + 63) / 64 * 64;
    switch (mode) {
    case 0: return launch_mode<0>(p, depth, ctas, stream);
    case 1: return launch_mode<1>(p, depth, ctas, stream);
    case 2: return launch_mode<2>(p, depth, ctas, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace msda
