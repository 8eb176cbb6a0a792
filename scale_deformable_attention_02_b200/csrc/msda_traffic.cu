// msda_traffic.cu -- the memory-system floor of the path: replays a list of
// 32-element value rows (fp32 or bf16) as plain gathers, as vector
// reductions into an fp32 gradient, or as both,
// with no index arithmetic, so the kernels' times can be set against what
// the memory system does with the same rows in the same order.  Test and
// benchmark support (msda_debug_row_traffic), not part of the compute path.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

// Warps sweep contiguous ranges of the row list.  A row is 32 elements: 128
// bytes of fp32 or 64 bytes of bf16 value, and always 128 bytes of fp32
// gradient.  Eight lanes move one row (16 bytes of fp32 or 8 bytes of bf16
// each), except for a bare bf16 gather, where four lanes take 16 bytes each,
// so a warp instruction covers four rows (eight for that gather); each lane
// keeps kB rows in flight.
template <typename VT, int MODE, int kB>  // MODE 0: gather, 1: reduce a row of ones, 2: both
__global__ void __launch_bounds__(256) row_traffic_kernel(const __grid_constant__ TrafficParams p)
{
    constexpr bool kWide = MODE == 0 && sizeof(VT) == 2;  // bf16 gather: 16 bytes per lane
    constexpr int kLanes = kWide ? 4 : 8;                 // lanes per row
    constexpr int kRows = 32 / kLanes;                    // rows per warp instruction
    constexpr int kElems = 32 / kLanes;                   // elements per lane
    constexpr int kGrid = sizeof(VT) == 2 ? 8 : 4;        // row offsets must be multiples
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int slot = lane / kLanes, chunk = lane % kLanes;
    const int64_t r0 = gw * p.per_warp;
    const int64_t r1 = r0 + p.per_warp < p.n_rows ? r0 + p.per_warp : p.n_rows;
    const VT *value = static_cast<const VT *>(p.value);
    float acc = 0.f;
    for (int64_t r = r0; r < r1; r += kRows * kB) {
        int64_t o[kB];
        float v[kB][kElems];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            const int64_t i = r + kRows * b + slot;
            o[b] = i < r1 ? (int64_t)__ldg(p.rows + i) : -1;
            // rows outside the buffers or off the vector grid are skipped
            if (o[b] < 0 || o[b] + 32 > p.n_value || (o[b] % kGrid) != 0) o[b] = -1;
#pragma unroll
            for (int e = 0; e < kElems; ++e) v[b][e] = 1.f;
            if (MODE != 1 && o[b] >= 0) {
                const VT *src = value + o[b] + kElems * chunk;
                if constexpr (sizeof(VT) == 4) {
                    const float4 t = __ldg(reinterpret_cast<const float4 *>(src));
                    v[b][0] = t.x; v[b][1] = t.y; v[b][2] = t.z; v[b][3] = t.w;
                } else if constexpr (kWide) {
                    const uint4 t = __ldg(reinterpret_cast<const uint4 *>(src));
                    const unsigned w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        v[b][2 * e] = __uint_as_float(w[e] << 16);
                        v[b][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                    }
                } else {
                    const uint2 t = __ldg(reinterpret_cast<const uint2 *>(src));
                    v[b][0] = __uint_as_float(t.x << 16);
                    v[b][1] = __uint_as_float(t.x & 0xffff0000u);
                    v[b][2] = __uint_as_float(t.y << 16);
                    v[b][3] = __uint_as_float(t.y & 0xffff0000u);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (o[b] < 0) continue;
            if constexpr (MODE != 0)
                red_add_v4(p.grad + o[b] + 4 * chunk, v[b][0], v[b][1], v[b][2], v[b][3]);
#pragma unroll
            for (int e = 0; e < kElems; ++e) acc += v[b][e];
        }
    }
    if (p.sink_len > 0) p.sink[(gw * 32 + lane) % p.sink_len] = acc;
}

}  // namespace

template <typename VT, int MODE>
cudaError_t launch_mode(const TrafficParams &p, int depth, int ctas, cudaStream_t stream)
{
    switch (depth) {
    case 2: row_traffic_kernel<VT, MODE, 2><<<ctas, 256, 0, stream>>>(p); break;
    case 4: row_traffic_kernel<VT, MODE, 4><<<ctas, 256, 0, stream>>>(p); break;
    case 8: row_traffic_kernel<VT, MODE, 8><<<ctas, 256, 0, stream>>>(p); break;
    case 16: row_traffic_kernel<VT, MODE, 16><<<ctas, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename VT>
cudaError_t launch_vt(const TrafficParams &p, int mode, int depth, int ctas, cudaStream_t stream)
{
    switch (mode) {
    case 0: return launch_mode<VT, 0>(p, depth, ctas, stream);
    case 1: return launch_mode<VT, 1>(p, depth, ctas, stream);
    case 2: return launch_mode<VT, 2>(p, depth, ctas, stream);
    default: return cudaErrorInvalidValue;
    }
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
    return p.bf16 ? launch_vt<__nv_bfloat16>(p, mode, depth, ctas, stream)
                  : launch_vt<float>(p, mode, depth, ctas, stream);
}

}  // namespace msda
