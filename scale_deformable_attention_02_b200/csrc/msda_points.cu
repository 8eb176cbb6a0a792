// msda_points.cu -- per-sample cell record, produced by the same msda_cell()
// and msda_row() the forward and backward kernels use, so that the integer
// side of the path (pixel coordinate, cell, corner rows) can be compared bit
// for bit with an independent implementation.  One thread per sample.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

__global__ void __launch_bounds__(256) points_kernel(const __grid_constant__ PointsParams p)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= p.samples) return;
    const int l = (int)((i / p.K) % p.L);
    const int H = p.lv.H[l], W = p.lv.W[l], start = p.lv.start[l];
    const float2 t = reinterpret_cast<const float2 *>(p.loc)[i];
    float x, y, fx, fy;
    int x0 = 0, y0 = 0;
    const bool ok = msda_cell(t.x, t.y, H, W, x, y, x0, y0, fx, fy);
    p.valid[i] = ok ? 1 : 0;
    p.x0[i] = ok ? x0 : 0;
    p.y0[i] = ok ? y0 : 0;
    p.x[i] = x;
    p.y[i] = y;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        p.rows[4 * i + j] = ok ? (int64_t)msda_row(start, H, W, y0 + (j >> 1), x0 + (j & 1)) : -1;
}

}  // namespace

cudaError_t launch_sample_points(const PointsParams &p, cudaStream_t stream)
{
    if (p.samples == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((p.samples + 255) / 256);
    points_kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace msda
