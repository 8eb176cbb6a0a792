// msda_tile_plan.cu -- the tile plan of the tiled kernels: the queries of
// every batch entry sorted into the cells of a gx x gy grid over the unit
// square by reference point (a counting sort, one CTA per batch entry), and
// the device word in which the tiled kernels count bounded waits that ran
// out.
//
// Queries of Deformable DETR's encoder sample around their own reference
// point on every level ("Deformable DETR" wiki page, "Multi-scale deformable
// attention"), so the queries of one cell read overlapping windows of every
// value map; the tiled kernels stage those windows once per cell.
#include "msda_internal.h"

namespace msda {
namespace {

constexpr int kPlanThreads = 1024;

// [0] = bounded waits of the tiled kernels that ran out.
__device__ unsigned g_stall_word[4];

// Cell of a reference point: column floor(x * gx), row floor(y * gy), both
// clamped to the grid; NaN goes to column (row) 0, +Inf to the last.
__device__ __forceinline__ int plan_cell(float x, float y, int gx, int gy)
{
    const float fx = x * (float)gx, fy = y * (float)gy;
    const int cx = fx >= 0.f ? min((int)fx, gx - 1) : 0;  // (int) saturates at 2^31 - 1
    const int cy = fy >= 0.f ? min((int)fy, gy - 1) : 0;
    return cy * gx + cx;
}

// Inclusive prefix sum of v over the CTA (kPlanThreads threads).
__device__ __forceinline__ int block_inclusive_scan(int v, int *warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kPlanThreads / 32 ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    return v + (warp > 0 ? warp_tot[warp - 1] : 0);
}

__global__ void __launch_bounds__(kPlanThreads) tile_plan_kernel(const __grid_constant__ TilePlanParams p)
{
    extern __shared__ int cnt[];  // [G] counts, then running positions
    __shared__ int warp_tot[32];
    const int n = blockIdx.x;
    const int G = p.gx * p.gy;
    for (int c = threadIdx.x; c < G; c += kPlanThreads) cnt[c] = 0;
    __syncthreads();
    const float *ref = p.ref + (int64_t)n * p.Lq * p.ref_dim;
    for (int q = threadIdx.x; q < p.Lq; q += kPlanThreads) {
        const float2 r = __ldg(reinterpret_cast<const float2 *>(ref + (int64_t)q * p.ref_dim));
        atomicAdd(&cnt[plan_cell(r.x, r.y, p.gx, p.gy)], 1);
    }
    __syncthreads();
    // exclusive prefix sum over the cells: each thread takes a contiguous run
    const int per = (G + kPlanThreads - 1) / kPlanThreads;
    const int c0 = min((int)threadIdx.x * per, G), c1 = min(c0 + per, G);
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += cnt[c];
    int run = block_inclusive_scan(sum, warp_tot) - sum;
    int *start = p.cell_start + (int64_t)n * (G + 1);
    for (int c = c0; c < c1; ++c) {
        const int k = cnt[c];
        cnt[c] = run;
        start[c] = run;
        run += k;
    }
    if (threadIdx.x == 0) start[G] = p.Lq;
    __syncthreads();
    int *perm = p.perm + (int64_t)n * p.Lq;
    for (int q = threadIdx.x; q < p.Lq; q += kPlanThreads) {
        const float2 r = __ldg(reinterpret_cast<const float2 *>(ref + (int64_t)q * p.ref_dim));
        perm[atomicAdd(&cnt[plan_cell(r.x, r.y, p.gx, p.gy)], 1)] = q;
    }
}

}  // namespace

cudaError_t launch_tile_plan(const TilePlanParams &p, cudaStream_t stream)
{
    const int smem = p.gx * p.gy * (int)sizeof(int);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            tile_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    tile_plan_kernel<<<p.N, kPlanThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

unsigned *stall_word()
{
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_stall_word) != cudaSuccess) return nullptr;
    return static_cast<unsigned *>(ptr);
}

}  // namespace msda
