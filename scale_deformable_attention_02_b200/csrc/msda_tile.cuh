// msda_tile.cuh -- window geometry shared by the tiled kernels
// (msda_fwd_tiled.cu, msda_bwd_tiled.cu).
#pragma once

#include <cuda_runtime.h>

namespace msda {

// First pixel (column or row) of a level's window for cell index cc of g
// cells along that axis: the cell's first edge u = cc/g lies at pixel
// coordinate u*W - 0.5, so its first cell column is floor((2 cc W - g) /
// (2 g)); the window starts `halo` pixels before it, and is kept inside
// [-1, W + 1 - ww] so that it never holds more than the level and its
// one-pixel zero border.
__device__ __forceinline__ int window_origin(int cc, int g, int W, int halo, int ww)
{
    const int num = 2 * cc * W - g;
    const int den = 2 * g;
    int o = (num >= 0 ? num / den : -((-num + den - 1) / den)) - halo;
    o = min(o, W + 1 - ww);
    return max(o, -1);
}

// A corner entry's x: >= 0 a global element offset inside the (n, m) map;
// <= -2 a shared-memory byte offset b stored as -2 - b; -1 no corner.
__device__ __forceinline__ int shared_entry(int byte_off) { return -2 - byte_off; }

// A sample record's first word: >= 0 for a sample whose four corners lie in
// its level's window, with the byte offset of its first corner row in the
// low kRecOffBits bits and the window's row step in 16-byte units above;
// <= -2 for a sample read from global memory, whose cell (x0, y0) of a level
// of width W is stored as -2 - ((y0 + 1) (W + 1) + x0 + 1); -1 for a sample
// that adds nothing.  Offsets stay below 2^18 (a CTA's shared memory) and
// steps below 2^12 16-byte units (256 pixels of at most 128 bytes).
constexpr int kRecOffBits = 18;
constexpr int kRecOffMask = (1 << kRecOffBits) - 1;
__device__ __forceinline__ int window_record(int byte_off, int row_step_bytes)
{
    return byte_off | ((row_step_bytes >> 4) << kRecOffBits);
}
__device__ __forceinline__ int global_record(int x0, int y0, int W)
{
    return -2 - ((y0 + 1) * (W + 1) + x0 + 1);
}

}  // namespace msda
