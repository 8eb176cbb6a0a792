// msda_internal.h -- launch parameters shared by the host entry points and
// the kernels.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msda_types.h"

namespace msda {

// Everything a forward launch needs.  Checked on the host before launch:
// S*M*D < 2^31 (row offsets are int32), L*K <= 32, rows of 16..512 bytes.
struct FwdParams {
    const void *value;
    // unfused inputs
    const float *loc;   // [N,Lq,G,L,K,2]
    const float *attn;  // [N,Lq,M,L,K]
    // fused inputs
    const float *ref;     // [N,Lq,ref_dim]
    const float *off;     // [N,Lq,G,L,K,2]
    const float *logits;  // [N,Lq,M,L,K]
    int ref_dim;
    // outputs
    float *out;       // [N,Lq,M*D]
    float *loc_out;   // nullable (fused) [N,Lq,G,L,K,2]
    float *attn_out;  // nullable (fused)
    int64_t items;    // N*Lq*M
    int64_t chunk;    // items per CTA (set by the launcher)
    int Lq, S, M, D, L, K;
    int G, Hg;    // deformable groups and heads per group (G = M: one per head)
    FastDiv dM, dLq, dHg;  // division by M, Lq and Hg
    int nchunks;  // 16-byte chunks per value row
    Levels lv;
    // bounds-checked build only (-DMSDA_CHECKED): value elements an access
    // may touch, and the device word counting skipped accesses
    // ([0] = count, [1] = first element index)
    int64_t check_limit;
    unsigned long long *check;
};

struct BwdParams {
    const void *value;
    const float *loc;   // unfused inputs
    const float *attn;
    const float *ref;     // fused inputs: [N,Lq,ref_dim]
    const float *off;     // [N,Lq,G,L,K,2]
    const float *logits;  // [N,Lq,M,L,K]
    int ref_dim;
    const float *grad_out;
    float *grad_value;
    float *grad_loc;     // nullable (unfused) [N,Lq,G,L,K,2]; zeroed by the host if G < M
    float *grad_attn;    // nullable (unfused)
    float *grad_ref;     // nullable (fused; zeroed by the host, accumulated over heads)
    float *grad_off;     // nullable (fused) [N,Lq,G,L,K,2]; zeroed by the host if G < M
    float *grad_logits;  // nullable (fused)
    int64_t items;
    int64_t chunk;  // items per CTA (set by the launcher)
    int Lq, S, M, D, L, K;
    int G, Hg;  // deformable groups and heads per group (G = M: one per head)
    FastDiv dM, dLq, dHg;  // division by M, Lq and Hg
    int nchunks;
    Levels lv;
    // bounds-checked build only (-DMSDA_CHECKED): value elements an access
    // may touch, and the device word counting skipped accesses
    // ([0] = count, [1] = first element index)
    int64_t check_limit;
    unsigned long long *check;
};

struct PointsParams {
    const float *loc;
    int32_t *valid, *x0, *y0;
    float *x, *y;
    int64_t *rows;
    int64_t samples;  // N*Lq*M*L*K
    int L, K;
    Levels lv;
};

// CTAs for a persistent launch: (SMs x resident CTAs of `kernel`) on the
// current device, but no more than the rounds of `round` items there are.
int64_t persistent_ctas(const void *kernel, int threads, int64_t items, int round);

// Whether one item per warp round finishes sooner than two.  A persistent
// grid whose last round of two-item steps holds only a few warps leaves the
// rest of the GPU idle for a whole step; counted in item times per warp,
// ceil(items / 2W) * 2 against ceil(items / W1) for W and W1 resident warps
// of the two layouts.  True when the one-item layout needs at least 15%
// fewer item times (the decoder backward: 3 against 4).
bool one_item_rounds(const void *two_item_kernel, const void *one_item_kernel, int warps,
                     int64_t items);

// Launchers (return the launch's cudaError_t).
cudaError_t launch_forward(const FwdParams &p, bool bf16, bool fused, int lanes_per_row,
                           cudaStream_t stream);
cudaError_t launch_backward(const BwdParams &p, bool bf16, int lanes_per_row,
                            cudaStream_t stream);
// Backward of the fused forward (chained to ref, offsets and logits).
cudaError_t launch_backward_fused(const BwdParams &p, bool bf16, int lanes_per_row,
                                  cudaStream_t stream);
cudaError_t launch_sample_points(const PointsParams &p, cudaStream_t stream);

// Row replay of msda_debug_row_traffic (msda_traffic.cu).
struct TrafficParams {
    const void *value;    // fp32 or bf16 (bf16 set)
    float *grad;
    const int32_t *rows;  // element offsets of 32-element rows
    int64_t n_rows;
    int64_t n_value;      // elements in value and in grad
    float *sink;          // per-lane sums of the gathered rows (nullable if sink_len == 0)
    int64_t sink_len;
    int64_t per_warp;     // set by the launcher
    bool bf16;
};
cudaError_t launch_row_traffic(TrafficParams p, int mode, int depth, int ctas,
                               cudaStream_t stream);

#ifdef MSDA_CHECKED
// The current device's check word (two zero-initialised 64-bit counters in a
// file-scope __device__ array), or nullptr if the runtime cannot give its
// address.
unsigned long long *check_word();
#endif

// ---------------------------------------------------------------------------
// Tiled kernels (msda_tiled.h): a tile plan sorts each batch entry's queries
// into the cells of a gx x gy grid over the unit square; a work unit is one
// (batch entry, cell, head) and stages the head's value window around the
// cell on every level into shared memory.
// ---------------------------------------------------------------------------
constexpr int kTileLevels = 8;     // levels a tiled call takes
constexpr int kTileMaxCells = 8192;

// Device view of a plan and the unit schedule.  Checked on the host: the plan
// matches the call's dims; windows are 0 (level not staged) or at least 2 x 2
// pixels and at most 256 x 256.
struct TileView {
    const int *cell_start;  // [N][G + 1]: first sorted query of every cell
    const int *perm;        // [N][Lq]: queries sorted by cell
    int gx, gy, G, halo;
    FastDiv dG;              // division by G
    int ww[kTileLevels];     // window width and height per level, pixels
    int wh[kTileLevels];
    int soff[kTileLevels];   // byte offset of the level's window in dynamic shared memory
    unsigned window_tx;      // bytes the windows of one unit bring in
    int units;               // N * G * M
    unsigned *stall;         // device word: waits that ran out (never expected)
};

// Tensor maps first: each CUtensorMap is 64-byte aligned.
struct FwdTiledParams {
    CUtensorMap maps[kTileLevels];  // value of level l as a 5-d tensor (D, M, W_l, H_l, N)
    FwdParams f;
    TileView t;
};

// The tiled backward also keeps, per chunk of up to T queries of a cell, the
// chunk's grad_out rows, one record per sample inside its window, the pixels'
// contribution counts (then run starts) and placement cursors, and the
// chunk's queries.  Byte offsets into dynamic shared memory, after the
// windows, whose space then holds the sorted contributions.
struct BwdTiledParams {
    CUtensorMap maps[kTileLevels];
    BwdParams b;
    TileView t;
    int T;                     // queries per chunk
    int keys;                  // window pixels of all levels
    int roff[kTileLevels + 1]; // first key of each level's window; roff[L] = keys
    int off_g, off_rec, off_start, off_cursor, off_queue;
};

struct TilePlanParams {
    const float *ref;  // [N, Lq, ref_dim]
    int ref_dim;
    int N, Lq, gx, gy;
    int *cell_start;   // [N][gx*gy + 1]
    int *perm;         // [N][Lq]
};

cudaError_t launch_tile_plan(const TilePlanParams &p, cudaStream_t stream);
cudaError_t launch_forward_tiled(const FwdTiledParams &p, bool bf16, bool fused,
                                 int ctas_per_sm, int dyn_smem, cudaStream_t stream);
cudaError_t launch_backward_tiled(const BwdTiledParams &p, bool bf16, bool fused, int dyn_smem,
                                  cudaStream_t stream);
// Static shared memory of the tiled backward kernel for these dims, or < 0.
int backward_tiled_static_smem(bool bf16, bool fused, int D, int LK);
// The device word that counts bounded waits that ran out, or nullptr.
unsigned *stall_word();

}  // namespace msda
