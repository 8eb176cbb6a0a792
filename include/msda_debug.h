/*
 * msda_debug.h -- test and benchmark support of the MSDeformAttn library.
 *
 * Not part of the compute path.  msda_debug_sample_points exposes the
 * per-sample cell arithmetic that the forward and backward kernels share, so
 * a test can compare the integer side of the computation (pixel coordinate,
 * cell, corner rows) bit for bit with an independent implementation.
 * msda_debug_row_traffic replays a row list as bare gathers and reductions:
 * the memory-system floor the kernels are measured against.
 */
#ifndef MSDA_DEBUG_H
#define MSDA_DEBUG_H

#include "msda.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * For every sample i of sampling_locations [N,Lq,M,L,K,2] (level l = (i/K)%L):
 *   x[i], y[i]   pixel coordinates loc_x*W_l - 0.5, loc_y*H_l - 0.5 (fp32,
 *                each as two IEEE operations; "Deformable DETR" wiki page,
 *                "Multi-scale deformable attention": phi_l rescales the
 *                normalised point to the level's pixel grid)
 *   valid[i]     1 if some corner can lie inside the level (-1 < x < W_l and
 *                -1 < y < H_l), else 0 (NaN/Inf give 0)
 *   x0[i], y0[i] floor(x), floor(y) (0 when not valid)
 *   rows[4i+j]   value row of corner j = (y0 + j/2, x0 + j%2), or -1 when the
 *                corner lies outside the level or the sample is not valid
 * All outputs are device arrays with one entry per sample (rows: four),
 * 4-byte aligned (rows: 8-byte); sampling_locations is 8-byte aligned.  The
 * value pointer is not needed; dims.S, dims.M, dims.D are checked as in
 * msda_forward (D = 4 and M = 1 may be passed when no value map exists).
 * Errors: as msda_forward.
 */
MSDA_API msda_status msda_debug_sample_points(const int64_t *spatial_shapes,
                                     const int64_t *level_start_index,
                                     const float *sampling_locations, msda_dims dims,
                                     int32_t *valid, int32_t *x0, int32_t *y0,
                                     float *x, float *y, int64_t *rows,
                                     msda_stream_t stream);

/*
 * The memory-system floor of the path.  Replays a list of 32-element rows
 * (128 bytes of fp32 or 64 bytes of bf16 value; the gradient is always fp32,
 * 128 bytes a row) in list order, with no index arithmetic:
 *   mode 0  gather every value row (what the forward's corner loads do);
 *   mode 1  add a row of ones into grad at every row with one vector
 *           reduction per 16 bytes (what the backward's scatter does);
 *   mode 2  gather every value row and add it into grad (the backward's
 *           memory operations).
 * Timing it on the corner rows of a workload gives the floor that the
 * gathers and reductions of the kernels cannot go below on this GPU.
 *
 *   value           device [n_value] of value_dtype, 16-byte aligned (unused
 *                   in mode 1; may then be NULL)
 *   value_dtype     MSDA_F32 or MSDA_BF16
 *   grad            device [n_value] fp32, 16-byte aligned (unused in mode 0;
 *                   may then be NULL)
 *   row_offsets     device [n_rows] int32 element offsets; rows that start
 *                   below 0, end past n_value, or are not a multiple of 4
 *                   (fp32) or 8 (bf16) elements are skipped
 *   sink            device [sink_len] fp32, receives per-lane sums of the
 *                   gathered rows so the loads cannot be dropped; may be NULL
 *                   when sink_len is 0
 *   depth           rows in flight per lane: 2, 4, 8 or 16 (0 gives 8)
 *   ctas            thread blocks of 256 threads; <= 0 gives 8 per SM
 * A caller after the floor times a few (depth, ctas) pairs and keeps the
 * fastest.
 * Errors: MSDA_ERR_NULL, MSDA_ERR_DTYPE, MSDA_ERR_SHAPE (mode, depth,
 * n_rows < 0, n_value < 32, sink_len < 0), MSDA_ERR_ALIGN, MSDA_ERR_ALIAS
 * (grad or sink overlapping value, row_offsets or each other).
 */
MSDA_API msda_status msda_debug_row_traffic(int mode, const void *value, msda_dtype value_dtype,
                                            float *grad, int64_t n_value,
                                            const int32_t *row_offsets, int64_t n_rows,
                                            float *sink, int64_t sink_len, int depth, int ctas,
                                            msda_stream_t stream);

/*
 * Bounded waits of the tiled kernels (msda_tiled.h) that ran out on the
 * current device since the last call: a tiled kernel waits for its tensor
 * copies with a bounded number of tries, and if a wait ever ran out it would
 * count it here and stop instead of spinning.  Synchronises the current
 * device, reads the count into *count and clears it.
 * Errors: MSDA_ERR_NULL, MSDA_ERR_CUDA.
 */
MSDA_API msda_status msda_debug_tiled_stalls(int64_t *count);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_DEBUG_H */
