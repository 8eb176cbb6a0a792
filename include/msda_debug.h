/*
 * msda_debug.h -- test-support entry point of the MSDeformAttn library.
 *
 * Not part of the compute path: it exposes the per-sample cell arithmetic
 * that the forward and backward kernels share, so a test can compare the
 * integer side of the computation (pixel coordinate, cell, corner rows) bit
 * for bit with an independent implementation.
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

#ifdef __cplusplus
}
#endif

#endif /* MSDA_DEBUG_H */
