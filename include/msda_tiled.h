/*
 * msda_tiled.h -- spatially tiled entry points of the MSDeformAttn core for
 * NVIDIA B200 (sm_100a).
 *
 * The calls below compute exactly what their untiled counterparts in msda.h
 * compute (same operation, same layouts, same conventions and errors); only
 * the schedule differs.  In the encoder of Deformable DETR every query sits
 * on a pixel of one of the levels and samples a few points around its own
 * position on every level ("Deformable DETR" wiki page, "Multi-scale
 * deformable attention": each query samples around its rescaled reference
 * point phi_l(p_q) plus small offsets; "Limitations": the cost of the method
 * is its unordered memory access).  Queries whose reference points are close
 * therefore read overlapping windows of every value map.
 *
 * A tile plan sorts the queries of each batch entry into the cells of a
 * grid_x x grid_y grid over the unit square of normalised coordinates, by
 * reference point.  A tiled call then works cell by cell and head by head:
 * for each level it copies the head's value window around the cell (the
 * cell's pixels plus `halo` pixels on every side) into shared memory with
 * one tensor copy, and reads the four corner rows of every sample from
 * there.  A sample whose cell lies outside the window (an offset of more
 * than `halo` pixels) reads its corners from global memory instead, so the
 * results never depend on the plan or on the halo: a poor plan is slow, not
 * wrong.  The backward accumulates the gradient of every window row in
 * registers and adds it to grad_value once per (cell, head), instead of once
 * per sample corner.
 *
 * Use: fill an msda_tile_plan with msda_tile_plan_init (host only), allocate
 * plan.device_bytes of device memory, run msda_tile_plan_build on the
 * reference points, then pass the same plan and buffer to the tiled calls.
 * A plan stays valid for as long as the reference points it was built from
 * do not change (in the encoder they are the pixel centres, fixed per image
 * size, so one plan serves every layer and every step).  Building is stream
 * ordered like every other call: the tiled calls must run on the build's
 * stream, or after it.
 *
 * Limits of the tiled calls (MSDA_ERR_UNSUPPORTED beyond them): L <= 8,
 * L*K <= 32, D*sizeof(value element) <= 128 bytes and a multiple of 16, every
 * H_l, W_l < 2^15, one set of locations per head (no deformable groups), and
 * the msda.h limits.
 */
#ifndef MSDA_TILED_H
#define MSDA_TILED_H

#include <stdint.h>

#include "msda.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MSDA_TILE_MAX_LEVELS 8

/* Host description of a tile plan: filled by msda_tile_plan_init, read by
 * every other call here, never written by the caller. */
typedef struct {
    int64_t N, Lq, S, L, D;  /* problem the plan was made for               */
    int32_t value_dtype;     /* msda_dtype                                   */
    int32_t halo;            /* pixels a window reaches past its cell        */
    int32_t grid_x, grid_y;  /* cells along x and y of the unit square       */
    int32_t ctas_per_sm;     /* resident CTAs the windows were sized for     */
    int32_t reserved;
    int64_t shapes[2 * MSDA_TILE_MAX_LEVELS];      /* (H_l, W_l)              */
    int32_t window_w[MSDA_TILE_MAX_LEVELS];        /* window size per level,  */
    int32_t window_h[MSDA_TILE_MAX_LEVELS];        /* in pixels (0: none)     */
    int64_t window_bytes;    /* shared memory of all windows of one CTA      */
    int64_t device_bytes;    /* device memory the plan occupies              */
} msda_tile_plan;

/*
 * Choose the cell grid and the per-level windows of a plan (host only, no
 * device work).  The cells are square in pixels of the largest level and as
 * large as the shared memory of `ctas_per_sm` resident CTAs per SM allows,
 * given the windows' size (the cell's extent on level l plus `halo` pixels
 * and one corner on every side), but small enough that N * cells * M work
 * units give every resident CTA of a 148-SM B200 about four.
 *
 *   value_dtype, spatial_shapes, level_start_index, dims   as in msda.h
 *   halo         pixels, 0 <= halo <= 64; a sample whose offset from its
 *                reference point exceeds it reads from global memory
 *   ctas_per_sm  1, 2 or 3; 0 picks 2
 *   plan         written
 *
 * Errors: MSDA_ERR_NULL, the msda.h dimension errors, MSDA_ERR_SHAPE (halo
 * or ctas_per_sm out of range), MSDA_ERR_UNSUPPORTED (beyond the tiled
 * limits).
 */
MSDA_API msda_status msda_tile_plan_init(msda_dtype value_dtype, const int64_t *spatial_shapes,
                                         const int64_t *level_start_index, msda_dims dims,
                                         int halo, int ctas_per_sm, msda_tile_plan *plan);

/*
 * Sort the queries of every batch entry into the plan's cells by reference
 * point: query q of entry n goes to the cell holding (x, y) =
 * reference_points[n, q, 0:2] (the box centre when reference_dim = 4);
 * points outside the unit square, NaN included, go to the nearest edge cell.
 * The order of the queries inside a cell is unspecified.
 *
 *   reference_points  device [N, Lq, reference_dim] fp32, 8-byte aligned
 *   reference_dim     2 or 4
 *   plan_buffer       device, plan->device_bytes, 16-byte aligned (written)
 *
 * Errors: MSDA_ERR_NULL, MSDA_ERR_SHAPE, MSDA_ERR_ALIGN, MSDA_ERR_ALIAS
 * (the buffer overlaps the reference points), MSDA_ERR_CUDA.
 */
MSDA_API msda_status msda_tile_plan_build(const msda_tile_plan *plan,
                                          const float *reference_points, int reference_dim,
                                          void *plan_buffer, msda_stream_t stream);

/*
 * msda_forward, msda_forward_fused, msda_backward and msda_backward_fused on
 * a tile plan.  Arguments, outputs and errors are those of the msda.h calls,
 * plus the plan (built for these dims, spatial shapes and value dtype, else
 * MSDA_ERR_SHAPE) and its device buffer (read only; MSDA_ERR_NULL if NULL,
 * MSDA_ERR_ALIAS if an output overlaps it).  The backward calls zero
 * grad_value (and grad_reference_points) on `stream` first, as the untiled
 * ones do.  Where D > 32, or where the problem's per-query shared memory
 * leaves no room for a chunk of 32 queries beside the plan's windows, they
 * run the untiled backward, which computes the same gradients.
 */
MSDA_API msda_status msda_forward_tiled(const void *value, msda_dtype value_dtype,
                                        const int64_t *spatial_shapes,
                                        const int64_t *level_start_index,
                                        const float *sampling_locations,
                                        const float *attention_weights, float *out,
                                        msda_dims dims, const msda_tile_plan *plan,
                                        const void *plan_buffer, msda_stream_t stream);

MSDA_API msda_status msda_forward_fused_tiled(const void *value, msda_dtype value_dtype,
                                              const int64_t *spatial_shapes,
                                              const int64_t *level_start_index,
                                              const float *reference_points, int reference_dim,
                                              const float *offsets, const float *logits,
                                              float *out, float *sampling_locations_out,
                                              float *attention_weights_out, msda_dims dims,
                                              const msda_tile_plan *plan,
                                              const void *plan_buffer, msda_stream_t stream);

MSDA_API msda_status msda_backward_tiled(const void *value, msda_dtype value_dtype,
                                         const int64_t *spatial_shapes,
                                         const int64_t *level_start_index,
                                         const float *sampling_locations,
                                         const float *attention_weights, const float *grad_out,
                                         float *grad_value, float *grad_sampling_locations,
                                         float *grad_attention_weights, msda_dims dims,
                                         const msda_tile_plan *plan, const void *plan_buffer,
                                         msda_stream_t stream);

MSDA_API msda_status msda_backward_fused_tiled(const void *value, msda_dtype value_dtype,
                                               const int64_t *spatial_shapes,
                                               const int64_t *level_start_index,
                                               const float *reference_points, int reference_dim,
                                               const float *offsets, const float *logits,
                                               const float *grad_out, float *grad_value,
                                               float *grad_reference_points, float *grad_offsets,
                                               float *grad_logits, msda_dims dims,
                                               const msda_tile_plan *plan,
                                               const void *plan_buffer, msda_stream_t stream);

/*
 * msda_forward_fused_tiled without a caller-provided plan buffer: the call
 * chooses the plan (as msda_tile_plan_init with `halo` and `ctas_per_sm`),
 * sorts the queries into it and runs the tiled fused forward, keeping the
 * plan in a device array that belongs to the library.  Nothing in the pages
 * corresponds to this call; it exists for callers that cannot give the
 * library device memory beyond their inputs and outputs (a plugin whose host
 * framework owns all device memory and offers no workspace, or a caller that
 * may not call cudaMalloc, which can synchronise the device and fail under
 * memory pressure).  It allocates nothing.
 *
 *  - The array holds plans of up to 4 MiB (plan.device_bytes; about a million
 *    queries): larger problems return MSDA_ERR_UNSUPPORTED.  Every GPU that
 *    loads the library keeps the array until the process exits.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and keeps it; make that first call before any
 *    stream capture.
 *  - Every call on a device uses the same array.  Each call rewrites every
 *    entry it reads, so nothing needs clearing between calls, but calls whose
 *    work overlaps on the GPU (other streams, other host threads) race on the
 *    array and must be serialised by the caller.
 *
 * Arguments, outputs and errors are those of msda_forward_fused and
 * msda_tile_plan_init; every check runs before any device work.
 */
MSDA_API msda_status msda_forward_fused_tiled_noalloc(
    const void *value, msda_dtype value_dtype, const int64_t *spatial_shapes,
    const int64_t *level_start_index, const float *reference_points, int reference_dim,
    const float *offsets, const float *logits, float *out, float *sampling_locations_out,
    float *attention_weights_out, msda_dims dims, int halo, int ctas_per_sm,
    msda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_TILED_H */
