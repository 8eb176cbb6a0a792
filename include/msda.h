/*
 * msda.h -- C ABI of the multi-scale deformable attention (MSDeformAttn) core
 * for NVIDIA B200 (sm_100a).
 *
 * The operation ("Deformable DETR" wiki page, "Multi-scale deformable
 * attention" equation) is, for every batch entry n, query q and head m,
 *
 *   out[n,q,m*D:(m+1)*D] = sum_l sum_k A[n,q,m,l,k] *
 *                          bilinear(value[n, level l, m, :], loc[n,q,m,l,k])
 *
 * over per-head value maps that the caller has already projected (the value
 * projection W'_m and the output projection W_m of the equation are dense
 * GEMMs outside this library; bilinear sampling commutes with W'_m because
 * both are linear).  Heads are concatenated in the output ("Deformable
 * Attention" glossary page, multi-head paragraph).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layouts are dense, row-major, C-contiguous:
 *      value               [N, S, M, D]   fp32 or bf16 (msda_dtype)
 *      sampling_locations  [N, Lq, M, L, K, 2]  fp32, normalised (x, y)
 *      attention_weights   [N, Lq, M, L, K]     fp32
 *      out / grad_out      [N, Lq, M*D]         fp32
 *    S = sum_l H_l*W_l; level l occupies value rows [start_l, start_l +
 *    H_l*W_l), row-major in (h, w).  Channel c of the output is m*D + d.
 *  - spatial_shapes is a HOST array [L, 2] of int64 (H_l, W_l) and
 *    level_start_index a HOST array [L] of int64; both are read during the
 *    call only.  All tensor pointers are DEVICE pointers owned by the
 *    caller; the library keeps no pointer after the call returns.
 *  - Locations are normalised: (0,0) is the top-left corner of the image and
 *    (1,1) the bottom-right ("Deformable DETR" wiki page, "Multi-scale
 *    deformable attention").  The pixel coordinate on level l is
 *    x = loc_x*W_l - 0.5, y = loc_y*H_l - 0.5 (pixel centres at
 *    half-integers; the same convention as grid_sample with
 *    align_corners=False), computed as two IEEE fp32 operations each.
 *    Corners outside the level contribute zero (zero padding); a location
 *    with no corner inside the level, or a NaN/Inf location, contributes
 *    nothing and gets zero gradient.  Locations outside [0,1] are not errors.
 *  - Attention weights are used as given (never renormalised).
 *  - Accumulation is fp32 for both value dtypes.
 *  - `value` must be 16-byte aligned.  A 32-byte aligned fp32 map of D = 32
 *    lets the forward gather rows with 256-bit loads (a few percent faster);
 *    results agree with the 16-byte path to fp32 rounding.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  The library allocates no memory and never
 *    synchronises.  Outputs are fully overwritten.
 *  - Every argument check happens before any device work: a call that
 *    returns an error has launched nothing and written nothing.
 *
 * Limits of this build: L <= 32 and 1 <= L*K <= 128; D*sizeof(value
 * element) a multiple of 16 bytes (else MSDA_ERR_ALIGN), of any length up to
 * the next limit (rows over 512 bytes are taken in passes of 512); H_l, W_l,
 * M*D, S*M*D below 2^31 (row offsets inside one batch entry are 32-bit);
 * N*Lq*M below 2^31 (the kernels split (query, head) item indices in 32
 * bits).  Other calls beyond them return MSDA_ERR_UNSUPPORTED.  N = 0
 * or Lq = 0 is a valid empty problem (the backward then only zeroes
 * grad_value).
 */
#ifndef MSDA_H
#define MSDA_H

#include <stdint.h>

/* Exported symbols keep default visibility when the library is built with
 * -fvisibility=hidden. */
#if defined(__GNUC__)
#define MSDA_API __attribute__((visibility("default")))
#else
#define MSDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MSDA_OK = 0,
    MSDA_ERR_NULL = 1,        /* a required pointer is NULL                      */
    MSDA_ERR_SHAPE = 2,       /* a dimension is out of range (e.g. M < 1)        */
    MSDA_ERR_LEVELS = 3,      /* spatial_shapes / level_start_index / S disagree */
    MSDA_ERR_DTYPE = 4,       /* unknown msda_dtype                              */
    MSDA_ERR_ALIGN = 5,       /* a pointer or row size breaks the alignment rule */
    MSDA_ERR_ALIAS = 6,       /* an output overlaps an input or another output   */
    MSDA_ERR_UNSUPPORTED = 7, /* valid problem outside this build's limits       */
    MSDA_ERR_CUDA = 8,        /* the CUDA runtime reported an error at launch    */
    MSDA_ERR_DEVICE_CHECK = 9 /* bounds-checked build only (msda_checked.h): a
                                 gather or scatter fell outside the value map
                                 and was skipped                                 */
} msda_status;

typedef enum {
    MSDA_F32 = 0,  /* IEEE binary32                                   */
    MSDA_BF16 = 1  /* bfloat16 (upper 16 bits of a binary32)          */
} msda_dtype;

/* Problem dimensions: batch N, queries Lq, value rows S = sum_l H_l*W_l,
 * heads M, channels per head D (= C/M), levels L, points per level K. */
typedef struct {
    int64_t N, Lq, S, M, D, L, K;
} msda_dims;

/* A cudaStream_t passed as an opaque handle (NULL = legacy default stream). */
typedef void *msda_stream_t;

/* Human-readable name of a status code (static storage; never NULL). */
MSDA_API const char *msda_status_string(msda_status status);

/* ABI version of this header: MAJOR*10000 + MINOR*100 + PATCH. */
MSDA_API int msda_abi_version(void);

/* The cudaError_t value behind the calling thread's last MSDA_ERR_CUDA
 * (0 if none has occurred on this thread). */
MSDA_API int msda_last_cuda_error(void);

/*
 * Level metadata: level_start_index[l] = sum_{j<l} H_j*W_j, and *S_out =
 * sum_l H_l*W_l ("Deformable DETR" wiki page, "Multi-scale deformable
 * attention": L levels x^l of size H^l x W^l stacked into one flattened
 * value map).  Host-only; spatial_shapes [L,2] (H, W) and level_start_index
 * [L] are host arrays; S_out may be NULL.
 * Errors: MSDA_ERR_NULL, MSDA_ERR_SHAPE (L < 1 or a negative H/W),
 * MSDA_ERR_UNSUPPORTED (S would overflow int64's 2^62 guard).
 */
MSDA_API msda_status msda_level_start_index(const int64_t *spatial_shapes, int64_t L,
                                   int64_t *level_start_index, int64_t *S_out);

/*
 * Forward from given sampling locations and attention weights
 * ("Deformable DETR" wiki page, "Multi-scale deformable attention"
 * equation, each sample read by bilinear interpolation between the four
 * pixels around it, as in "Deformable attention module").
 *
 *   value               device [N,S,M,D] of value_dtype, 16-byte aligned
 *   spatial_shapes      host   [L,2] int64 (H_l, W_l), H_l, W_l >= 0
 *   level_start_index   host   [L] int64, must equal msda_level_start_index
 *   sampling_locations  device [N,Lq,M,L,K,2] fp32, 8-byte aligned
 *   attention_weights   device [N,Lq,M,L,K] fp32, 4-byte aligned
 *   out                 device [N,Lq,M*D] fp32, 16-byte aligned (written)
 *
 * Errors: MSDA_ERR_NULL (a non-empty tensor pointer or a host array is NULL),
 * MSDA_ERR_SHAPE, MSDA_ERR_LEVELS, MSDA_ERR_DTYPE, MSDA_ERR_ALIGN,
 * MSDA_ERR_ALIAS (out overlaps an input), MSDA_ERR_UNSUPPORTED,
 * MSDA_ERR_CUDA.
 */
MSDA_API msda_status msda_forward(const void *value, msda_dtype value_dtype,
                         const int64_t *spatial_shapes,
                         const int64_t *level_start_index,
                         const float *sampling_locations,
                         const float *attention_weights, float *out,
                         msda_dims dims, msda_stream_t stream);

/*
 * Fused forward: the attention weights and sampling locations are formed
 * inside the kernel from the raw projection outputs.
 *
 *  - A[n,q,m,:,:] = softmax over the L*K logits of head m, jointly across
 *    levels ("Deformable DETR" wiki page, "Multi-scale deformable attention":
 *    sum_l sum_k A_mlqk = 1; "Deformable attention module": the query
 *    projection's final MK channels are normalised by a softmax).
 *  - loc = phi_l(p_q) + dp in level-l pixels, i.e. in normalised units
 *    loc_x = ref_x + off_x / W_l and loc_y = ref_y + off_y / H_l (fp32 IEEE
 *    divide, then fp32 add) ("Deformable DETR" wiki page, "Multi-scale
 *    deformable attention": offsets are added after the rescaling phi_l).
 *    With reference_dim = 4 the reference is a box (cx, cy, w, h) and the
 *    offsets are in box units: loc_x = cx + off_x * w, loc_y = cy + off_y * h
 *    (fp32 multiply, then fp32 add) ("Deformable DETR" wiki page,
 *    "Variants / Iterative bounding box refinement": offsets modulated by the
 *    previous box's width and height).
 *  Then the forward above.  The locations and weights are bit-identical to
 *  what the composition msda_forward(loc, A) would be given.
 *
 *   reference_points    device [N,Lq,reference_dim] fp32, 8-byte aligned
 *   reference_dim       2 (point) or 4 (box)
 *   offsets             device [N,Lq,M,L,K,2] fp32 pixels (dx, dy), 8-byte aligned
 *                       (box units when reference_dim = 4)
 *   logits              device [N,Lq,M,L,K] fp32, 4-byte aligned
 *   out                 device [N,Lq,M*D] fp32, 16-byte aligned (written)
 *   sampling_locations_out  NULL or device [N,Lq,M,L,K,2] fp32 (written)
 *   attention_weights_out   NULL or device [N,Lq,M,L,K] fp32 (written)
 *
 * Errors: as msda_forward; MSDA_ERR_SHAPE also for reference_dim not 2 or 4.
 */
MSDA_API msda_status msda_forward_fused(const void *value, msda_dtype value_dtype,
                               const int64_t *spatial_shapes,
                               const int64_t *level_start_index,
                               const float *reference_points, int reference_dim,
                               const float *offsets, const float *logits,
                               float *out, float *sampling_locations_out,
                               float *attention_weights_out, msda_dims dims,
                               msda_stream_t stream);

/*
 * Backward of msda_forward: gradients flow through the bilinear
 * interpolation to the value map, to the sampling locations and to the
 * attention weights ("Deformable DETR" wiki page, "Deformable attention
 * module": the interpolation lets gradients reach the offsets; "Deformable
 * Attention" glossary page: the interpolation passes gradients on to the
 * offset prediction).  With g = grad_out[n,q,m*D:(m+1)*D] and corner weights w_j:
 *   grad_attention_weights = sum_j w_j <v_j, g>
 *   grad_value[corner j]  += A w_j g        (corners inside the level)
 *   grad_sampling_locations = A * (W_l, H_l) * sum_j (dw_j/dfx, dw_j/dfy) <v_j, g>
 * At a cell boundary the derivative of the cell chosen by floor() is taken.
 *
 *   grad_out                 device [N,Lq,M*D] fp32, 16-byte aligned
 *   grad_value               device [N,S,M,D] fp32 (fp32 for both value
 *                            dtypes), 16-byte aligned; zeroed by the call on
 *                            `stream`, then accumulated with atomics (the
 *                            summation order, and so the last bits, vary
 *                            from run to run)
 *   grad_sampling_locations  NULL or device [N,Lq,M,L,K,2] fp32 (written)
 *   grad_attention_weights   NULL or device [N,Lq,M,L,K] fp32 (written)
 *
 * Errors: as msda_forward (grad_value, grad_sampling_locations and
 * grad_attention_weights are outputs for the alias check).
 */
MSDA_API msda_status msda_backward(const void *value, msda_dtype value_dtype,
                          const int64_t *spatial_shapes,
                          const int64_t *level_start_index,
                          const float *sampling_locations,
                          const float *attention_weights, const float *grad_out,
                          float *grad_value, float *grad_sampling_locations,
                          float *grad_attention_weights, msda_dims dims,
                          msda_stream_t stream);

/*
 * Backward of msda_forward_fused, chained to the raw projection outputs.
 * The attention weights and sampling locations are recomputed from the
 * inputs exactly as msda_forward_fused forms them (bit for bit), the
 * gradients through the interpolation are formed as in msda_backward, and
 * the chain rule is applied inside the kernel ("Deformable DETR" wiki page,
 * "Multi-scale deformable attention" and "Variants"; the gradients reach the
 * 3MK projection through the offsets and the softmax):
 *   point reference (loc = ref + off / W_l):
 *     grad_offsets = grad_loc / W_l (per level),  grad_reference = sum of grad_loc
 *   box reference (loc = (cx, cy) + off * (w, h)):
 *     grad_offsets = grad_loc * (w, h),
 *     grad_reference = (sum grad_loc_x, sum grad_loc_y,
 *                       sum grad_loc_x * off_x, sum grad_loc_y * off_y)
 *   grad_logits = A * (grad_A - sum_j A_j grad_A_j)     (per head, over L*K)
 * where the sums run over the heads, levels and points of the query.
 *
 *   reference_points, reference_dim, offsets, logits  as msda_forward_fused
 *   grad_out                device [N,Lq,M*D] fp32, 16-byte aligned
 *   grad_value              device [N,S,M,D] fp32; zeroed, then accumulated
 *   grad_reference_points   NULL or device [N,Lq,reference_dim] fp32;
 *                           zeroed, then accumulated over heads (atomics)
 *   grad_offsets            NULL or device [N,Lq,M,L,K,2] fp32 (written)
 *   grad_logits             NULL or device [N,Lq,M,L,K] fp32 (written)
 *
 * Limits: as msda_forward_fused.  Errors: as msda_forward_fused; every
 * gradient buffer is an output for the alias check.
 */
MSDA_API msda_status msda_backward_fused(const void *value, msda_dtype value_dtype,
                                         const int64_t *spatial_shapes,
                                         const int64_t *level_start_index,
                                         const float *reference_points, int reference_dim,
                                         const float *offsets, const float *logits,
                                         const float *grad_out, float *grad_value,
                                         float *grad_reference_points, float *grad_offsets,
                                         float *grad_logits, msda_dims dims,
                                         msda_stream_t stream);

/*
 * Deformable groups ("Deformable Attention" glossary page, multi-head
 * paragraph: heads may be gathered into fewer groups whose members look up
 * the same key locations while keeping their own projections).  The M heads form `groups` groups of
 * Hg = M/groups consecutive heads (head m is in group m / Hg); the heads of a
 * group sample the same locations, each with its own attention weights and
 * its own value channels.  The four calls below are msda_forward,
 * msda_forward_fused, msda_backward and msda_backward_fused with every
 * per-location tensor indexed by group instead of head:
 *
 *   sampling_locations, offsets,
 *   sampling_locations_out, grad_sampling_locations, grad_offsets
 *                                 [N, Lq, groups, L, K, 2]
 *   attention_weights, logits, attention_weights_out, grad_attention_weights,
 *   grad_logits                   [N, Lq, M, L, K]      (per head, unchanged)
 *
 * The fused forward writes each group's locations once.  In the backward the
 * Hg heads of a group add into one location gradient: grad_sampling_locations
 * and grad_offsets are then zeroed by the call and accumulated with atomics
 * (groups < M; with groups == M they are written, as in the ungrouped calls,
 * which these equal).
 * Errors: as the ungrouped calls, plus MSDA_ERR_SHAPE unless
 * 1 <= groups <= M and groups divides M.
 */
MSDA_API msda_status msda_forward_grouped(const void *value, msda_dtype value_dtype,
                                          const int64_t *spatial_shapes,
                                          const int64_t *level_start_index,
                                          const float *sampling_locations,
                                          const float *attention_weights, float *out,
                                          msda_dims dims, int64_t groups, msda_stream_t stream);

MSDA_API msda_status msda_forward_fused_grouped(const void *value, msda_dtype value_dtype,
                                                const int64_t *spatial_shapes,
                                                const int64_t *level_start_index,
                                                const float *reference_points,
                                                int reference_dim, const float *offsets,
                                                const float *logits, float *out,
                                                float *sampling_locations_out,
                                                float *attention_weights_out, msda_dims dims,
                                                int64_t groups, msda_stream_t stream);

MSDA_API msda_status msda_backward_grouped(const void *value, msda_dtype value_dtype,
                                           const int64_t *spatial_shapes,
                                           const int64_t *level_start_index,
                                           const float *sampling_locations,
                                           const float *attention_weights,
                                           const float *grad_out, float *grad_value,
                                           float *grad_sampling_locations,
                                           float *grad_attention_weights, msda_dims dims,
                                           int64_t groups, msda_stream_t stream);

MSDA_API msda_status msda_backward_fused_grouped(const void *value, msda_dtype value_dtype,
                                                 const int64_t *spatial_shapes,
                                                 const int64_t *level_start_index,
                                                 const float *reference_points,
                                                 int reference_dim, const float *offsets,
                                                 const float *logits, const float *grad_out,
                                                 float *grad_value,
                                                 float *grad_reference_points,
                                                 float *grad_offsets, float *grad_logits,
                                                 msda_dims dims, int64_t groups,
                                                 msda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_H */
