// msda_api.cpp -- the C entry points: argument checks, then launches.
//
// Every check runs before any CUDA call, so a rejected call has no side
// effect at all (and the checks themselves work on a machine without a GPU).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "msda.h"
#include "msda_debug.h"
#include "msda_api_util.h"
#include "msda_internal.h"
#ifdef MSDA_CHECKED
#include "msda_checked.h"
#endif

namespace {

using msda::Levels;
using msda::kMaxLK;
using namespace msda::api;

constexpr int kAbiVersion = 10300;  // 1.3.0: value rows of any width (1.2.0: tiled entry points)

}  // namespace

namespace msda {
namespace api {

thread_local int g_last_cuda_error = 0;

// a * b with a, b >= 0; false if the product exceeds `limit`.
bool mul_le(int64_t a, int64_t b, int64_t limit, int64_t *out)
{
    if (a != 0 && b > limit / a) return false;
    *out = a * b;
    return *out <= limit;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(Span a, Span b)
{
    if (!a.p || !b.p || a.bytes <= 0 || b.bytes <= 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a.p);
    const uintptr_t pb = reinterpret_cast<uintptr_t>(b.p);
    return pa < pb + (uintptr_t)b.bytes && pb < pa + (uintptr_t)a.bytes;
}

// True if any output overlaps any input or another output.
bool any_alias(const Span *outs, int nout, const Span *ins, int nin)
{
    for (int i = 0; i < nout; ++i) {
        for (int j = 0; j < nin; ++j)
            if (overlap(outs[i], ins[j])) return true;
        for (int j = i + 1; j < nout; ++j)
            if (overlap(outs[i], outs[j])) return true;
    }
    return false;
}

// Dims, level metadata and size limits (no pointers).
msda_status check_dims(msda_dtype dt, const int64_t *shapes, const int64_t *starts,
                       const msda_dims &d, Problem *pr)
{
    if (!shapes || !starts) return MSDA_ERR_NULL;
    if (dt != MSDA_F32 && dt != MSDA_BF16) return MSDA_ERR_DTYPE;
    if (d.N < 0 || d.Lq < 0 || d.S < 0 || d.M < 1 || d.D < 1 || d.L < 1 || d.K < 1)
        return MSDA_ERR_SHAPE;
    if (d.L > msda::kMaxLevels || d.K > kMaxLK || d.L * d.K > kMaxLK)
        return MSDA_ERR_UNSUPPORTED;
    memset(&pr->lv, 0, sizeof pr->lv);
    int64_t acc = 0;
    for (int64_t l = 0; l < d.L; ++l) {
        const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
        if (H < 0 || W < 0) return MSDA_ERR_SHAPE;
        if (H > kI32Max || W > kI32Max) return MSDA_ERR_UNSUPPORTED;
        if (starts[l] != acc) return MSDA_ERR_LEVELS;
        acc += H * W;  // < 2^62: both factors < 2^31
        if (acc > kI32Max) return MSDA_ERR_UNSUPPORTED;
        pr->lv.H[l] = (int)H;
        pr->lv.W[l] = (int)W;
        pr->lv.start[l] = (int)starts[l];
    }
    if (acc != d.S) return MSDA_ERR_LEVELS;
    pr->esz = dt == MSDA_F32 ? 4 : 2;
    if (d.D > kI32Max) return MSDA_ERR_UNSUPPORTED;
    const int64_t rowbytes = d.D * pr->esz;
    if (rowbytes % 16 != 0) return MSDA_ERR_ALIGN;
    if (d.Lq > kI32Max || d.M > kI32Max) return MSDA_ERR_UNSUPPORTED;
    int64_t smd, md, t;
    if (!mul_le(d.M, d.D, kI32Max, &md) || !mul_le(d.S, md, kI32Max, &smd))
        return MSDA_ERR_UNSUPPORTED;  // row offsets inside one batch entry are int32
    if (!mul_le(d.N, smd, kGuard, &pr->n_value)) return MSDA_ERR_UNSUPPORTED;
    if (!mul_le(d.N, d.Lq, kGuard, &t) || !mul_le(t, d.M, kGuard, &pr->items))
        return MSDA_ERR_UNSUPPORTED;
    // the kernels split item indices (n, q, m) in 32 bits
    if (pr->items > kI32Max) return MSDA_ERR_UNSUPPORTED;
    if (!mul_le(pr->items, d.L * d.K * 2, kGuard, &t)) return MSDA_ERR_UNSUPPORTED;
    pr->samples = pr->items * d.L * d.K;
    pr->n_out = pr->items * d.D;
    pr->nchunks = (int)(rowbytes / 16);
    // one 16-byte chunk per lane; rows of more than 32 chunks take passes of 32
    int lanes = 1;
    while (lanes < pr->nchunks && lanes < 32) lanes <<= 1;
    pr->lanes = lanes;
    return MSDA_OK;
}

// Deformable groups: G groups of M/G consecutive heads share one set of
// sampling locations (G = M: every head has its own).
msda_status check_groups(const msda_dims &d, int64_t G, Problem *pr)
{
    if (G < 1 || G > d.M || d.M % G != 0) return MSDA_ERR_SHAPE;
    pr->lsamples = pr->samples / d.M * G;
    return MSDA_OK;
}

msda_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return MSDA_OK;
    g_last_cuda_error = (int)e;
    return MSDA_ERR_CUDA;
}

#ifdef MSDA_CHECKED
std::atomic<int64_t> g_check_limit{-1};
thread_local int64_t g_violation_count = 0;
thread_local int64_t g_violation_first = -1;
#endif

// Status of a launch.  The bounds-checked build also waits for the stream,
// reads the device word, and clears it if the kernel recorded a violation.
msda_status launched(cudaError_t e, cudaStream_t s)
{
    msda_status st = cuda_status(e);
#ifdef MSDA_CHECKED
    if (st != MSDA_OK) return st;
    unsigned long long *dw = msda::check_word();
    unsigned long long h[2] = {0, 0};
    st = cuda_status(cudaMemcpyAsync(h, dw, sizeof h, cudaMemcpyDeviceToHost, s));
    if (st == MSDA_OK) st = cuda_status(cudaStreamSynchronize(s));
    if (st != MSDA_OK || h[0] == 0) return st;
    g_violation_count = (int64_t)h[0];
    g_violation_first = (int64_t)h[1];
    st = cuda_status(cudaMemsetAsync(dw, 0, sizeof h, s));
    if (st == MSDA_OK) st = cuda_status(cudaStreamSynchronize(s));
    return st == MSDA_OK ? MSDA_ERR_DEVICE_CHECK : st;
#else
    (void)s;
    return st;
#endif
}

}  // namespace api
}  // namespace msda

extern "C" {

const char *msda_status_string(msda_status status)
{
    switch (status) {
    case MSDA_OK: return "MSDA_OK";
    case MSDA_ERR_NULL: return "MSDA_ERR_NULL: a required pointer is NULL";
    case MSDA_ERR_SHAPE: return "MSDA_ERR_SHAPE: a dimension is out of range";
    case MSDA_ERR_LEVELS:
        return "MSDA_ERR_LEVELS: spatial_shapes, level_start_index and S disagree";
    case MSDA_ERR_DTYPE: return "MSDA_ERR_DTYPE: unknown value dtype";
    case MSDA_ERR_ALIGN: return "MSDA_ERR_ALIGN: a pointer or row size breaks the alignment rule";
    case MSDA_ERR_ALIAS: return "MSDA_ERR_ALIAS: an output overlaps an input or another output";
    case MSDA_ERR_UNSUPPORTED: return "MSDA_ERR_UNSUPPORTED: outside this build's limits";
    case MSDA_ERR_CUDA: return "MSDA_ERR_CUDA: the CUDA runtime reported an error";
    case MSDA_ERR_DEVICE_CHECK:
        return "MSDA_ERR_DEVICE_CHECK: a bounds check skipped a value-map access";
    }
    return "MSDA_ERR_UNKNOWN";
}

int msda_abi_version(void) { return kAbiVersion; }

int msda_last_cuda_error(void) { return g_last_cuda_error; }

msda_status msda_level_start_index(const int64_t *spatial_shapes, int64_t L,
                                   int64_t *level_start_index, int64_t *S_out)
{
    if (!spatial_shapes || !level_start_index) return MSDA_ERR_NULL;
    if (L < 1) return MSDA_ERR_SHAPE;
    int64_t acc = 0;
    for (int64_t l = 0; l < L; ++l) {
        const int64_t H = spatial_shapes[2 * l], W = spatial_shapes[2 * l + 1];
        if (H < 0 || W < 0) return MSDA_ERR_SHAPE;
        int64_t hw;
        if (!mul_le(H, W, kGuard, &hw) || acc > kGuard - hw) return MSDA_ERR_UNSUPPORTED;
        level_start_index[l] = acc;
        acc += hw;
    }
    if (S_out) *S_out = acc;
    return MSDA_OK;
}

}  // extern "C"

namespace {

msda_status forward_impl(const void *value, msda_dtype value_dtype, const int64_t *spatial_shapes,
                         const int64_t *level_start_index, const float *sampling_locations,
                         const float *attention_weights, float *out, msda_dims d, int64_t G,
                         msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, G, &pr)) != MSDA_OK) return st;
    if (pr.n_out > 0 && (!sampling_locations || !attention_weights || !out))
        return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(out, 16) || !aligned(sampling_locations, 8) ||
        !aligned(attention_weights, 4))
        return MSDA_ERR_ALIGN;
    const Span outs[] = {{out, pr.n_out * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {sampling_locations, pr.lsamples * 8},
                        {attention_weights, pr.samples * 4}};
    if (any_alias(outs, 1, ins, 3)) return MSDA_ERR_ALIAS;
    if (pr.n_out == 0) return MSDA_OK;

    msda::FwdParams p;
    memset(&p, 0, sizeof p);
    p.value = value;
    p.loc = sampling_locations;
    p.attn = attention_weights;
    p.out = out;
    set_dims(&p, d, G, pr);
    if ((st = set_checks(&p, pr)) != MSDA_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launched(msda::launch_forward(p, value_dtype == MSDA_BF16, false, pr.lanes, s), s);
}

msda_status forward_fused_impl(const void *value, msda_dtype value_dtype,
                               const int64_t *spatial_shapes, const int64_t *level_start_index,
                               const float *reference_points, int reference_dim,
                               const float *offsets, const float *logits, float *out,
                               float *sampling_locations_out, float *attention_weights_out,
                               msda_dims d, int64_t G, msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, G, &pr)) != MSDA_OK) return st;
    if (reference_dim != 2 && reference_dim != 4) return MSDA_ERR_SHAPE;
    if (pr.n_out > 0 && (!reference_points || !offsets || !logits || !out))
        return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(out, 16) || !aligned(reference_points, 8) ||
        !aligned(offsets, 8) || !aligned(logits, 4) || !aligned(sampling_locations_out, 8) ||
        !aligned(attention_weights_out, 4))
        return MSDA_ERR_ALIGN;
    const int64_t nq = pr.items / d.M;
    const Span outs[] = {{out, pr.n_out * 4},
                         {sampling_locations_out, pr.lsamples * 8},
                         {attention_weights_out, pr.samples * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {reference_points, nq * reference_dim * 4},
                        {offsets, pr.lsamples * 8},
                        {logits, pr.samples * 4}};
    if (any_alias(outs, 3, ins, 4)) return MSDA_ERR_ALIAS;
    if (pr.n_out == 0) return MSDA_OK;

    msda::FwdParams p;
    memset(&p, 0, sizeof p);
    p.value = value;
    p.ref = reference_points;
    p.ref_dim = reference_dim;
    p.off = offsets;
    p.logits = logits;
    p.out = out;
    p.loc_out = sampling_locations_out;
    p.attn_out = attention_weights_out;
    set_dims(&p, d, G, pr);
    if ((st = set_checks(&p, pr)) != MSDA_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launched(msda::launch_forward(p, value_dtype == MSDA_BF16, true, pr.lanes, s), s);
}

msda_status backward_impl(const void *value, msda_dtype value_dtype,
                          const int64_t *spatial_shapes, const int64_t *level_start_index,
                          const float *sampling_locations, const float *attention_weights,
                          const float *grad_out, float *grad_value,
                          float *grad_sampling_locations, float *grad_attention_weights,
                          msda_dims d, int64_t G, msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, G, &pr)) != MSDA_OK) return st;
    if (pr.n_value > 0 && !grad_value) return MSDA_ERR_NULL;
    if (pr.n_out > 0 && (!sampling_locations || !attention_weights || !grad_out))
        return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(grad_out, 16) || !aligned(grad_value, 16) ||
        !aligned(sampling_locations, 8) || !aligned(attention_weights, 4) ||
        !aligned(grad_sampling_locations, 8) || !aligned(grad_attention_weights, 4))
        return MSDA_ERR_ALIGN;
    const Span outs[] = {{grad_value, pr.n_value * 4},
                         {grad_sampling_locations, pr.lsamples * 8},
                         {grad_attention_weights, pr.samples * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {sampling_locations, pr.lsamples * 8},
                        {attention_weights, pr.samples * 4},
                        {grad_out, pr.n_out * 4}};
    if (any_alias(outs, 3, ins, 4)) return MSDA_ERR_ALIAS;

    msda::BwdParams p;
    memset(&p, 0, sizeof p);
    p.value = value;
    p.loc = sampling_locations;
    p.attn = attention_weights;
    p.grad_out = grad_out;
    p.grad_value = grad_value;
    p.grad_loc = grad_sampling_locations;
    p.grad_attn = grad_attention_weights;
    set_dims(&p, d, G, pr);
    // before any device work, so that a failure here has launched nothing
    // (a problem with no queries launches no kernel and needs no checks)
    if (pr.n_out > 0 && (st = set_checks(&p, pr)) != MSDA_OK) return st;

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pr.n_value > 0) {
        st = cuda_status(cudaMemsetAsync(grad_value, 0, (size_t)pr.n_value * 4, s));
        if (st != MSDA_OK) return st;
    }
    if (grad_sampling_locations && G < d.M && pr.lsamples > 0) {  // heads of a group add up
        st = cuda_status(
            cudaMemsetAsync(grad_sampling_locations, 0, (size_t)pr.lsamples * 8, s));
        if (st != MSDA_OK) return st;
    }
    if (pr.n_out == 0) return MSDA_OK;
    return launched(msda::launch_backward(p, value_dtype == MSDA_BF16, pr.lanes, s), s);
}

msda_status backward_fused_impl(const void *value, msda_dtype value_dtype,
                                const int64_t *spatial_shapes, const int64_t *level_start_index,
                                const float *reference_points, int reference_dim,
                                const float *offsets, const float *logits,
                                const float *grad_out, float *grad_value,
                                float *grad_reference_points, float *grad_offsets,
                                float *grad_logits, msda_dims d, int64_t G, msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, G, &pr)) != MSDA_OK) return st;
    if (reference_dim != 2 && reference_dim != 4) return MSDA_ERR_SHAPE;
    if (pr.n_value > 0 && !grad_value) return MSDA_ERR_NULL;
    if (pr.n_out > 0 && (!reference_points || !offsets || !logits || !grad_out))
        return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(grad_out, 16) || !aligned(grad_value, 16) ||
        !aligned(reference_points, 8) || !aligned(offsets, 8) || !aligned(logits, 4) ||
        !aligned(grad_reference_points, 8) || !aligned(grad_offsets, 8) ||
        !aligned(grad_logits, 4))
        return MSDA_ERR_ALIGN;
    const int64_t nq = pr.items / d.M;
    const Span outs[] = {{grad_value, pr.n_value * 4},
                         {grad_reference_points, nq * reference_dim * 4},
                         {grad_offsets, pr.lsamples * 8},
                         {grad_logits, pr.samples * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {reference_points, nq * reference_dim * 4},
                        {offsets, pr.lsamples * 8},
                        {logits, pr.samples * 4},
                        {grad_out, pr.n_out * 4}};
    if (any_alias(outs, 4, ins, 5)) return MSDA_ERR_ALIAS;

    msda::BwdParams p;
    memset(&p, 0, sizeof p);
    p.value = value;
    p.ref = reference_points;
    p.ref_dim = reference_dim;
    p.off = offsets;
    p.logits = logits;
    p.grad_out = grad_out;
    p.grad_value = grad_value;
    p.grad_ref = grad_reference_points;
    p.grad_off = grad_offsets;
    p.grad_logits = grad_logits;
    set_dims(&p, d, G, pr);
    // before any device work, so that a failure here has launched nothing
    // (a problem with no queries launches no kernel and needs no checks)
    if (pr.n_out > 0 && (st = set_checks(&p, pr)) != MSDA_OK) return st;

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pr.n_value > 0) {
        st = cuda_status(cudaMemsetAsync(grad_value, 0, (size_t)pr.n_value * 4, s));
        if (st != MSDA_OK) return st;
    }
    if (grad_reference_points && nq > 0) {
        st = cuda_status(
            cudaMemsetAsync(grad_reference_points, 0, (size_t)(nq * reference_dim) * 4, s));
        if (st != MSDA_OK) return st;
    }
    if (grad_offsets && G < d.M && pr.lsamples > 0) {  // heads of a group add up
        st = cuda_status(cudaMemsetAsync(grad_offsets, 0, (size_t)pr.lsamples * 8, s));
        if (st != MSDA_OK) return st;
    }
    if (pr.n_out == 0) return MSDA_OK;
    return launched(msda::launch_backward_fused(p, value_dtype == MSDA_BF16, pr.lanes, s), s);
}

}  // namespace

extern "C" {

msda_status msda_forward(const void *value, msda_dtype value_dtype,
                         const int64_t *spatial_shapes, const int64_t *level_start_index,
                         const float *sampling_locations, const float *attention_weights,
                         float *out, msda_dims d, msda_stream_t stream)
{
    return forward_impl(value, value_dtype, spatial_shapes, level_start_index,
                        sampling_locations, attention_weights, out, d, d.M, stream);
}

msda_status msda_forward_grouped(const void *value, msda_dtype value_dtype,
                                 const int64_t *spatial_shapes,
                                 const int64_t *level_start_index,
                                 const float *sampling_locations,
                                 const float *attention_weights, float *out, msda_dims d,
                                 int64_t groups, msda_stream_t stream)
{
    return forward_impl(value, value_dtype, spatial_shapes, level_start_index,
                        sampling_locations, attention_weights, out, d, groups, stream);
}

msda_status msda_forward_fused(const void *value, msda_dtype value_dtype,
                               const int64_t *spatial_shapes,
                               const int64_t *level_start_index,
                               const float *reference_points, int reference_dim,
                               const float *offsets, const float *logits, float *out,
                               float *sampling_locations_out, float *attention_weights_out,
                               msda_dims d, msda_stream_t stream)
{
    return forward_fused_impl(value, value_dtype, spatial_shapes, level_start_index,
                              reference_points, reference_dim, offsets, logits, out,
                              sampling_locations_out, attention_weights_out, d, d.M, stream);
}

msda_status msda_forward_fused_grouped(const void *value, msda_dtype value_dtype,
                                       const int64_t *spatial_shapes,
                                       const int64_t *level_start_index,
                                       const float *reference_points, int reference_dim,
                                       const float *offsets, const float *logits, float *out,
                                       float *sampling_locations_out,
                                       float *attention_weights_out, msda_dims d,
                                       int64_t groups, msda_stream_t stream)
{
    return forward_fused_impl(value, value_dtype, spatial_shapes, level_start_index,
                              reference_points, reference_dim, offsets, logits, out,
                              sampling_locations_out, attention_weights_out, d, groups, stream);
}

msda_status msda_backward(const void *value, msda_dtype value_dtype,
                          const int64_t *spatial_shapes, const int64_t *level_start_index,
                          const float *sampling_locations, const float *attention_weights,
                          const float *grad_out, float *grad_value,
                          float *grad_sampling_locations, float *grad_attention_weights,
                          msda_dims d, msda_stream_t stream)
{
    return backward_impl(value, value_dtype, spatial_shapes, level_start_index,
                         sampling_locations, attention_weights, grad_out, grad_value,
                         grad_sampling_locations, grad_attention_weights, d, d.M, stream);
}

msda_status msda_backward_grouped(const void *value, msda_dtype value_dtype,
                                  const int64_t *spatial_shapes,
                                  const int64_t *level_start_index,
                                  const float *sampling_locations,
                                  const float *attention_weights, const float *grad_out,
                                  float *grad_value, float *grad_sampling_locations,
                                  float *grad_attention_weights, msda_dims d, int64_t groups,
                                  msda_stream_t stream)
{
    return backward_impl(value, value_dtype, spatial_shapes, level_start_index,
                         sampling_locations, attention_weights, grad_out, grad_value,
                         grad_sampling_locations, grad_attention_weights, d, groups, stream);
}

msda_status msda_backward_fused(const void *value, msda_dtype value_dtype,
                                const int64_t *spatial_shapes,
                                const int64_t *level_start_index,
                                const float *reference_points, int reference_dim,
                                const float *offsets, const float *logits,
                                const float *grad_out, float *grad_value,
                                float *grad_reference_points, float *grad_offsets,
                                float *grad_logits, msda_dims d, msda_stream_t stream)
{
    return backward_fused_impl(value, value_dtype, spatial_shapes, level_start_index,
                               reference_points, reference_dim, offsets, logits, grad_out,
                               grad_value, grad_reference_points, grad_offsets, grad_logits, d,
                               d.M, stream);
}

msda_status msda_backward_fused_grouped(const void *value, msda_dtype value_dtype,
                                        const int64_t *spatial_shapes,
                                        const int64_t *level_start_index,
                                        const float *reference_points, int reference_dim,
                                        const float *offsets, const float *logits,
                                        const float *grad_out, float *grad_value,
                                        float *grad_reference_points, float *grad_offsets,
                                        float *grad_logits, msda_dims d, int64_t groups,
                                        msda_stream_t stream)
{
    return backward_fused_impl(value, value_dtype, spatial_shapes, level_start_index,
                               reference_points, reference_dim, offsets, logits, grad_out,
                               grad_value, grad_reference_points, grad_offsets, grad_logits, d,
                               groups, stream);
}

msda_status msda_debug_sample_points(const int64_t *spatial_shapes,
                                     const int64_t *level_start_index,
                                     const float *sampling_locations, msda_dims d,
                                     int32_t *valid, int32_t *x0, int32_t *y0, float *x,
                                     float *y, int64_t *rows, msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(MSDA_F32, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if (pr.samples > 0 && (!sampling_locations || !valid || !x0 || !y0 || !x || !y || !rows))
        return MSDA_ERR_NULL;
    if (!aligned(sampling_locations, 8) || !aligned(valid, 4) || !aligned(x0, 4) ||
        !aligned(y0, 4) || !aligned(x, 4) || !aligned(y, 4) || !aligned(rows, 8))
        return MSDA_ERR_ALIGN;
    const int64_t n = pr.samples;
    const Span outs[] = {{valid, n * 4}, {x0, n * 4}, {y0, n * 4},
                         {x, n * 4},     {y, n * 4},  {rows, n * 32}};
    const Span ins[] = {{sampling_locations, n * 8}};
    if (any_alias(outs, 6, ins, 1)) return MSDA_ERR_ALIAS;
    if (n == 0) return MSDA_OK;
    msda::PointsParams p;
    memset(&p, 0, sizeof p);
    p.loc = sampling_locations;
    p.valid = valid;
    p.x0 = x0;
    p.y0 = y0;
    p.x = x;
    p.y = y;
    p.rows = rows;
    p.samples = n;
    p.L = (int)d.L;
    p.K = (int)d.K;
    p.lv = pr.lv;
    return cuda_status(msda::launch_sample_points(p, static_cast<cudaStream_t>(stream)));
}

msda_status msda_debug_row_traffic(int mode, const void *value, msda_dtype value_dtype,
                                   float *grad, int64_t n_value, const int32_t *row_offsets,
                                   int64_t n_rows, float *sink, int64_t sink_len, int depth,
                                   int ctas, msda_stream_t stream)
{
    if (value_dtype != MSDA_F32 && value_dtype != MSDA_BF16) return MSDA_ERR_DTYPE;
    if (mode < 0 || mode > 2 || n_rows < 0 || n_value < 32 || sink_len < 0)
        return MSDA_ERR_SHAPE;
    if (depth != 0 && depth != 2 && depth != 4 && depth != 8 && depth != 16)
        return MSDA_ERR_SHAPE;
    if (n_rows > 0 && !row_offsets) return MSDA_ERR_NULL;
    if (mode != 1 && !value) return MSDA_ERR_NULL;
    if (mode != 0 && !grad) return MSDA_ERR_NULL;
    if (sink_len > 0 && !sink) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(grad, 16) || !aligned(row_offsets, 4) ||
        !aligned(sink, 4))
        return MSDA_ERR_ALIGN;
    const Span outs[] = {{grad, n_value * 4}, {sink, sink_len * 4}};
    const int64_t vbytes = value_dtype == MSDA_BF16 ? 2 : 4;
    const Span ins[] = {{value, n_value * vbytes}, {row_offsets, n_rows * 4}};
    if (any_alias(outs, 2, ins, 2)) return MSDA_ERR_ALIAS;
    if (n_rows == 0) return MSDA_OK;
    msda::TrafficParams p;
    memset(&p, 0, sizeof p);
    p.value = value;
    p.bf16 = value_dtype == MSDA_BF16;
    p.grad = grad;
    p.rows = row_offsets;
    p.n_rows = n_rows;
    p.n_value = n_value;
    p.sink = sink;
    p.sink_len = sink_len;
    return cuda_status(
        msda::launch_row_traffic(p, mode, depth, ctas, static_cast<cudaStream_t>(stream)));
}

#ifdef MSDA_CHECKED
msda_status msda_checked_set_limit(int64_t value_elements)
{
    g_check_limit.store(value_elements < 0 ? -1 : value_elements);
    return MSDA_OK;
}

msda_status msda_checked_last_violation(int64_t *count, int64_t *first_element)
{
    if (count) *count = g_violation_count;
    if (first_element) *first_element = g_violation_first;
    return MSDA_OK;
}
#endif

}  // extern "C"
