// msda_noalloc.cu -- the allocation-free form of the tiled fused forward
// (msda_forward_fused_tiled_noalloc in msda_tiled.h).
//
// The tiled forward needs a tile plan in device memory.  Some callers cannot
// hand the library any device memory beyond their inputs and outputs: a
// plugin whose host framework owns every device allocation and offers no
// workspace, or a caller on a latency-critical path that may not call
// cudaMalloc, which can synchronise the device and can fail under memory
// pressure.  For them this file keeps the plan in a file-scope device array
// of fixed size (every GPU that loads the library holds it until the process
// exits) and builds it there on every call.
//
// The array's name, in host code, stands for a host-side symbol, not a device
// address: a kernel given it would fault, or silently use the wrong memory.
// So the first call on each device asks the runtime for the array's device
// address (cudaGetSymbolAddress, with that device current) and every call on
// that device passes the address it got.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "msda.h"
#include "msda_api_util.h"
#include "msda_tiled.h"

namespace {

// Largest tile plan the array holds: 4 MiB, enough for a million queries per
// call (a plan takes 4 bytes per query and 4 per cell and batch entry).
constexpr int64_t kNoAllocPlanBytes = int64_t(4) << 20;

static __device__ __align__(256) unsigned char g_noalloc_plan[kNoAllocPlanBytes];

constexpr int kMaxDevices = 64;

// The array's device address on the current device, looked up once per
// device; nullptr (with the CUDA error recorded) if the runtime cannot give it.
void *plan_scratch(cudaError_t *err)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_noalloc_plan);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

// The fused forward's argument checks (msda_forward_fused), run before the
// plan is built so that a rejected call launches nothing.
msda_status check_forward_args(const void *value, msda_dtype dt, const int64_t *shapes,
                               const int64_t *starts, const float *ref, int ref_dim,
                               const float *off, const float *logits, const float *out,
                               const float *loc_out, const float *attn_out, const msda_dims &d)
{
    using namespace msda::api;
    Problem pr;
    msda_status st = check_dims(dt, shapes, starts, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, d.M, &pr)) != MSDA_OK) return st;
    if (ref_dim != 2 && ref_dim != 4) return MSDA_ERR_SHAPE;
    if (pr.n_out > 0 && (!ref || !off || !logits || !out)) return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(out, 16) || !aligned(ref, 8) || !aligned(off, 8) ||
        !aligned(logits, 4) || !aligned(loc_out, 8) || !aligned(attn_out, 4))
        return MSDA_ERR_ALIGN;
    const int64_t nq = pr.items / d.M;
    const Span outs[] = {{out, pr.n_out * 4}, {loc_out, pr.lsamples * 8},
                         {attn_out, pr.samples * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {ref, nq * ref_dim * 4},
                        {off, pr.lsamples * 8},
                        {logits, pr.samples * 4}};
    if (any_alias(outs, 3, ins, 4)) return MSDA_ERR_ALIAS;
    return MSDA_OK;
}

}  // namespace

extern "C" {

msda_status msda_forward_fused_tiled_noalloc(const void *value, msda_dtype value_dtype,
                                             const int64_t *spatial_shapes,
                                             const int64_t *level_start_index,
                                             const float *reference_points, int reference_dim,
                                             const float *offsets, const float *logits,
                                             float *out, float *sampling_locations_out,
                                             float *attention_weights_out, msda_dims dims,
                                             int halo, int ctas_per_sm, msda_stream_t stream)
{
    // the plan's description: host arithmetic only
    msda_tile_plan plan;
    msda_status st = msda_tile_plan_init(value_dtype, spatial_shapes, level_start_index, dims,
                                         halo, ctas_per_sm, &plan);
    if (st != MSDA_OK) return st;
    if (plan.device_bytes > kNoAllocPlanBytes) return MSDA_ERR_UNSUPPORTED;
    st = check_forward_args(value, value_dtype, spatial_shapes, level_start_index,
                            reference_points, reference_dim, offsets, logits, out,
                            sampling_locations_out, attention_weights_out, dims);
    if (st != MSDA_OK) return st;
    if (dims.N == 0 || dims.Lq == 0) {
        // nothing to sort or compute; the tiled forward checks the rest
        return msda_forward_fused_tiled(value, value_dtype, spatial_shapes, level_start_index,
                                        reference_points, reference_dim, offsets, logits, out,
                                        sampling_locations_out, attention_weights_out, dims,
                                        &plan, nullptr, stream);
    }
    cudaError_t err = cudaSuccess;
    void *scratch = plan_scratch(&err);
    if (!scratch) return msda::api::cuda_status(err != cudaSuccess ? err : cudaErrorUnknown);
    // The build writes every cell start and every sorted query before the
    // forward reads them, so nothing left in the array by an earlier call
    // needs clearing.
    st = msda_tile_plan_build(&plan, reference_points, reference_dim, scratch, stream);
    if (st != MSDA_OK) return st;
    return msda_forward_fused_tiled(value, value_dtype, spatial_shapes, level_start_index,
                                    reference_points, reference_dim, offsets, logits, out,
                                    sampling_locations_out, attention_weights_out, dims, &plan,
                                    scratch, stream);
}

}  // extern "C"
