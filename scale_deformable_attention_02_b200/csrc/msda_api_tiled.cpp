// msda_api_tiled.cpp -- the C entry points of msda_tiled.h: tile plans and
// the tiled forward and backward calls.  As in msda_api.cpp, every argument
// check runs before any CUDA call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "msda.h"
#include "msda_api_util.h"
#include "msda_debug.h"
#include "msda_internal.h"
#include "msda_tiled.h"

using namespace msda::api;

namespace {

static_assert(MSDA_TILE_MAX_LEVELS == msda::kTileLevels, "one level limit");

// Shared memory of one B200 SM, and what each resident CTA reserves.
constexpr int64_t kSmemPerSM = 233472;
constexpr int64_t kSmemPerCtaMax = 232448;
constexpr int64_t kSmemReserved = 1024;
// Static shared memory of the tiled kernels (corner entries, barrier) and
// the 128 bytes that align the windows, bound.
constexpr int64_t kTiledStatic = 14 * 1024;
constexpr int kMaxHalo = 64;
// Work units (batch entry, cell, head) per resident CTA the grid aims for.
constexpr int64_t kUnitsPerCta = 4;
constexpr int64_t kDesignSMs = 148;
constexpr int kMaxBox = 256;  // tensor-copy box limit per dimension

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Window bytes per level and in all, for a grid of gx x gy cells.
struct Windows {
    int ww[msda::kTileLevels], wh[msda::kTileLevels];
    int64_t soff[msda::kTileLevels];
    int64_t bytes;
};

Windows windows_for(const int64_t *shapes, int64_t L, int gx, int gy, int halo, int64_t rowb)
{
    Windows w;
    memset(&w, 0, sizeof w);
    int64_t off = 0;
    for (int64_t l = 0; l < L; ++l) {
        const int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
        w.soff[l] = off;
        if (H <= 0 || W <= 0) continue;  // empty level: nothing to stage
        // the cell's extent on this level, the halo and one corner on each side,
        // never more than the level and its one-pixel zero border
        int64_t bw = (W + gx - 1) / gx + 2 * (int64_t)halo + 2;
        int64_t bh = (H + gy - 1) / gy + 2 * (int64_t)halo + 2;
        if (bw > W + 2) bw = W + 2;
        if (bh > H + 2) bh = H + 2;
        if (bw > kMaxBox) bw = kMaxBox;
        if (bh > kMaxBox) bh = kMaxBox;
        w.ww[l] = (int)bw;
        w.wh[l] = (int)bh;
        off += round_up(bw * bh * rowb, 128);
    }
    w.bytes = off;
    return w;
}

bool same_plan_problem(const msda_tile_plan *pl, msda_dtype dt, const int64_t *shapes,
                       const msda_dims &d)
{
    if (pl->N != d.N || pl->Lq != d.Lq || pl->S != d.S || pl->L != d.L || pl->D != d.D ||
        pl->value_dtype != (int32_t)dt)
        return false;
    for (int64_t i = 0; i < 2 * d.L; ++i)
        if (pl->shapes[i] != shapes[i]) return false;
    return true;
}

// The tiled kernels' own limits, beyond check_dims.
msda_status check_tiled(const msda_dims &d, const int64_t *shapes, const Problem &pr)
{
    if (d.L > msda::kTileLevels || d.L * d.K > 32) return MSDA_ERR_UNSUPPORTED;
    if (d.D * pr.esz > 128) return MSDA_ERR_UNSUPPORTED;
    for (int64_t l = 0; l < d.L; ++l)
        if (shapes[2 * l] >= (1 << 15) || shapes[2 * l + 1] >= (1 << 15))
            return MSDA_ERR_UNSUPPORTED;
    return MSDA_OK;
}

// Dynamic shared memory a tiled CTA may give its windows, with ctas_per_sm
// CTAs resident per SM.
int64_t smem_budget(int ctas_per_sm)
{
    int64_t per_cta = kSmemPerSM / ctas_per_sm - kSmemReserved;
    if (per_cta > kSmemPerCtaMax) per_cta = kSmemPerCtaMax;
    return per_cta - kTiledStatic;
}

int64_t plan_device_bytes(int64_t N, int64_t Lq, int64_t G)
{
    return round_up(round_up(N * (G + 1) * 4, 256) + N * Lq * 4, 256);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The value map of each staged level as a 5-d tensor (D, M, W_l, H_l, N),
// boxes of one head's window.
msda_status encode_maps(CUtensorMap *maps, const void *value, msda_dtype dt,
                        const msda_dims &d, const Problem &pr, const msda_tile_plan *pl)
{
    auto fn = encode_fn();
    if (!fn) return cuda_status(cudaErrorNotSupported);
    const int64_t esz = pr.esz;
    for (int64_t l = 0; l < d.L; ++l) {
        memset(&maps[l], 0, sizeof(CUtensorMap));
        if (pl->window_w[l] == 0) continue;
        const int64_t H = pl->shapes[2 * l], W = pl->shapes[2 * l + 1];
        const char *base = static_cast<const char *>(value) +
                           (int64_t)pr.lv.start[l] * d.M * d.D * esz;
        cuuint64_t dims[5] = {(cuuint64_t)d.D, (cuuint64_t)d.M, (cuuint64_t)W, (cuuint64_t)H,
                              (cuuint64_t)d.N};
        cuuint64_t strides[4] = {(cuuint64_t)(d.D * esz), (cuuint64_t)(d.M * d.D * esz),
                                 (cuuint64_t)(W * d.M * d.D * esz),
                                 (cuuint64_t)(d.S * d.M * d.D * esz)};
        cuuint32_t box[5] = {(cuuint32_t)d.D, 1, (cuuint32_t)pl->window_w[l],
                             (cuuint32_t)pl->window_h[l], 1};
        cuuint32_t estr[5] = {1, 1, 1, 1, 1};
        const CUresult r = fn(&maps[l],
                              dt == MSDA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                              5, const_cast<char *>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cuda_status(cudaErrorInvalidValue);
    }
    return MSDA_OK;
}

// The device view of a checked plan.
msda::TileView tile_view(const msda_tile_plan *pl, const void *buf, const msda_dims &d)
{
    msda::TileView t;
    memset(&t, 0, sizeof t);
    const int64_t G = (int64_t)pl->grid_x * pl->grid_y;
    t.cell_start = static_cast<const int *>(buf);
    t.perm = reinterpret_cast<const int *>(static_cast<const char *>(buf) +
                                           round_up(d.N * (G + 1) * 4, 256));
    t.gx = pl->grid_x;
    t.gy = pl->grid_y;
    t.G = (int)G;
    t.halo = pl->halo;
    t.dG = msda::make_fastdiv((unsigned)G);
    int64_t off = 0, tx = 0;
    for (int64_t l = 0; l < d.L; ++l) {
        t.ww[l] = pl->window_w[l];
        t.wh[l] = pl->window_h[l];
        t.soff[l] = (int)off;
        const int64_t b = (int64_t)pl->window_w[l] * pl->window_h[l] * d.D *
                          (pl->value_dtype == MSDA_BF16 ? 2 : 4);
        off += round_up(b, 128);
        tx += b;
    }
    t.window_tx = (unsigned)tx;
    t.units = (int)(d.N * G * d.M);
    t.stall = msda::stall_word();
    return t;
}

// Checks shared by the tiled calls: the plan matches, the buffer is there.
msda_status check_plan_args(const msda_tile_plan *pl, const void *buf, msda_dtype dt,
                            const int64_t *shapes, const msda_dims &d, const Problem &pr)
{
    if (!pl) return MSDA_ERR_NULL;
    msda_status st = check_tiled(d, shapes, pr);
    if (st != MSDA_OK) return st;
    if (!same_plan_problem(pl, dt, shapes, d)) return MSDA_ERR_SHAPE;
    // the grid, the windows and the sizes must be what msda_tile_plan_init
    // gives for this grid, so that no kernel can leave its shared memory
    if (pl->grid_x < 1 || pl->grid_y < 1 ||
        (int64_t)pl->grid_x * pl->grid_y > msda::kTileMaxCells || pl->halo < 0 ||
        pl->halo > kMaxHalo || pl->ctas_per_sm < 1 || pl->ctas_per_sm > 3)
        return MSDA_ERR_SHAPE;
    const Windows w = windows_for(shapes, d.L, pl->grid_x, pl->grid_y, pl->halo, d.D * pr.esz);
    if (w.bytes != pl->window_bytes || w.bytes > smem_budget(pl->ctas_per_sm) ||
        pl->device_bytes != plan_device_bytes(d.N, d.Lq, (int64_t)pl->grid_x * pl->grid_y))
        return MSDA_ERR_SHAPE;
    for (int64_t l = 0; l < d.L; ++l)
        if (w.ww[l] != pl->window_w[l] || w.wh[l] != pl->window_h[l]) return MSDA_ERR_SHAPE;
    if (pr.n_out > 0 && !buf) return MSDA_ERR_NULL;
    if (!aligned(buf, 16)) return MSDA_ERR_ALIGN;
    // units N*G*M are counted in 32 bits
    if (d.N * (int64_t)pl->grid_x * pl->grid_y * d.M > kI32Max) return MSDA_ERR_UNSUPPORTED;
    return MSDA_OK;
}

msda_status launch_fwd_tiled(const void *value, msda_dtype dt, const msda_dims &d,
                             const Problem &pr, const msda_tile_plan *pl, const void *buf,
                             msda::FwdParams &f, bool fused, cudaStream_t s)
{
    msda_status st = set_checks(&f, pr);
    if (st != MSDA_OK) return st;
    msda::FwdTiledParams p;
    memset(&p, 0, sizeof p);
    if ((st = encode_maps(p.maps, value, dt, d, pr, pl)) != MSDA_OK) return st;
    p.f = f;
    p.t = tile_view(pl, buf, d);
    // the windows, plus 128 bytes to put their base on a 128-byte boundary
    const int dyn = (int)round_up(pl->window_bytes, 128) + 128;
    return launched(msda::launch_forward_tiled(p, dt == MSDA_BF16, fused, pl->ctas_per_sm, dyn, s),
                    s);
}

// The tiled backward's shared-memory layout after the windows, for the
// largest chunk of queries (a multiple of 32, at most 512) that fits one CTA
// per SM.  False if not even 32 queries fit, or if a row needs more than
// eight four-element lanes (D > 32): the call then runs the untiled backward,
// which computes the same gradients.
bool backward_layout(msda::BwdTiledParams *p, const msda_tile_plan *pl, const msda_dims &d,
                     bool bf16, bool fused, int *dyn)
{
    const int LK = (int)(d.L * d.K);
    if (d.D % 4 != 0 || d.D > 32) return false;  // four-element lanes, at most eight a row
    const int stat = msda::backward_tiled_static_smem(bf16, fused, (int)d.D, LK);
    if (stat < 0) return false;
    int keys = 0;
    for (int64_t l = 0; l < d.L; ++l) {
        p->roff[l] = keys;
        keys += pl->window_w[l] * pl->window_h[l];
    }
    p->roff[d.L] = keys;
    if (keys >= (1 << 16)) return false;  // records keep the pixel in 16 bits
    p->keys = keys;
    for (int T = 512; T >= 32; T -= 32) {
        // the chunk's sorted (query, coefficient) entries, four per sample at
        // most, take the windows' place after phase A
        if ((int64_t)T * LK * 4 * 8 > pl->window_bytes) continue;
        int64_t off = round_up(pl->window_bytes, 128);
        p->off_g = (int)off;
        off = round_up(off + (int64_t)T * d.D * 4, 16);
        p->off_rec = (int)off;
        off = round_up(off + (int64_t)T * LK * 16, 16);
        p->off_start = (int)off;
        off = round_up(off + (int64_t)(keys + 1) * 4, 16);
        p->off_cursor = (int)off;
        off = round_up(off + (int64_t)keys * 4, 16);
        p->off_queue = (int)off;
        off = round_up(off + (int64_t)T * 4, 16) + 128;  // + the window base alignment
        if (off + stat <= kSmemPerCtaMax) {
            p->T = T;
            *dyn = (int)off;
            return true;
        }
    }
    return false;
}

}  // namespace

extern "C" {

msda_status msda_tile_plan_init(msda_dtype value_dtype, const int64_t *spatial_shapes,
                                const int64_t *level_start_index, msda_dims d, int halo,
                                int ctas_per_sm, msda_tile_plan *plan)
{
    if (!plan) return MSDA_ERR_NULL;
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if (halo < 0 || halo > kMaxHalo) return MSDA_ERR_SHAPE;
    if (ctas_per_sm == 0) ctas_per_sm = 2;
    if (ctas_per_sm < 1 || ctas_per_sm > 3) return MSDA_ERR_SHAPE;
    if ((st = check_tiled(d, spatial_shapes, pr)) != MSDA_OK) return st;
    const int64_t rowb = d.D * pr.esz;
    const int64_t budget = smem_budget(ctas_per_sm);
    // the level with the most pixels sets the cells' aspect: square in its pixels
    int64_t ref_l = 0;
    for (int64_t l = 1; l < d.L; ++l)
        if (spatial_shapes[2 * l] * spatial_shapes[2 * l + 1] >
            spatial_shapes[2 * ref_l] * spatial_shapes[2 * ref_l + 1])
            ref_l = l;
    const double H0 = (double)(spatial_shapes[2 * ref_l] > 0 ? spatial_shapes[2 * ref_l] : 1);
    const double W0 =
        (double)(spatial_shapes[2 * ref_l + 1] > 0 ? spatial_shapes[2 * ref_l + 1] : 1);
    // The coarsest grid whose windows fit (fewest cells, so fewest window
    // copies), refined until there are kUnitsPerCta work units per resident
    // CTA of a 148-SM B200, so that the last wave of units is short.  Finer
    // grids have smaller windows, so they fit too.
    int best_gx = 0, best_gy = 0;
    const int64_t want_units = kUnitsPerCta * kDesignSMs * ctas_per_sm;
    for (int gx = 1; gx <= kMaxBox * 2; ++gx) {
        int gy = (int)lround(gx * H0 / W0);
        if (gy < 1) gy = 1;
        if ((int64_t)gx * gy > msda::kTileMaxCells) break;
        const Windows w = windows_for(spatial_shapes, d.L, gx, gy, halo, rowb);
        if (w.bytes > budget) continue;
        best_gx = gx;
        best_gy = gy;
        if (d.N * (int64_t)gx * gy * d.M >= want_units) break;
    }
    if (best_gx == 0) return MSDA_ERR_UNSUPPORTED;  // the halo alone overflows shared memory
    const Windows w = windows_for(spatial_shapes, d.L, best_gx, best_gy, halo, rowb);
    memset(plan, 0, sizeof *plan);
    plan->N = d.N;
    plan->Lq = d.Lq;
    plan->S = d.S;
    plan->L = d.L;
    plan->D = d.D;
    plan->value_dtype = (int32_t)value_dtype;
    plan->halo = halo;
    plan->grid_x = best_gx;
    plan->grid_y = best_gy;
    plan->ctas_per_sm = ctas_per_sm;
    for (int64_t l = 0; l < d.L; ++l) {
        plan->shapes[2 * l] = spatial_shapes[2 * l];
        plan->shapes[2 * l + 1] = spatial_shapes[2 * l + 1];
        plan->window_w[l] = w.ww[l];
        plan->window_h[l] = w.wh[l];
    }
    plan->window_bytes = w.bytes;
    plan->device_bytes = plan_device_bytes(d.N, d.Lq, (int64_t)best_gx * best_gy);
    return MSDA_OK;
}

msda_status msda_tile_plan_build(const msda_tile_plan *plan, const float *reference_points,
                                 int reference_dim, void *plan_buffer, msda_stream_t stream)
{
    if (!plan) return MSDA_ERR_NULL;
    if (reference_dim != 2 && reference_dim != 4) return MSDA_ERR_SHAPE;
    if (plan->N < 0 || plan->Lq < 0 || plan->grid_x < 1 || plan->grid_y < 1 ||
        (int64_t)plan->grid_x * plan->grid_y > msda::kTileMaxCells || plan->N > kI32Max ||
        plan->Lq > kI32Max)
        return MSDA_ERR_SHAPE;
    const int64_t G = (int64_t)plan->grid_x * plan->grid_y;
    if (plan->device_bytes != plan_device_bytes(plan->N, plan->Lq, G)) return MSDA_ERR_SHAPE;
    if (plan->N == 0) return MSDA_OK;
    if (!plan_buffer || (plan->Lq > 0 && !reference_points)) return MSDA_ERR_NULL;
    if (!aligned(plan_buffer, 16) || !aligned(reference_points, 8)) return MSDA_ERR_ALIGN;
    const Span outs[] = {{plan_buffer, plan->device_bytes}};
    const Span ins[] = {{reference_points, plan->N * plan->Lq * reference_dim * 4}};
    if (any_alias(outs, 1, ins, 1)) return MSDA_ERR_ALIAS;
    msda::TilePlanParams p;
    memset(&p, 0, sizeof p);
    p.ref = reference_points;
    p.ref_dim = reference_dim;
    p.N = (int)plan->N;
    p.Lq = (int)plan->Lq;
    p.gx = plan->grid_x;
    p.gy = plan->grid_y;
    p.cell_start = static_cast<int *>(plan_buffer);
    p.perm = reinterpret_cast<int *>(static_cast<char *>(plan_buffer) +
                                     round_up(plan->N * (G + 1) * 4, 256));
    return cuda_status(msda::launch_tile_plan(p, static_cast<cudaStream_t>(stream)));
}

msda_status msda_forward_tiled(const void *value, msda_dtype value_dtype,
                               const int64_t *spatial_shapes, const int64_t *level_start_index,
                               const float *sampling_locations, const float *attention_weights,
                               float *out, msda_dims d, const msda_tile_plan *plan,
                               const void *plan_buffer, msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, d.M, &pr)) != MSDA_OK) return st;
    if ((st = check_plan_args(plan, plan_buffer, value_dtype, spatial_shapes, d, pr)) != MSDA_OK)
        return st;
    if (pr.n_out > 0 && (!sampling_locations || !attention_weights || !out))
        return MSDA_ERR_NULL;
    if (pr.n_out > 0 && pr.n_value > 0 && !value) return MSDA_ERR_NULL;
    if (!aligned(value, 16) || !aligned(out, 16) || !aligned(sampling_locations, 8) ||
        !aligned(attention_weights, 4))
        return MSDA_ERR_ALIGN;
    const Span outs[] = {{out, pr.n_out * 4}};
    const Span ins[] = {{value, pr.n_value * pr.esz},
                        {sampling_locations, pr.lsamples * 8},
                        {attention_weights, pr.samples * 4},
                        {plan_buffer, plan->device_bytes}};
    if (any_alias(outs, 1, ins, 4)) return MSDA_ERR_ALIAS;
    if (pr.n_out == 0) return MSDA_OK;
    msda::FwdParams f;
    memset(&f, 0, sizeof f);
    f.value = value;
    f.loc = sampling_locations;
    f.attn = attention_weights;
    f.out = out;
    set_dims(&f, d, d.M, pr);
    return launch_fwd_tiled(value, value_dtype, d, pr, plan, plan_buffer, f, false,
                            static_cast<cudaStream_t>(stream));
}

msda_status msda_forward_fused_tiled(const void *value, msda_dtype value_dtype,
                                     const int64_t *spatial_shapes,
                                     const int64_t *level_start_index,
                                     const float *reference_points, int reference_dim,
                                     const float *offsets, const float *logits, float *out,
                                     float *sampling_locations_out,
                                     float *attention_weights_out, msda_dims d,
                                     const msda_tile_plan *plan, const void *plan_buffer,
                                     msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, d.M, &pr)) != MSDA_OK) return st;
    if (reference_dim != 2 && reference_dim != 4) return MSDA_ERR_SHAPE;
    if ((st = check_plan_args(plan, plan_buffer, value_dtype, spatial_shapes, d, pr)) != MSDA_OK)
        return st;
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
                        {logits, pr.samples * 4},
                        {plan_buffer, plan->device_bytes}};
    if (any_alias(outs, 3, ins, 5)) return MSDA_ERR_ALIAS;
    if (pr.n_out == 0) return MSDA_OK;
    msda::FwdParams f;
    memset(&f, 0, sizeof f);
    f.value = value;
    f.ref = reference_points;
    f.ref_dim = reference_dim;
    f.off = offsets;
    f.logits = logits;
    f.out = out;
    f.loc_out = sampling_locations_out;
    f.attn_out = attention_weights_out;
    set_dims(&f, d, d.M, pr);
    return launch_fwd_tiled(value, value_dtype, d, pr, plan, plan_buffer, f, true,
                            static_cast<cudaStream_t>(stream));
}

msda_status msda_backward_tiled(const void *value, msda_dtype value_dtype,
                                const int64_t *spatial_shapes, const int64_t *level_start_index,
                                const float *sampling_locations, const float *attention_weights,
                                const float *grad_out, float *grad_value,
                                float *grad_sampling_locations, float *grad_attention_weights,
                                msda_dims d, const msda_tile_plan *plan, const void *plan_buffer,
                                msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, d.M, &pr)) != MSDA_OK) return st;
    if ((st = check_plan_args(plan, plan_buffer, value_dtype, spatial_shapes, d, pr)) != MSDA_OK)
        return st;
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
                        {grad_out, pr.n_out * 4},
                        {plan_buffer, plan->device_bytes}};
    if (any_alias(outs, 3, ins, 5)) return MSDA_ERR_ALIAS;
    const bool bf16 = value_dtype == MSDA_BF16;
    msda::BwdTiledParams p;
    memset(&p, 0, sizeof p);
    int dyn = 0;
    if (pr.n_out > 0 && !backward_layout(&p, plan, d, bf16, false, &dyn))
        return msda_backward(value, value_dtype, spatial_shapes, level_start_index,
                             sampling_locations, attention_weights, grad_out, grad_value,
                             grad_sampling_locations, grad_attention_weights, d, stream);
    p.b.value = value;
    p.b.loc = sampling_locations;
    p.b.attn = attention_weights;
    p.b.grad_out = grad_out;
    p.b.grad_value = grad_value;
    p.b.grad_loc = grad_sampling_locations;
    p.b.grad_attn = grad_attention_weights;
    set_dims(&p.b, d, d.M, pr);
    // before any device work, so that a failure here has launched nothing
    if (pr.n_out > 0) {
        if ((st = set_checks(&p.b, pr)) != MSDA_OK) return st;
        if ((st = encode_maps(p.maps, value, value_dtype, d, pr, plan)) != MSDA_OK) return st;
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pr.n_value > 0) {
        st = cuda_status(cudaMemsetAsync(grad_value, 0, (size_t)pr.n_value * 4, s));
        if (st != MSDA_OK) return st;
    }
    if (pr.n_out == 0) return MSDA_OK;
    p.t = tile_view(plan, plan_buffer, d);
    return launched(msda::launch_backward_tiled(p, bf16, false, dyn, s), s);
}

msda_status msda_backward_fused_tiled(const void *value, msda_dtype value_dtype,
                                      const int64_t *spatial_shapes,
                                      const int64_t *level_start_index,
                                      const float *reference_points, int reference_dim,
                                      const float *offsets, const float *logits,
                                      const float *grad_out, float *grad_value,
                                      float *grad_reference_points, float *grad_offsets,
                                      float *grad_logits, msda_dims d,
                                      const msda_tile_plan *plan, const void *plan_buffer,
                                      msda_stream_t stream)
{
    Problem pr;
    msda_status st = check_dims(value_dtype, spatial_shapes, level_start_index, d, &pr);
    if (st != MSDA_OK) return st;
    if ((st = check_groups(d, d.M, &pr)) != MSDA_OK) return st;
    if (reference_dim != 2 && reference_dim != 4) return MSDA_ERR_SHAPE;
    if ((st = check_plan_args(plan, plan_buffer, value_dtype, spatial_shapes, d, pr)) != MSDA_OK)
        return st;
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
                        {grad_out, pr.n_out * 4},
                        {plan_buffer, plan->device_bytes}};
    if (any_alias(outs, 4, ins, 6)) return MSDA_ERR_ALIAS;
    const bool bf16 = value_dtype == MSDA_BF16;
    msda::BwdTiledParams p;
    memset(&p, 0, sizeof p);
    int dyn = 0;
    if (pr.n_out > 0 && !backward_layout(&p, plan, d, bf16, true, &dyn))
        return msda_backward_fused(value, value_dtype, spatial_shapes, level_start_index,
                                   reference_points, reference_dim, offsets, logits, grad_out,
                                   grad_value, grad_reference_points, grad_offsets, grad_logits,
                                   d, stream);
    p.b.value = value;
    p.b.ref = reference_points;
    p.b.ref_dim = reference_dim;
    p.b.off = offsets;
    p.b.logits = logits;
    p.b.grad_out = grad_out;
    p.b.grad_value = grad_value;
    p.b.grad_ref = grad_reference_points;
    p.b.grad_off = grad_offsets;
    p.b.grad_logits = grad_logits;
    set_dims(&p.b, d, d.M, pr);
    // before any device work, so that a failure here has launched nothing
    if (pr.n_out > 0) {
        if ((st = set_checks(&p.b, pr)) != MSDA_OK) return st;
        if ((st = encode_maps(p.maps, value, value_dtype, d, pr, plan)) != MSDA_OK) return st;
    }
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
    if (pr.n_out == 0) return MSDA_OK;
    p.t = tile_view(plan, plan_buffer, d);
    return launched(msda::launch_backward_tiled(p, bf16, true, dyn, s), s);
}

msda_status msda_debug_tiled_stalls(int64_t *count)
{
    if (!count) return MSDA_ERR_NULL;
    *count = 0;
    unsigned *w = msda::stall_word();
    if (!w) return cuda_status(cudaErrorInvalidDevicePointer);
    unsigned h = 0;
    msda_status st = cuda_status(cudaDeviceSynchronize());
    if (st == MSDA_OK) st = cuda_status(cudaMemcpy(&h, w, sizeof h, cudaMemcpyDeviceToHost));
    if (st == MSDA_OK) st = cuda_status(cudaMemset(w, 0, sizeof h));
    if (st == MSDA_OK) *count = (int64_t)h;
    return st;
}

}  // extern "C"
