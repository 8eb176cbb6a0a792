// msda_common.cuh -- device helpers shared by the MSDeformAttn kernels.
//
// Every kernel (forward, fused forward, backward, index record) derives a
// sample's cell from its normalised location through msda_cell(), so the
// integer cell, the corner rows and the fractions are computed by one piece
// of code everywhere.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "msda_types.h"

namespace msda {

constexpr unsigned kFull = 0xffffffffu;

// Pixel coordinate and cell of one sample on a level of size H x W
// ("Deformable DETR" wiki page, "Multi-scale deformable attention": phi_l
// rescales the normalised point by the level's size).  Pixel centres sit at
// half-integers: x = loc_x * W - 0.5, each step one IEEE fp32 operation with
// no contraction into an FMA.  Returns false when no corner of the cell can
// lie inside the level (x outside (-1, W) or y outside (-1, H)); NaN and Inf
// fail this test too.
__device__ __forceinline__ bool msda_cell(float lx, float ly, int H, int W, float &x,
                                          float &y, int &x0, int &y0, float &fx,
                                          float &fy)
{
    x = __fadd_rn(__fmul_rn(lx, (float)W), -0.5f);
    y = __fadd_rn(__fmul_rn(ly, (float)H), -0.5f);
    if (!(x > -1.0f && x < (float)W && y > -1.0f && y < (float)H)) return false;
    const float xf = floorf(x);
    const float yf = floorf(y);
    x0 = (int)xf;
    y0 = (int)yf;
    fx = __fsub_rn(x, xf);
    fy = __fsub_rn(y, yf);
    return true;
}

// Sampling location of one sample of the fused path ("Deformable DETR" wiki
// page: the reference point plus the predicted offset, "Multi-scale
// deformable attention"; offsets scaled by the box in iterative refinement,
// "Variants").  Point reference ref[nq] = (x, y) with offsets in pixels of a
// level of H x W: loc = ref + off / (W, H).  Box reference
// ref[nq] = (cx, cy, w, h) with offsets in box units: loc = (cx, cy) +
// off * (w, h).  Each component is one IEEE fp32 divide or multiply, then one
// fp32 add, so every kernel forms the same bits.
__device__ __forceinline__ float2 msda_fused_location(const float *ref, int ref_dim, int64_t nq,
                                                      float ox, float oy, int H, int W)
{
    if (ref_dim == 2) {
        const float2 r = __ldg(reinterpret_cast<const float2 *>(ref) + nq);
        return make_float2(__fadd_rn(r.x, __fdiv_rn(ox, (float)W)),
                           __fadd_rn(r.y, __fdiv_rn(oy, (float)H)));
    }
    const float2 c = __ldg(reinterpret_cast<const float2 *>(ref) + 2 * nq);
    const float2 s = __ldg(reinterpret_cast<const float2 *>(ref) + 2 * nq + 1);
    return make_float2(__fadd_rn(c.x, __fmul_rn(ox, s.x)), __fadd_rn(c.y, __fmul_rn(oy, s.y)));
}

// Bounds check of one access to the value map (or to grad_value, which has
// the same layout): value elements [first, first + count) against [0, limit).
// Only the bounds-checked build (-DMSDA_CHECKED) tests anything: there an
// access outside the range is to be skipped by the caller, and it is counted
// in check[0] with the first one's element index in check[1].  In the default
// build every index is in range by construction (cells come from msda_cell
// and msda_row, dims are validated on the host) and this is the constant true.
__device__ __forceinline__ bool msda_in_map(unsigned long long *check, int64_t limit,
                                            int64_t first, int count)
{
#ifdef MSDA_CHECKED
    if (first >= 0 && first + count <= limit) return true;
    if (check && atomicAdd(check, 1ull) == 0ull) check[1] = (unsigned long long)first;
    return false;
#else
    (void)check;
    (void)limit;
    (void)first;
    (void)count;
    return true;
#endif
}

// Item of the per-sample location tensors (sampling locations, offsets and
// their gradients) that item = (n*Lq + q)*M + m reads: the heads of one
// deformable group look up the same key locations ("Deformable Attention"
// glossary page, multi-head paragraph), so with G groups of Hg = M/G
// consecutive heads it is
// (n*Lq + q)*G + m/Hg.  Hg = 1 (a group per head) gives the item itself.
__device__ __forceinline__ int64_t msda_loc_item(int64_t item, const FastDiv &dM, int G,
                                                 const FastDiv &dHg)
{
    if (dHg.d == 1) return item;
    const unsigned u = (unsigned)item;
    const unsigned nq = fastdiv(dM, u);
    const unsigned m = u - nq * dM.d;
    return (int64_t)nq * G + fastdiv(dHg, m);
}

// Whether head m (of item) is the first of its deformable group, the one that
// stores the group's shared locations.
__device__ __forceinline__ bool msda_group_first_m(int m, const FastDiv &dHg)
{
    return dHg.d == 1 || (unsigned)m == fastdiv(dHg, (unsigned)m) * dHg.d;
}
__device__ __forceinline__ bool msda_group_first(int64_t item, const FastDiv &dM,
                                                 const FastDiv &dHg)
{
    if (dHg.d == 1) return true;
    const unsigned u = (unsigned)item;
    return msda_group_first_m((int)(u - fastdiv(dM, u) * dM.d), dHg);
}

// The (n*Lq + q, m) split of an item index, and n: items are (n, q, m) in
// storage order, fewer than 2^31.
struct ItemIdx {
    int m;
    int64_t nq, n;
};
__device__ __forceinline__ ItemIdx msda_item_idx(int64_t item, const FastDiv &dM,
                                                 const FastDiv &dLq)
{
    const unsigned u = (unsigned)item;
    const unsigned nq = fastdiv(dM, u);
    ItemIdx r;
    r.m = (int)(u - nq * dM.d);
    r.nq = nq;
    r.n = fastdiv(dLq, nq);
    return r;
}

// Writes the gradient of one shared location: a plain store when every head
// has its own locations, else a vector reduction into the zeroed output, since
// the Hg heads of a group add into one location (their order is unspecified).
__device__ __forceinline__ void msda_put_loc_grad(float *base, int64_t sl, float gx, float gy,
                                                  bool shared)
{
    float2 *dst = reinterpret_cast<float2 *>(base) + sl;
    if (!shared) {
        __stcs(dst, make_float2(gx, gy));
        return;
    }
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(gx), "f"(gy)
                 : "memory");
}

// Value row of pixel (yy, xx) on a level, or -1 outside the level (zero
// padding: such a corner contributes nothing).
__device__ __forceinline__ int msda_row(int start, int H, int W, int yy, int xx)
{
    return (xx >= 0 && xx < W && yy >= 0 && yy < H) ? start + yy * W + xx : -1;
}

// ---------------------------------------------------------------------------
// Loads of one 16-byte chunk of a value row, widened to fp32.
// ---------------------------------------------------------------------------
template <typename VT>
struct Chunk;

template <>
struct Chunk<float> {
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void load(const float *p, float (&v)[4])
    {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
        v[0] = t.x;
        v[1] = t.y;
        v[2] = t.z;
        v[3] = t.w;
    }
};

template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&v)[8])
    {
        const uint4 t = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bf16 -> fp32 widening is exact: the bf16 bits become the high half.
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// Vector atomic add of four fp32 values (sm_90+ `red.global.add.v4.f32`).
__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a),
                 "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Max / sum over aligned segments of P lanes (P a power of two <= 32).
template <int P>
__device__ __forceinline__ float seg_max(float v)
{
#pragma unroll
    for (int o = P / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

template <int P>
__device__ __forceinline__ float seg_sum(float v)
{
#pragma unroll
    for (int o = P / 2; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Joint softmax weight of this lane's sample over its aligned segment of P
// lanes, which holds the L*K logits of one (query, head) ("Deformable DETR"
// wiki page, "Multi-scale deformable attention": the weights of a head sum to
// one over all levels and points).  Max-subtracted; lanes with act false hold
// no sample and add nothing.  Every kernel with at most 32 samples per item
// forms its weights here, so the fused forward and backward agree bit for bit.
template <int P>
__device__ __forceinline__ float seg_softmax(float logit, bool act)
{
    const float z = act ? logit : -INFINITY;
    const float mx = seg_max<P>(z);
    const float e = act ? expf(__fsub_rn(z, mx)) : 0.f;
    const float sum = seg_sum<P>(e);
    return __fdiv_rn(e, sum);
}

// Joint softmax statistics of one item of more than 32 samples, held by one
// warp: lane j holds the logits of samples j, j + 32, ... in z[] (NB = the
// blocks of 32 there can be; entries past L*K are -inf).  On return z[b] is
// exp(z[b] - max) and the result is the sum over all samples, so that the
// weight of sample b*32 + j is __fdiv_rn(z[b], sum).  The forward and the
// backward both call this, so they form bit-identical weights.
template <int NB>
__device__ __forceinline__ float long_softmax(float (&z)[NB])
{
    float mx = z[0];
#pragma unroll
    for (int b = 1; b < NB; ++b) mx = fmaxf(mx, z[b]);
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        z[b] = z[b] == -INFINITY ? 0.f : expf(__fsub_rn(z[b], mx));
        sum += z[b];
    }
    return warp_sum(sum);
}

// z[i] for a run-time i < NB, as a chain of selects (no local memory).
template <int NB>
__device__ __forceinline__ float pick(const float (&z)[NB], int i)
{
    float r = z[0];
#pragma unroll
    for (int b = 1; b < NB; ++b) r = (i == b) ? z[b] : r;
    return r;
}

}  // namespace msda
