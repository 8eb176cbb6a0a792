// msda_bwd.cu -- backward kernel of the MSDeformAttn core (sm_100a).
//
// Gradients flow through the bilinear interpolation to the value map, the
// sampling locations and the attention weights ("Deformable DETR" wiki
// page, "Deformable attention module"; "Deformable Attention" glossary
// page, gradients through the interpolation grid).  Per sample, with
// g = grad_out[n,q,m,:], corner weights w_j(fx, fy) and t_j = <v_j, g>:
//   dA        = sum_j w_j t_j
//   dloc_x    = A * W * sum_j (dw_j/dfx) t_j,  dloc_y = A * H * sum_j (dw_j/dfy) t_j
//   dvalue_j += A * w_j * g            (scatter; corners inside the level)
//
// Two kernels:
//   * bwd_kernel (value rows of at most 128 bytes): a group of R lanes owns
//     whole samples and sums their four corners inside each lane, so only
//     the R chunk lanes need combining (see its comment).  Persistent CTAs
//     sweep contiguous item ranges.
//   * bwd_kernel_wide (rows wider than 128 bytes): one warp per item; lane j
//     finds sample j's cell and stores per-corner (row offset, w, dw/dfx,
//     dw/dfy) in shared memory; min(32, 4R) lanes work on one sample, and the
//     per-sample partial sums are reduced every 8 samples with a butterfly
//     reduce-scatter.
// Both scatter A w_j g with one vector `red.global.add.v4.f32` per 16 bytes.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

constexpr int kWarps = 8;
constexpr int kBatch = 8;  // samples per lane group between reductions
constexpr int kNV = 32;    // reduce-scatter width: 3 * kBatch used, padded

struct __align__(16) CornerB {
    int off;  // element offset of the corner row inside the (n, m) map; -1 = outside
    float w;    // bilinear weight
    float dwx;  // d w / d fx
    float dwy;  // d w / d fy
};

// A raw 16-byte chunk of a value row, widened to fp32 (bf16 widening is exact).
template <typename VT>
__device__ __forceinline__ void widen(const uint4 &r, float (&v)[Chunk<VT>::kVec]);

template <>
__device__ __forceinline__ void widen<float>(const uint4 &r, float (&v)[4])
{
    v[0] = __uint_as_float(r.x);
    v[1] = __uint_as_float(r.y);
    v[2] = __uint_as_float(r.z);
    v[3] = __uint_as_float(r.w);
}

template <>
__device__ __forceinline__ void widen<__nv_bfloat16>(const uint4 &r, float (&v)[8])
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// 512 bytes of zeros: the row that corners outside the level read.
__device__ __align__(128) float4 kZeroRowB[32] = {};

// Butterfly reduce-scatter over aligned groups of SPAN lanes.  Before: every
// lane holds N partial values.  After: lane (lane % SPAN) = b holds, in
// v[0 .. N/SPAN), the group totals of values b*N/SPAN .. (b+1)*N/SPAN - 1.
template <int SPAN, int N>
__device__ __forceinline__ void reduce_scatter(float (&v)[kNV], int lane)
{
    if constexpr (SPAN > 1) {
        constexpr int o = SPAN / 2;
        constexpr int h = N / 2;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? v[i] : v[i + h];
            const float keep = upper ? v[i + h] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
        reduce_scatter<o, h>(v, lane);
    }
}

// Butterfly reduce-scatter of the first CNT values of v over aligned groups
// of SPAN lanes (CNT a multiple of SPAN): afterwards lane b = lane % SPAN holds
// in v[0, CNT/SPAN) the group totals of values b*CNT/SPAN ... (b+1)*CNT/SPAN - 1.
template <int SPAN, int CNT, int N>
__device__ __forceinline__ void reduce_scatter_n(float (&v)[N], int lane)
{
    static_assert(CNT <= N && CNT % SPAN == 0, "reduce-scatter shape");
    if constexpr (SPAN > 1) {
        constexpr int o = SPAN / 2;
        constexpr int h = CNT / 2;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = upper ? v[i] : v[i + h];
            const float keep = upper ? v[i + h] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
        reduce_scatter_n<o, h, N>(v, lane);  // the kept half now sits in v[0, h)
    }
}

// Generic path (any row width): one warp per item, partial sums of 32 lanes
// reduced every 8 samples.  Used for rows wider than 128 bytes.
template <typename VT, int R>
__global__ void __launch_bounds__(kWarps * 32)
    bwd_kernel_wide(const __grid_constant__ BwdParams p)
{
    constexpr int kVec = Chunk<VT>::kVec;
    constexpr int kSpan = (4 * R < 32) ? 4 * R : 32;  // lanes per sample
    constexpr int kGroups = 32 / kSpan;               // samples in flight per warp
    constexpr int kCornerSlots = kSpan / R;           // 4, 2 or 1
    constexpr int kCpl = 4 / kCornerSlots;            // corners per lane
    constexpr int kPer = kNV / kSpan;                 // finished sums per lane

    __shared__ CornerB corners[kWarps][kMaxLK * 4];
    __shared__ float sA[kWarps][kMaxLK];
    __shared__ int sH[kMaxLevels], sW[kMaxLevels], sStart[kMaxLevels];

    const int tid = threadIdx.x;
    if (tid < p.L) {
        sH[tid] = p.lv.H[tid];
        sW[tid] = p.lv.W[tid];
        sStart[tid] = p.lv.start[tid];
    }
    __syncthreads();

    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t item = (int64_t)blockIdx.x * kWarps + warp;
    if (item >= p.items) return;

    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int m = (int)(item % M);
    const int64_t nq = item / M;
    const int64_t n = nq / p.Lq;
    const int64_t sbase = item * LK;

    // ---- phase 1: cell and corner derivatives of sample `lane` -------------
    if (lane < LK) {
        const int l = lane / K;
        const int H = sH[l], W = sW[l], start = sStart[l];
        const float2 t = __ldg(reinterpret_cast<const float2 *>(p.loc) + sbase + lane);
        sA[warp][lane] = __ldg(p.attn + sbase + lane);
        CornerB c[4] = {{-1, 0.f, 0.f, 0.f}, {-1, 0.f, 0.f, 0.f}, {-1, 0.f, 0.f, 0.f},
                        {-1, 0.f, 0.f, 0.f}};
        float x, y, fx, fy;
        int x0, y0;
        if (msda_cell(t.x, t.y, H, W, x, y, x0, y0, fx, fy)) {
            const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
            // corner j = (dy, dx) = (j >> 1, j & 1)
            const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
            const float dwx[4] = {-hy, hy, -fy, fy};
            const float dwy[4] = {-hx, -fx, hx, fx};
            const int MD = M * D;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = msda_row(start, H, W, y0 + (j >> 1), x0 + (j & 1));
                c[j].off = r < 0 ? -1 : r * MD;
                c[j].w = w[j];
                c[j].dwx = dwx[j];
                c[j].dwy = dwy[j];
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) corners[warp][lane * 4 + j] = c[j];
    }
    __syncwarp();

    // ---- phase 2/3 -------------------------------------------------------
    const int grp = lane / kSpan;
    const int lin = lane % kSpan;
    const int cslot = lin / R;
    const int chunk = lin % R;
    const bool chunk_ok = chunk < p.nchunks;

    float g[kVec];
    if (chunk_ok) {
        const float4 *gp = reinterpret_cast<const float4 *>(
            p.grad_out + nq * (int64_t)(M * D) + m * D + chunk * kVec);
#pragma unroll
        for (int i = 0; i < kVec / 4; ++i) {
            const float4 t = __ldg(gp + i);
            g[4 * i] = t.x;
            g[4 * i + 1] = t.y;
            g[4 * i + 2] = t.z;
            g[4 * i + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < kVec; ++i) g[i] = 0.f;
    }
    const int64_t rowbase = (n * p.S * M + m) * (int64_t)D + chunk * kVec;
    const VT *vbase = static_cast<const VT *>(p.value) + rowbase;
    float *gvbase = p.grad_value + rowbase;

    const int per_batch = kBatch * kGroups;
    for (int b0 = 0; b0 < LK; b0 += per_batch) {
        float v[kNV];
#pragma unroll
        for (int i = 0; i < kNV; ++i) v[i] = 0.f;
#pragma unroll
        for (int it = 0; it < kBatch; ++it) {
            const int s = b0 + it * kGroups + grp;
            if (s < LK) {
                const float a = sA[warp][s];
#pragma unroll
                for (int ci = 0; ci < kCpl; ++ci) {
                    const CornerB e = corners[warp][s * 4 + cslot * kCpl + ci];
                    float t = 0.f;
                    if (e.off >= 0 && chunk_ok) {
                        float x[kVec];
                        Chunk<VT>::load(vbase + e.off, x);
#pragma unroll
                        for (int i = 0; i < kVec; ++i) t = fmaf(x[i], g[i], t);
                        const float aw = a * e.w;
                        float *dst = gvbase + e.off;
#pragma unroll
                        for (int i = 0; i < kVec; i += 4)
                            red_add_v4(dst + i, aw * g[i], aw * g[i + 1], aw * g[i + 2],
                                       aw * g[i + 3]);
                    }
                    v[it] = fmaf(e.w, t, v[it]);
                    v[kBatch + it] = fmaf(e.dwx, t, v[kBatch + it]);
                    v[2 * kBatch + it] = fmaf(e.dwy, t, v[2 * kBatch + it]);
                }
            }
        }
        reduce_scatter<kSpan, kNV>(v, lane);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int idx = lin * kPer + i;
            const int qty = idx / kBatch;
            const int it = idx % kBatch;
            const int s = b0 + it * kGroups + grp;
            if (qty < 3 && s < LK) {
                const int64_t si = sbase + s;
                if (qty == 0) {
                    if (p.grad_attn) p.grad_attn[si] = v[i];
                } else if (p.grad_loc) {
                    const int l = s / K;
                    const float scale = (qty == 1) ? (float)sW[l] : (float)sH[l];
                    p.grad_loc[2 * si + (qty - 1)] = sA[warp][s] * (scale * v[i]);
                }
            }
        }
    }
}

// Fast path for value rows of at most 128 bytes (R <= 8 lanes per row).
//
// Lane layout as in the forward fast path: G = 32/R groups of R lanes, group g
// owns samples g, g+G, ... of the item with all four corners, lane `chunk` owns
// 16 bytes of every row.  Per sample a lane gathers the four corner chunks,
// forms t_c = <v_c, g_chunk>, scatters A*w_c*g_chunk with a vector reduction
// (corners inside the level only; outside corners read a zero row), and adds
// w_c t_c, dw_c/dfx t_c, dw_c/dfy t_c into three per-sample partial sums.
// The four corners are summed inside the lane, so only the R chunk lanes of a
// group have to be combined: one butterfly reduce-scatter of all the item's
// partial sums at the end.
template <typename VT, int R, int NS, int NB>
__global__ void __launch_bounds__(kWarps * 32, 2)
    bwd_kernel(const __grid_constant__ BwdParams p)
{
    static_assert(R <= 8 && NS * (32 / R) <= 32, "fast path shape");
    constexpr int G = 32 / R;
    constexpr int kVec = Chunk<VT>::kVec;
    constexpr int kQ = 3 * NS;                           // partial sums per lane
    constexpr int kCnt = (kQ + R - 1) / R * R;           // padded to the chunk lanes
    constexpr int kPer = kCnt / R;                       // finished sums per lane
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane / R;
    const int chunk = lane % R;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int nsl = (LK + G - 1) / G;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_off = chunk_ok ? chunk * 16 : 0;
    const char *zrow = reinterpret_cast<const char *>(kZeroRowB) + lane_off;
    const int64_t rowbytes = (int64_t)MD * (int64_t)sizeof(VT);

    int lvW[NS], lvH[NS], lvS[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int s = g + G * i;
        const int l = s < LK ? s / K : 0;
        lvW[i] = p.lv.W[l];
        lvH[i] = p.lv.H[l];
        lvS[i] = p.lv.start[l];
    }

    const int64_t begin = (int64_t)blockIdx.x * p.chunk;
    const int64_t end = begin + p.chunk < p.items ? begin + p.chunk : p.items;
    for (int64_t item = begin + warp; item < end; item += kWarps) {
        const int m = (int)(item % M);
        const int64_t nq = item / M;
        const int64_t n = nq / p.Lq;
        const int64_t sbase = item * LK;
        const int64_t mapoff = (n * p.S * M + m) * (int64_t)D;  // element offset of the (n, m) map
        const char *mapb = static_cast<const char *>(p.value) + mapoff * (int64_t)sizeof(VT) +
                           lane_off;
        float *gmap = p.grad_value + mapoff + chunk * kVec;

        float gv[kVec];
        if (chunk_ok) {
            const float4 *gp = reinterpret_cast<const float4 *>(
                p.grad_out + nq * (int64_t)MD + m * D + chunk * kVec);
#pragma unroll
            for (int i = 0; i < kVec / 4; ++i) {
                const float4 t = __ldcs(gp + i);
                gv[4 * i] = t.x;
                gv[4 * i + 1] = t.y;
                gv[4 * i + 2] = t.z;
                gv[4 * i + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < kVec; ++i) gv[i] = 0.f;
        }

        float q[kCnt];  // [quantity * NS + slot]: dA, dfx, dfy partial sums
        float aS[NS];   // attention weight of each slot's sample
#pragma unroll
        for (int i = 0; i < kCnt; ++i) q[i] = 0.f;
#pragma unroll
        for (int i = 0; i < NS; ++i) aS[i] = 0.f;

#pragma unroll
        for (int i0 = 0; i0 < NS; i0 += NB) {
            if (i0 >= nsl) break;  // uniform
            const char *ptr[NB][4];
            int goff[NB][4];
            float w[NB][4], dwx[NB][4], dwy[NB][4];
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                const int i = i0 + u;
                const int s = g + G * i;
                float lx = 0.f, ly = 0.f, a = 0.f;
                if (s < LK) {
                    const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sbase + s);
                    lx = t.x;
                    ly = t.y;
                    a = __ldcs(p.attn + sbase + s);
                }
                aS[i] = a;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ptr[u][c] = zrow;
                    goff[u][c] = -1;
                    w[u][c] = dwx[u][c] = dwy[u][c] = 0.f;
                }
                float x, y, fx, fy;
                int x0, y0;
                if (s < LK && msda_cell(lx, ly, lvH[i], lvW[i], x, y, x0, y0, fx, fy)) {
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    w[u][0] = hy * hx;
                    w[u][1] = hy * fx;
                    w[u][2] = fy * hx;
                    w[u][3] = fy * fx;
                    dwx[u][0] = -hy;
                    dwx[u][1] = hy;
                    dwx[u][2] = -fy;
                    dwx[u][3] = fy;
                    dwy[u][0] = -hx;
                    dwy[u][1] = -fx;
                    dwy[u][2] = hx;
                    dwy[u][3] = fx;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = msda_row(lvS[i], lvH[i], lvW[i], y0 + (c >> 1), x0 + (c & 1));
                        if (r >= 0) {
                            ptr[u][c] = mapb + (int64_t)r * rowbytes;
                            goff[u][c] = r * MD;
                        }
                    }
                }
            }
            uint4 raw[NB][4];
#pragma unroll
            for (int u = 0; u < NB; ++u)
#pragma unroll
                for (int c = 0; c < 4; ++c) raw[u][c] = __ldg(reinterpret_cast<const uint4 *>(ptr[u][c]));
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                const int i = i0 + u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float v[kVec];
                    widen<VT>(raw[u][c], v);
                    float t = 0.f;
#pragma unroll
                    for (int e = 0; e < kVec; ++e) t = fmaf(v[e], gv[e], t);
                    q[i] = fmaf(w[u][c], t, q[i]);
                    q[NS + i] = fmaf(dwx[u][c], t, q[NS + i]);
                    q[2 * NS + i] = fmaf(dwy[u][c], t, q[2 * NS + i]);
                    if (goff[u][c] >= 0 && chunk_ok) {
                        const float aw = aS[i] * w[u][c];
                        float *dst = gmap + goff[u][c];
#pragma unroll
                        for (int e = 0; e < kVec; e += 4)
                            red_add_v4(dst + e, aw * gv[e], aw * gv[e + 1], aw * gv[e + 2],
                                       aw * gv[e + 3]);
                    }
                }
            }
        }

        // combine the R chunk lanes of each group: lane `chunk` ends with the
        // totals of partial sums chunk*kPer ... chunk*kPer + kPer - 1
        reduce_scatter_n<R, kCnt, kCnt>(q, lane);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int idx = chunk * kPer + k;
            const int qty = idx / NS;
            const int i = idx % NS;
            const int s = g + G * i;
            if (qty < 3 && s < LK) {
                const int64_t si = sbase + s;
                if (qty == 0) {
                    if (p.grad_attn) __stcs(p.grad_attn + si, q[k]);
                } else if (p.grad_loc) {
                    // the slot's level: every lane holds lvW/lvH for all its slots
                    float scale = 0.f, a = 0.f;
#pragma unroll
                    for (int jj = 0; jj < NS; ++jj)
                        if (jj == i) {
                            scale = (qty == 1) ? (float)lvW[jj] : (float)lvH[jj];
                            a = aS[jj];
                        }
                    __stcs(p.grad_loc + 2 * si + (qty - 1), a * (scale * q[k]));
                }
            }
        }
    }
}

template <typename VT, int R, int NS>
cudaError_t launch_fast(BwdParams p, cudaStream_t stream)
{
    constexpr int NB = NS < 2 ? NS : 2;
    auto kern = bwd_kernel<VT, R, NS, NB>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kWarps);
    p.chunk = (p.items + ctas - 1) / ctas;
    p.chunk = (p.chunk + kWarps - 1) / kWarps * kWarps;
    const dim3 grid((unsigned)((p.items + p.chunk - 1) / p.chunk));
    kern<<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename VT, int R>
cudaError_t launch_fast_r(const BwdParams &p, cudaStream_t stream)
{
    constexpr int G = 32 / R;
    const int LK = p.L * p.K;
    const int nsl = (LK + G - 1) / G;
    if (nsl <= 1) return launch_fast<VT, R, 1>(p, stream);
    if constexpr (G <= 16) {
        if (nsl <= 2) return launch_fast<VT, R, 2>(p, stream);
    }
    if constexpr (G <= 8) {
        if (nsl <= 4) return launch_fast<VT, R, 4>(p, stream);
    }
    if constexpr (G <= 4) {
        return launch_fast<VT, R, 8>(p, stream);
    }
    return cudaErrorInvalidValue;  // not reached: L*K <= 32
}

template <typename VT>
cudaError_t launch_bwd_vt(const BwdParams &p, int R, cudaStream_t stream)
{
    const dim3 block(kWarps * 32);
    const dim3 grid((unsigned)((p.items + kWarps - 1) / kWarps));
    switch (R) {
    case 1: return launch_fast_r<VT, 1>(p, stream);
    case 2: return launch_fast_r<VT, 2>(p, stream);
    case 4: return launch_fast_r<VT, 4>(p, stream);
    case 8: return launch_fast_r<VT, 8>(p, stream);
    case 16: bwd_kernel_wide<VT, 16><<<grid, block, 0, stream>>>(p); break;
    case 32: bwd_kernel_wide<VT, 32><<<grid, block, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BwdParams &p, bool bf16, int lanes_per_row,
                            cudaStream_t stream)
{
    if (p.items == 0) return cudaSuccess;
    return bf16 ? launch_bwd_vt<__nv_bfloat16>(p, lanes_per_row, stream)
                : launch_bwd_vt<float>(p, lanes_per_row, stream);
}

}  // namespace msda
