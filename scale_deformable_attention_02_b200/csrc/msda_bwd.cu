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
// Work decomposition (one warp per (n, q, m), as in the forward):
//   1. Lane j < L*K finds sample j's cell and writes, per corner, the row
//      offset, w_j, dw_j/dfx and dw_j/dfy to shared memory.
//   2. SPAN = min(32, 4R) lanes work on one sample (R lanes per 16-byte-chunked
//      row, one corner per R lanes), 32/SPAN samples at a time.  Each lane
//      gathers its chunk of a corner row, forms its part of t_j, scatters
//      A w_j g with one vector `red.global.add.v4.f32` per chunk, and keeps
//      three running partial sums per sample.
//   3. Every 8 samples per lane group the 24 partial sums are reduced across
//      the SPAN lanes with a butterfly reduce-scatter (each step halves the
//      values a lane holds), which costs about 4 shuffles per sample instead
//      of 15, and the lanes holding finished sums write dA and dloc.
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

// Gather/scatter entry of one corner: its value row's address (already offset
// to the batch entry and head), A*w, and the element offset of the matching
// grad_value row inside the (n, m) map (-1: outside the level, nothing to
// scatter).  Corners outside the level read kZeroRowB, so the gathers need no
// predicate; only the scatter is predicated.
struct __align__(16) CornerG {
    const char *row;
    float aw;
    int goff;
};

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

// Fast path for rows of at most 128 bytes (R <= 8, so a warp instruction
// covers 32/R >= 4 (sample, corner) pairs: kSG = 8/R samples of four corners).
//   - Persistent CTAs sweep contiguous item ranges (L1 locality), a warp
//     takes 32/P items per round and phase 1 gives every lane one sample.
//   - Per item, 16 samples at a time (8 for bf16 rows of 128 bytes): all corner rows are loaded before any
//     is used; each lane forms t = <v_chunk, g_chunk> and scatters
//     A*w*g_chunk with a vector reduction.
//   - The 16 partial t of a lane are reduced over the R chunk lanes with a
//     butterfly reduce-scatter (each lane keeps two finished <v_c, g>), then
//     weighted by (w, dw/dfx, dw/dfy) of its corner and summed over the four
//     corner lanes with two xor steps: about 1.6 shuffles per sample.
template <typename VT, int R, int P>
__global__ void __launch_bounds__(kWarps * 32, 2)
    bwd_kernel(const __grid_constant__ BwdParams p)
{
    static_assert(R <= 8, "fast path needs at least four pairs per instruction");
    constexpr int kVec = Chunk<VT>::kVec;  // value elements per 16-byte chunk
    constexpr int kSlots = 32 / R;         // pairs per warp instruction
    constexpr int kSG = kSlots / 4;        // samples per warp instruction
    // instructions per batch: 16 samples, or fewer if the loaded chunks would
    // exceed 64 registers (bf16 with 128-byte rows: 8 samples)
    constexpr int kB = (2 * R < 64 / kVec) ? 2 * R : 64 / kVec;
    constexpr int kBS = kB * kSG;          // samples per batch
    constexpr int kItems = 32 / P;
    static_assert(kB % R == 0, "a batch must split evenly over the chunk lanes");
    static_assert(kBS <= P && P % kBS == 0, "a batch must stay inside the P sample slots");
    constexpr int kKeep = kB / R;          // finished <v_c, g> per lane after stage A

    // Per corner: (row offset, A*w) for the gather/scatter loop and
    // (w, dw/dfx, dw/dfy) for the reduction; corner-major with row stride
    // P + 2 (= 2 mod 8) so that both phases are free of bank conflicts.
    constexpr int kStride = P + 2;
    __shared__ CornerG cOff[kWarps][kItems][4 * kStride];
    __shared__ float4 cDer[kWarps][kItems][4 * kStride];
    __shared__ float sA[kWarps][kItems][P];
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
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int slot = lane / R;
    const int chunk = lane % R;
    const int corner = slot & 3;
    const int sg = slot >> 2;
    const bool chunk_ok = chunk < p.nchunks;

    const int64_t begin = (int64_t)blockIdx.x * p.chunk;
    const int64_t end = begin + p.chunk < p.items ? begin + p.chunk : p.items;

    for (int64_t item0 = begin + warp * kItems; item0 < end; item0 += kWarps * kItems) {
        // ---- phase 1: cell and corner derivatives, one sample per lane ----
        {
            const int seg = lane / P;
            const int j = lane % P;
            const int64_t item = item0 + seg;
            const bool act = j < LK && item < end;
            {  // every sample slot up to P gets entries; unused ones read zeros
                const int l = j < LK ? j / K : 0;
                const int H = sH[l], W = sW[l], start = sStart[l];
                const int m = (int)(item % M);
                const int64_t n = item / M / p.Lq;
                const char *mapb = static_cast<const char *>(p.value) +
                                   ((n * p.S * M + m) * (int64_t)D) * (int64_t)sizeof(VT);
                int off[4] = {-1, -1, -1, -1};
                float w[4] = {0.f, 0.f, 0.f, 0.f};
                float dwx[4] = {0.f, 0.f, 0.f, 0.f};
                float dwy[4] = {0.f, 0.f, 0.f, 0.f};
                float a = 0.f;
                if (act) {
                    const int64_t si = item * LK + j;
                    const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + si);
                    a = __ldcs(p.attn + si);
                    float x, y, fx, fy;
                    int x0, y0;
                    if (msda_cell(t.x, t.y, H, W, x, y, x0, y0, fx, fy)) {
                        const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                        w[0] = hy * hx;
                        w[1] = hy * fx;
                        w[2] = fy * hx;
                        w[3] = fy * fx;
                        dwx[0] = -hy;
                        dwx[1] = hy;
                        dwx[2] = -fy;
                        dwx[3] = fy;
                        dwy[0] = -hx;
                        dwy[1] = -fx;
                        dwy[2] = hx;
                        dwy[3] = fx;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int r = msda_row(start, H, W, y0 + (q >> 1), x0 + (q & 1));
                            off[q] = r < 0 ? -1 : r * MD;
                        }
                    }
                }
                sA[warp][seg][j] = a;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    CornerG g;
                    g.row = off[q] >= 0 ? mapb + (int64_t)off[q] * (int64_t)sizeof(VT)
                                        : reinterpret_cast<const char *>(kZeroRowB);
                    g.aw = a * w[q];
                    g.goff = off[q];
                    cOff[warp][seg][q * kStride + j] = g;
                    cDer[warp][seg][q * kStride + j] = make_float4(w[q], dwx[q], dwy[q], 0.f);
                }
            }
        }
        __syncwarp();

        // ---- phase 2: per item, 16 samples at a time ----------------------
#pragma unroll 1
        for (int it = 0; it < kItems; ++it) {
            const int64_t item = item0 + it;
            if (item >= end) break;  // uniform
            const int m = (int)(item % M);
            const int64_t nq = item / M;
            const int64_t n = nq / p.Lq;
            const int64_t sbase = item * LK;
            float g[kVec];
            if (chunk_ok) {
                const float4 *gp = reinterpret_cast<const float4 *>(
                    p.grad_out + nq * (int64_t)MD + m * D + chunk * kVec);
#pragma unroll
                for (int i = 0; i < kVec / 4; ++i) {
                    const float4 t = __ldcs(gp + i);
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
            float *gvb = p.grad_value + rowbase;
            // lanes past the last chunk re-read chunk 0 (their g is zero)
            const int lane_off = chunk_ok ? chunk * 16 : 0;

            for (int s0 = 0; s0 < LK; s0 += kBS) {
                // loads: instruction b covers samples s0 + b*kSG + (0..kSG-1)
                uint4 raw[kB];
                float aw[kB];
                int goff[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int s = s0 + b * kSG + sg;  // < P: every slot has an entry
                    const CornerG e = cOff[warp][it][corner * kStride + s];
                    raw[b] = __ldg(reinterpret_cast<const uint4 *>(e.row + lane_off));
                    aw[b] = e.aw;
                    goff[b] = e.goff;
                }
                float t[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    float v[kVec];
                    widen<VT>(raw[b], v);
                    t[b] = 0.f;
#pragma unroll
                    for (int i = 0; i < kVec; ++i) t[b] = fmaf(v[i], g[i], t[b]);
                    if (goff[b] >= 0 && chunk_ok) {
                        float *dst = gvb + goff[b];
#pragma unroll
                        for (int i = 0; i < kVec; i += 4)
                            red_add_v4(dst + i, aw[b] * g[i], aw[b] * g[i + 1], aw[b] * g[i + 2],
                                       aw[b] * g[i + 3]);
                    }
                }
                // stage A: reduce t over the R chunk lanes (lane bits below R)
                reduce_scatter_n<R, kB, kB>(t, lane);
                // lane now holds <v_corner, g> of instructions b = chunk*kKeep + k
                float q[3][kKeep];
#pragma unroll
                for (int k = 0; k < kKeep; ++k) {
                    const int b = chunk * kKeep + k;
                    const int s = s0 + b * kSG + sg;
                    float4 e = make_float4(0.f, 0.f, 0.f, 0.f);  // (w, dw/dfx, dw/dfy, -)
                    if (s < LK) e = cDer[warp][it][corner * kStride + s];
                    q[0][k] = e.x * t[k];
                    q[1][k] = e.y * t[k];
                    q[2][k] = e.z * t[k];
                }
                // stage B: sum over the four corner lanes of each sample
#pragma unroll
                for (int o = R; o < 4 * R; o <<= 1)
#pragma unroll
                    for (int k = 0; k < kKeep; ++k) {
                        q[0][k] += __shfl_xor_sync(kFull, q[0][k], o);
                        q[1][k] += __shfl_xor_sync(kFull, q[1][k], o);
                        q[2][k] += __shfl_xor_sync(kFull, q[2][k], o);
                    }
                if (corner == 0) {
#pragma unroll
                    for (int k = 0; k < kKeep; ++k) {
                        const int b = chunk * kKeep + k;
                        const int s = s0 + b * kSG + sg;
                        if (s < LK) {
                            const int64_t si = sbase + s;
                            if (p.grad_attn) __stcs(p.grad_attn + si, q[0][k]);
                            if (p.grad_loc) {
                                const int l = s / K;
                                const float a = sA[warp][it][s];
                                __stcs(reinterpret_cast<float2 *>(p.grad_loc) + si,
                                       make_float2(a * ((float)sW[l] * q[1][k]),
                                                   a * ((float)sH[l] * q[2][k])));
                            }
                        }
                    }
                }
            }
        }
        __syncwarp();
    }
}

template <typename VT, int R, int P>
cudaError_t launch_fast(BwdParams p, cudaStream_t stream)
{
    constexpr int kRound = kWarps * (32 / P);
    auto kern = bwd_kernel<VT, R, P>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kRound);
    p.chunk = (p.items + ctas - 1) / ctas;
    p.chunk = (p.chunk + kRound - 1) / kRound * kRound;
    const dim3 grid((unsigned)((p.items + p.chunk - 1) / p.chunk));
    kern<<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

// Samples per batch of the fast path (compile-time, per value type and R).
template <typename VT, int R>
constexpr int batch_samples()
{
    constexpr int kVec = Chunk<VT>::kVec;
    constexpr int kB = (2 * R < 64 / kVec) ? 2 * R : 64 / kVec;
    return kB * (8 / R);
}

template <typename VT, int R>
cudaError_t launch_fast_r(const BwdParams &p, cudaStream_t stream)
{
    // P: a power of two >= L*K and >= the samples of one batch
    constexpr int kBS = batch_samples<VT, R>();
    const int LK = p.L * p.K;
    const int need = LK > kBS ? LK : kBS;
    if constexpr (kBS <= 8) {
        if (need <= 8) return launch_fast<VT, R, 8>(p, stream);
    }
    if (need <= 16) return launch_fast<VT, R, 16>(p, stream);
    return launch_fast<VT, R, 32>(p, stream);
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
