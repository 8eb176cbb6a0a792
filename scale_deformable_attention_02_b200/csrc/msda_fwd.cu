// msda_fwd.cu -- forward kernels of the MSDeformAttn core (sm_100a).
//
// Computes, per batch entry n, query q and head m ("Deformable DETR" wiki
// page, "Multi-scale deformable attention" equation):
//   out[n,q,m,:] = sum_{l,k} A[n,q,m,l,k] * bilinear(value[n, level l, m, :], loc)
//
// An "item" is one (n, q, m); it has L*K samples, each with four corner rows of
// D elements.  A (pixel, head) row is split into 16-byte chunks and R lanes
// cover one row, so a warp instruction gathers 32/R whole rows with 16 bytes
// per lane (fp32, D = 32: R = 8; bf16, D = 32: R = 4); lanes accumulate their
// chunk in fp32 with packed FMA (`__ffma2_rn`).  Two kernels:
//   * fwd_kernel (rows of at most 128 bytes): a group of R lanes owns whole
//     samples; every lane forms its corner addresses and weights in registers
//     (see its comment).
//   * fwd_kernel_wide (wider rows): lane j of an item's P-lane segment forms
//     sample j's cell and writes four (row address, weight) entries to shared
//     memory; the warp then walks the (sample, corner) pairs.
// Both run persistent CTAs that sweep contiguous item ranges (neighbouring
// queries sample neighbouring pixels, so rows are reused from L1), issue a
// batch of gathers before consuming any, and send corners outside the level
// to a zero row instead of branching.
// Single-use data (locations, weights, logits, offsets, outputs) is read and
// written with evict-first hints so that the value map, which every sample
// gathers from, keeps the L2.  The gather is the whole cost ("Deformable
// DETR" wiki page, "Limitations": deformable sampling means unordered memory
// access); there is no dense contraction, so no tensor-core path.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

constexpr int kWarps = 8;  // warps per CTA

// One corner of one sample: the address of its row (already offset to the
// batch entry and head, not yet to the lane's chunk) and its weight (bilinear
// weight times attention weight) twice, as the operand pair of __ffma2_rn.
// A corner outside the level points at kZeroRow with weight 0, so the gather
// loop needs neither a predicate nor a bounds check.
struct __align__(16) Corner {
    const char *row;
    float2 w;
};

// 512 bytes of zeros: the row that corners outside the level read.
__device__ __align__(128) float4 kZeroRow[32] = {};

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

// One 16-byte chunk of a value row: loaded raw (4 registers), widened to
// float pairs only when it is consumed, so a batch of loads in flight costs
// the same registers for fp32 and bf16.
template <typename VT>
struct Pairs;

template <>
struct Pairs<float> {
    static constexpr int kN = 2;  // float pairs per chunk
    __device__ __forceinline__ static void widen(const uint4 &r, float2 (&v)[2])
    {
        v[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
        v[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
    }
};

template <>
struct Pairs<__nv_bfloat16> {
    static constexpr int kN = 4;
    __device__ __forceinline__ static void widen(const uint4 &r, float2 (&v)[4])
    {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)  // exact widening: bf16 bits become the high half
            v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    }
};

template <typename VT, int R, int P, bool kFused, bool kExact>
__global__ void __launch_bounds__(kWarps * 32, 3)
    fwd_kernel_wide(const __grid_constant__ FwdParams p)
{
    constexpr int kNP = Pairs<VT>::kN;  // float pairs per 16-byte chunk
    constexpr int kSlots = 32 / R;      // (sample, corner) pairs per warp instruction
    constexpr int kItems = 32 / P;      // items per warp per round
    // gathers issued before the first is consumed (64 pairs = 16 samples)
    // (at most 16 raw 16-byte chunks, 64 registers)
    constexpr int kB1 = (64 / kSlots) < 4 ? 4 : ((64 / kSlots) > 16 ? 16 : 64 / kSlots);
    // a batch covers kB*kSlots pairs and must stay inside the 4*P entries
    constexpr int kB = kB1 * kSlots <= 4 * P ? kB1 : (4 * P) / kSlots;
    static_assert(kB >= 1 && (4 * P) % (kB * kSlots) == 0, "batch must tile the entries");
    // Corner entries, corner-major with row stride P + 2 (= 2 mod 8): the
    // phase-1 stores (consecutive samples) and the phase-2 loads (four
    // corners of one or two samples) both fall in distinct banks.
    constexpr int kStride = P + 2;
    __shared__ Corner corners[kWarps][kItems][4 * kStride];
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
    const int npairs = 4 * LK;
    const int slot = lane / R;
    const int chunk = lane % R;
    const bool chunk_ok = kExact || chunk < p.nchunks;

    // This CTA sweeps the contiguous item range [begin, end): neighbouring
    // queries sample neighbouring pixels, so the sweep keeps rows in L1.
    const int64_t begin = (int64_t)blockIdx.x * p.chunk;
    const int64_t end = begin + p.chunk < p.items ? begin + p.chunk : p.items;

    for (int64_t item0 = begin + warp * kItems; item0 < end; item0 += kWarps * kItems) {
        // ---- phase 1: one sample per lane ---------------------------------
        {
            const int seg = lane / P;  // item within the round
            const int j = lane % P;    // sample within the item
            const int64_t item = item0 + seg;
            const bool act = j < LK && item < end;
            const int64_t si = item * LK + j;
            const int l = act ? j / K : 0;
            float lx = 0.f, ly = 0.f, a = 0.f;
            if constexpr (kFused) {
                const float z = act ? __ldcs(p.logits + si) : -INFINITY;
                const float mx = seg_max<P>(z);
                const float e = act ? expf(__fsub_rn(z, mx)) : 0.f;
                const float s = seg_sum<P>(e);
                a = __fdiv_rn(e, s);
                if (act) {
                    const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + si);
                    const int64_t nq = item / M;
                    if (p.ref_dim == 2) {
                        // point reference: offsets are level-l pixels
                        const float2 r = __ldg(reinterpret_cast<const float2 *>(p.ref) + nq);
                        lx = __fadd_rn(r.x, __fdiv_rn(o.x, (float)sW[l]));
                        ly = __fadd_rn(r.y, __fdiv_rn(o.y, (float)sH[l]));
                    } else {
                        // box reference (cx, cy, w, h): offsets are in box units
                        const float2 c = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq);
                        const float2 s2 =
                            __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
                        lx = __fadd_rn(c.x, __fmul_rn(o.x, s2.x));
                        ly = __fadd_rn(c.y, __fmul_rn(o.y, s2.y));
                    }
                    if (p.loc_out)
                        __stcs(reinterpret_cast<float2 *>(p.loc_out) + si, make_float2(lx, ly));
                    if (p.attn_out) __stcs(p.attn_out + si, a);
                }
            } else if (act) {
                const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + si);
                lx = t.x;
                ly = t.y;
                a = __ldcs(p.attn + si);
            }
            {  // every sample slot up to P gets four entries; unused ones read zeros
                const int H = sH[l], W = sW[l], start = sStart[l];
                const int m = (int)(item % M);
                const int64_t n = item / M / p.Lq;
                const char *mapb = static_cast<const char *>(p.value) +
                                   ((n * p.S * M + m) * (int64_t)D) * (int64_t)sizeof(VT);
                Corner c[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    c[q] = {reinterpret_cast<const char *>(kZeroRow), make_float2(0.f, 0.f)};
                float x, y, fx, fy;
                int x0, y0;
                if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int r = msda_row(start, H, W, y0 + (q >> 1), x0 + (q & 1));
                        if (r >= 0) {
                            const float wa = w[q] * a;
                            c[q] = {mapb + (int64_t)r * MD * (int64_t)sizeof(VT),
                                    make_float2(wa, wa)};
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) corners[warp][seg][q * kStride + j] = c[q];
            }
        }
        __syncwarp();

        // ---- phase 2: gather, item by item --------------------------------
#pragma unroll 1
        for (int it = 0; it < kItems; ++it) {
            const int64_t item = item0 + it;
            if (item >= end) break;  // uniform across the warp
            const int m = (int)(item % M);
            const int64_t nq = item / M;
            // byte offset of this lane's chunk in a row; lanes past the last chunk
            // (D*size not a power-of-two multiple of 16 bytes) re-read chunk 0 and
            // their sums are discarded, so no lane reads past a row
            const int lane_off = chunk_ok ? chunk * 16 : 0;
            float2 acc[kNP];
#pragma unroll
            for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
            const Corner *ent = corners[warp][it];
            for (int t0 = 0; t0 < npairs; t0 += kB * kSlots) {
                uint4 raw[kB];
                float w[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int t = t0 + b * kSlots + slot;  // pair t = (sample t/4, corner t%4)
                    const Corner e = ent[(t & 3) * kStride + (t >> 2)];
                    w[b] = e.w.x;
                    raw[b] = __ldg(reinterpret_cast<const uint4 *>(e.row + lane_off));
                }
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    float2 v[kNP];
                    Pairs<VT>::widen(raw[b], v);
                    const float2 wb = make_float2(w[b], w[b]);
#pragma unroll
                    for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(wb, v[i], acc[i]);
                }
            }
            // combine the slots of each chunk, store the item's D outputs
#pragma unroll
            for (int o = R; o < 32; o <<= 1)
#pragma unroll
                for (int i = 0; i < kNP; ++i) {
                    acc[i].x += __shfl_xor_sync(kFull, acc[i].x, o);
                    acc[i].y += __shfl_xor_sync(kFull, acc[i].y, o);
                }
            if (slot == 0 && chunk_ok) {
                float4 *dst = reinterpret_cast<float4 *>(p.out + nq * (int64_t)MD + m * D +
                                                         chunk * (2 * kNP));
#pragma unroll
                for (int i = 0; i < kNP / 2; ++i)
                    __stcs(dst + i, make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x,
                                                acc[2 * i + 1].y));
            }
        }
        __syncwarp();  // the next round overwrites this warp's corner entries
    }
}

// ---------------------------------------------------------------------------
// Fast path for value rows of at most 128 bytes (R <= 8 lanes per row).
//
// Lane layout: G = 32/R groups of R lanes; group g owns samples g, g+G, g+2G,
// ... of the item (all four corners of each), lane `chunk` of the group owns
// 16 bytes of every row.  So every lane forms the row addresses and weights
// it gathers with in its own registers -- no shared-memory entries -- and a
// warp instruction still gathers G whole rows, 16 bytes per lane.  The
// per-level metadata of a lane's sample slots is the same for every item and
// is read once.  Fused: lane j first forms sample j's location and attention
// weight (one IEEE divide per coordinate, one softmax per item), and the
// group lanes fetch them with three shuffles.
// ---------------------------------------------------------------------------
template <typename VT, int R, int NS, int NB, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, 3)
    fwd_kernel(const __grid_constant__ FwdParams p)
{
    static_assert(R <= 8 && NS * (32 / R) <= 32, "fast path shape");
    constexpr int G = 32 / R;           // samples gathered per warp instruction
    constexpr int kNP = Pairs<VT>::kN;  // float pairs per 16-byte chunk
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane / R;
    const int chunk = lane % R;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int nsl = (LK + G - 1) / G;  // sample slots in use, <= NS
    const bool chunk_ok = chunk < p.nchunks;
    // lanes past the last chunk of a row re-read chunk 0; their sums are discarded
    const int lane_off = chunk_ok ? chunk * 16 : 0;
    const char *zrow = reinterpret_cast<const char *>(kZeroRow) + lane_off;
    const int64_t rowbytes = (int64_t)MD * (int64_t)sizeof(VT);

    int lvW[NS], lvH[NS], lvS[NS];  // level of sample slot i (sample g + G*i)
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
        const char *mapb = static_cast<const char *>(p.value) +
                           (n * p.S * M + m) * (int64_t)D * (int64_t)sizeof(VT) + lane_off;

        float ax = 0.f, ay = 0.f, aa = 0.f;  // fused: sample `lane`'s location and weight
        if constexpr (kFused) {
            const bool act = lane < LK;
            const float z = act ? __ldcs(p.logits + sbase + lane) : -INFINITY;
            const float mx = warp_max(z);
            const float e = act ? expf(__fsub_rn(z, mx)) : 0.f;
            const float sum = warp_sum(e);
            aa = __fdiv_rn(e, sum);
            if (act) {
                const int l = lane / K;
                const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sbase + lane);
                if (p.ref_dim == 2) {
                    // point reference: offsets are level-l pixels
                    const float2 r = __ldg(reinterpret_cast<const float2 *>(p.ref) + nq);
                    ax = __fadd_rn(r.x, __fdiv_rn(o.x, (float)p.lv.W[l]));
                    ay = __fadd_rn(r.y, __fdiv_rn(o.y, (float)p.lv.H[l]));
                } else {
                    // box reference (cx, cy, w, h): offsets are in box units
                    const float2 c = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq);
                    const float2 s2 = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
                    ax = __fadd_rn(c.x, __fmul_rn(o.x, s2.x));
                    ay = __fadd_rn(c.y, __fmul_rn(o.y, s2.y));
                }
                if (p.loc_out)
                    __stcs(reinterpret_cast<float2 *>(p.loc_out) + sbase + lane,
                           make_float2(ax, ay));
                if (p.attn_out) __stcs(p.attn_out + sbase + lane, aa);
            }
        }

        float2 acc[kNP];
#pragma unroll
        for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i0 = 0; i0 < NS; i0 += NB) {
            if (i0 >= nsl) break;  // uniform across the warp
            const char *ptr[NB][4];
            float wt[NB][4];
#pragma unroll
            for (int u = 0; u < NB; ++u) {
                const int i = i0 + u;
                const int s = g + G * i;  // < 32
                const bool have = s < LK;
                float lx = 0.f, ly = 0.f, a = 0.f;
                if constexpr (kFused) {
                    lx = __shfl_sync(kFull, ax, s);
                    ly = __shfl_sync(kFull, ay, s);
                    a = __shfl_sync(kFull, aa, s);
                } else if (have) {
                    const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sbase + s);
                    lx = t.x;
                    ly = t.y;
                    a = __ldcs(p.attn + sbase + s);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ptr[u][c] = zrow;
                    wt[u][c] = 0.f;
                }
                float x, y, fx, fy;
                int x0, y0;
                if (have && msda_cell(lx, ly, lvH[i], lvW[i], x, y, x0, y0, fx, fy)) {
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = msda_row(lvS[i], lvH[i], lvW[i], y0 + (c >> 1), x0 + (c & 1));
                        if (r >= 0) {
                            ptr[u][c] = mapb + (int64_t)r * rowbytes;
                            wt[u][c] = w[c] * a;
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
            for (int u = 0; u < NB; ++u)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float2 v[kNP];
                    Pairs<VT>::widen(raw[u][c], v);
                    const float2 wb = make_float2(wt[u][c], wt[u][c]);
#pragma unroll
                    for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(wb, v[i], acc[i]);
                }
        }

        // sum over the G groups, then lanes 0..R-1 store the item's D outputs
#pragma unroll
        for (int o = R; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < kNP; ++i) {
                acc[i].x += __shfl_xor_sync(kFull, acc[i].x, o);
                acc[i].y += __shfl_xor_sync(kFull, acc[i].y, o);
            }
        if (g == 0 && chunk_ok) {
            float4 *dst = reinterpret_cast<float4 *>(p.out + nq * (int64_t)MD + m * D +
                                                     chunk * (2 * kNP));
#pragma unroll
            for (int i = 0; i < kNP / 2; ++i)
                __stcs(dst + i, make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x,
                                            acc[2 * i + 1].y));
        }
    }
}

template <typename VT, int R, int NS, bool kFused>
cudaError_t launch_fast(FwdParams p, cudaStream_t stream)
{
    constexpr int NB = NS < 2 ? NS : 2;  // sample slots gathered per batch (4 rows each)
    auto kern = fwd_kernel<VT, R, NS, NB, kFused>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kWarps);
    p.chunk = (p.items + ctas - 1) / ctas;
    p.chunk = (p.chunk + kWarps - 1) / kWarps * kWarps;
    const dim3 grid((unsigned)((p.items + p.chunk - 1) / p.chunk));
    kern<<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename VT, int R, bool kFused>
cudaError_t launch_fast_r(const FwdParams &p, cudaStream_t stream)
{
    constexpr int G = 32 / R;
    const int LK = p.L * p.K;
    const int nsl = (LK + G - 1) / G;  // sample slots per lane
    if (nsl <= 1) return launch_fast<VT, R, 1, kFused>(p, stream);
    if constexpr (G <= 16) {
        if (nsl <= 2) return launch_fast<VT, R, 2, kFused>(p, stream);
    }
    if constexpr (G <= 8) {
        if (nsl <= 4) return launch_fast<VT, R, 4, kFused>(p, stream);
    }
    if constexpr (G <= 4) {
        return launch_fast<VT, R, 8, kFused>(p, stream);
    }
    return cudaErrorInvalidValue;  // not reached: L*K <= 32
}


template <typename VT, int R, int P, bool kFused>
cudaError_t launch_p(FwdParams p, bool exact, cudaStream_t stream)
{
    constexpr int kRound = kWarps * (32 / P);  // items per CTA round
    auto kern = exact ? fwd_kernel_wide<VT, R, P, kFused, true>
                      : fwd_kernel_wide<VT, R, P, kFused, false>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kRound);
    p.chunk = (p.items + ctas - 1) / ctas;
    p.chunk = (p.chunk + kRound - 1) / kRound * kRound;
    const dim3 grid((unsigned)((p.items + p.chunk - 1) / p.chunk));
    kern<<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename VT, int R, bool kFused>
cudaError_t launch_r(const FwdParams &p, bool exact, cudaStream_t stream)
{
    // P: lanes per item in phase 1, a power of two >= L*K, and at least the 8/R
    // samples one warp instruction gathers, so a batch never leaves the entries
    const int LK = p.L * p.K;
    const int need = LK > 8 / R ? LK : 8 / R;
    if constexpr (8 / R <= 4) {
        if (need <= 4) return launch_p<VT, R, 4, kFused>(p, exact, stream);
    }
    if (need <= 8) return launch_p<VT, R, 8, kFused>(p, exact, stream);
    if (need <= 16) return launch_p<VT, R, 16, kFused>(p, exact, stream);
    return launch_p<VT, R, 32, kFused>(p, exact, stream);
}

template <typename VT, bool kFused>
cudaError_t launch_fwd_vt(const FwdParams &p, int R, cudaStream_t stream)
{
    const bool exact = p.nchunks == R;
    switch (R) {
    case 1: return launch_fast_r<VT, 1, kFused>(p, stream);
    case 2: return launch_fast_r<VT, 2, kFused>(p, stream);
    case 4: return launch_fast_r<VT, 4, kFused>(p, stream);
    case 8: return launch_fast_r<VT, 8, kFused>(p, stream);
    case 16: return launch_r<VT, 16, kFused>(p, exact, stream);
    case 32: return launch_r<VT, 32, kFused>(p, exact, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_forward(const FwdParams &p, bool bf16, bool fused, int lanes_per_row,
                           cudaStream_t stream)
{
    if (p.items == 0) return cudaSuccess;
    if (bf16)
        return fused ? launch_fwd_vt<__nv_bfloat16, true>(p, lanes_per_row, stream)
                     : launch_fwd_vt<__nv_bfloat16, false>(p, lanes_per_row, stream);
    return fused ? launch_fwd_vt<float, true>(p, lanes_per_row, stream)
                 : launch_fwd_vt<float, false>(p, lanes_per_row, stream);
}

}  // namespace msda
