// msda_fwd.cu -- forward kernels of the MSDeformAttn core (sm_100a).
//
// Computes, per batch entry n, query q and head m ("Deformable DETR" wiki
// page, "Multi-scale deformable attention" equation):
//   out[n,q,m,:] = sum_{l,k} A[n,q,m,l,k] * bilinear(value[n, level l, m, :], loc)
//
// Work decomposition.  An "item" is one (n, q, m); it has L*K samples.  A warp
// owns 32/P consecutive items, where P = max(4, next power of two >= L*K) is
// the number of lanes given to one item in phase 1.
//   1. Every lane owns one sample (lane j of an item's P-lane segment owns
//      sample j).  It reads the sample's location and weight -- or, fused,
//      forms them: the joint softmax over the item's L*K logits runs inside
//      the P-lane segment with xor shuffles, and the location map is an IEEE
//      divide and add -- finds the cell and writes four corner entries
//      (row offset, attention weight x bilinear weight) to shared memory.
//   2. The warp walks the 4*L*K (sample, corner) pairs of its items together.
//      A (pixel, head) row of D elements is split into 16-byte chunks; R lanes
//      cover one row and 32/R rows are gathered per warp instruction, so every
//      corner read is a coalesced 16-byte-per-lane load of whole rows (fp32,
//      D = 32: 8 lanes x 16 B, the four corners of a sample in one
//      instruction; bf16, D = 32: 4 lanes, two samples per instruction).
//      Lanes accumulate their chunk in fp32 with packed FMA (`__ffma2_rn`).
//   3. Xor shuffles combine the 32/R partial sums of a chunk, and lanes
//      0..R-1 store each item's D outputs.
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
    fwd_kernel(const __grid_constant__ FwdParams p)
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

template <typename VT, int R, int P, bool kFused>
cudaError_t launch_p(FwdParams p, bool exact, cudaStream_t stream)
{
    constexpr int kRound = kWarps * (32 / P);  // items per CTA round
    auto kern = exact ? fwd_kernel<VT, R, P, kFused, true> : fwd_kernel<VT, R, P, kFused, false>;
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
    case 1: return launch_r<VT, 1, kFused>(p, exact, stream);
    case 2: return launch_r<VT, 2, kFused>(p, exact, stream);
    case 4: return launch_r<VT, 4, kFused>(p, exact, stream);
    case 8: return launch_r<VT, 8, kFused>(p, exact, stream);
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
