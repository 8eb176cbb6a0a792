// msda_fwd.cu -- forward kernels of the MSDeformAttn core (sm_100a).
//
// Computes, per batch entry n, query q and head m ("Deformable DETR" wiki
// page, "Multi-scale deformable attention" equation):
//   out[n,q,m,:] = sum_{l,k} A[n,q,m,l,k] * bilinear(value[n, level l, m, :], loc)
//
// An "item" is one (n, q, m); it has L*K samples, each with four corner rows of
// D elements.  A (pixel, head) row is split into chunks and R lanes cover one
// row, so a warp instruction gathers 32/R whole rows: 16 bytes per lane in
// general (bf16, D = 32: R = 4), 32 bytes per lane with one 256-bit load for
// fp32 rows of D = 32 in a 32-byte aligned map (R = 4; otherwise eight
// 16-byte lanes); lanes accumulate their chunk in fp32 with packed FMA
// (`__ffma2_rn`).  Four kernels:
//   * fwd_kernel (rows of at most eight lanes, at most 32 samples per item;
//     items of 17..32 samples over 16-byte lanes go to fwd_kernel_item):
//     persistent CTAs whose warps take rounds of 32/P items grid-stride
//     (round r of CTA b starts at item (r * gridDim.x + b) * 8 * 32/P).
//     Lane j of an item's P-lane segment forms sample j's weight, location
//     and cell and writes four 8-byte (row offset, weight) corner entries to
//     shared memory; the warp then gathers the entries' rows, several
//     instructions in flight, and reduces the slot sums with a
//     reduce-scatter (see its comment).
//   * fwd_kernel_item (17..32 samples per item): one warp per item, a plain
//     grid over the items, the same entries and reduction.
//   * fwd_kernel_long (more than 32 samples): one warp per item and round,
//     samples taken in blocks of 32.
//   * fwd_kernel_wide (rows wider than eight lanes): each CTA sweeps one
//     contiguous item range with the same entries.
// A corner outside the level has no entry (row -1 or a zero row) and adds
// nothing.
// Single-use data (locations, weights, logits, offsets, outputs) is read and
// written with evict-first hints so that the value map, which every sample
// gathers from, keeps the L2.  The gather is the whole cost ("Deformable
// DETR" wiki page, "Limitations": deformable sampling means unordered memory
// access); there is no dense contraction, so no tensor-core path.
#include "msda_common.cuh"
#include "msda_internal.h"
#include "msda_rows.cuh"

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
    // rows of more than R 16-byte chunks (R = 32: over 512 bytes) take passes
    // of R chunks; the entries, which hold whole-row addresses, serve them all
    const int npass = R == 32 ? (p.nchunks + R - 1) / R : 1;  // narrower rows: one pass

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
            const int64_t si = item * LK + j;                               // per head
            const int64_t sl = msda_loc_item(item, p.dM, p.G, p.dHg) * LK + j;  // per group
            const int l = act ? j / K : 0;
            float lx = 0.f, ly = 0.f, a = 0.f;
            if constexpr (kFused) {
                a = seg_softmax<P>(act ? __ldcs(p.logits + si) : 0.f, act);
                if (act) {
                    const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sl);
                    const float2 loc =
                        msda_fused_location(p.ref, p.ref_dim, (int64_t)fastdiv(p.dM, (unsigned)item), o.x, o.y, sH[l], sW[l]);
                    lx = loc.x;
                    ly = loc.y;
                    if (p.loc_out && msda_group_first(item, p.dM, p.dHg))  // group's first head
                        __stcs(reinterpret_cast<float2 *>(p.loc_out) + sl, make_float2(lx, ly));
                    if (p.attn_out) __stcs(p.attn_out + si, a);
                }
            } else if (act) {
                const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sl);
                lx = t.x;
                ly = t.y;
                a = __ldcs(p.attn + si);
            }
            {  // every sample slot up to P gets four entries; unused ones read zeros
                const int H = sH[l], W = sW[l], start = sStart[l];
                const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
                const int m = ix.m;
                const int64_t n = ix.n;
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

        // ---- phase 2: gather, item by item, R chunks of the row per pass ----
#pragma unroll 1
        for (int it = 0; it < kItems * npass; ++it) {
            const int64_t item = item0 + it / npass;
            if (item >= end) break;  // uniform across the warp
            const int ck = (it % npass) * R + chunk;  // this lane's chunk of the row
            const bool chunk_ok = kExact || ck < p.nchunks;
            const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
            const int m = ix.m;
            const int64_t nq = ix.nq;
            // byte offset of this lane's chunk in a row; lanes past the last chunk
            // (D*size not a power-of-two multiple of 16 bytes) re-read chunk 0 and
            // their sums are discarded, so no lane reads past a row
            const int64_t lane_off = chunk_ok ? (int64_t)ck * 16 : 0;
            float2 acc[kNP];
#pragma unroll
            for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
            const Corner *ent = corners[warp][it / npass];
            for (int t0 = 0; t0 < npairs; t0 += kB * kSlots) {
                uint4 raw[kB];
                float w[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int t = t0 + b * kSlots + slot;  // pair t = (sample t/4, corner t%4)
                    const Corner e = ent[(t & 3) * kStride + (t >> 2)];
                    const char *row = e.row;
                    w[b] = e.w.x;
                    if (row != reinterpret_cast<const char *>(kZeroRow) &&
                        !msda_in_map(p.check, p.check_limit,
                                     (row - static_cast<const char *>(p.value) + lane_off) /
                                         (int64_t)sizeof(VT),
                                     16 / (int)sizeof(VT))) {
                        row = reinterpret_cast<const char *>(kZeroRow);  // skipped: reads zeros
                        w[b] = 0.f;
                    }
                    raw[b] = __ldg(reinterpret_cast<const uint4 *>(row + lane_off));
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
                                                         (int64_t)ck * (2 * kNP));
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
// The gather is bound by how many rows the L2 can return per second, which
// needs many warps per SM more than deep per-warp queues, so this kernel keeps
// its register footprint small (FWD_MIN_CTAS CTAs of 8 warps per SM):
//   * a warp loops over rounds of 32/P items (P = lanes per item); lane j of
//     an item's P-lane segment owns sample j, whose level metadata it keeps in
//     registers for the whole kernel;
//   * the inputs of the next round (logits and offsets, or locations and
//     weights) are loaded while the current round gathers;
//   * phase 1 forms the location, weight and cell of each sample and stores
//     its four corners as 8-byte (row offset, weight) entries, corner-major
//     with stride P + 2 so stores and loads are free of bank conflicts;
//   * phase 2 gathers FWD_BATCH corner-row groups before consuming them; a
//     corner outside the level predicates its load and its FMA off.
// ---------------------------------------------------------------------------
#ifndef MSDA_FWD_BATCH
#define MSDA_FWD_BATCH 4
#endif
#ifndef MSDA_FWD_MIN_CTAS
#define MSDA_FWD_MIN_CTAS 4
#endif
#ifndef MSDA_FWD_PREFETCH
#define MSDA_FWD_PREFETCH 1  // load the next round's inputs during this round's gathers
#endif

template <typename VT, int EPL, int R, int P, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, MSDA_FWD_MIN_CTAS)
    fwd_kernel(const __grid_constant__ FwdParams p)
{
    using LL = LaneLoad<VT, EPL>;
    constexpr int kSlots = 32 / R;      // (sample, corner) pairs per warp instruction
    constexpr int kItems = 32 / P;      // items per round
    constexpr int kStride = P + 2;      // = 2 mod 8 for P >= 8: conflict-free entries
    constexpr int kNP = EPL / 2;        // float pairs per lane
    // the same bytes in flight per lane whatever the lane width: 32-byte
    // lanes take half as many corner-row groups per batch
    constexpr int kLaneB = EPL * (int)sizeof(VT);
    constexpr int kB0 = kLaneB > 16 ? MSDA_FWD_BATCH * 16 / kLaneB : MSDA_FWD_BATCH;
    constexpr int kB = kB0 * kSlots <= 4 * P ? kB0 : (4 * P) / kSlots;
    static_assert(kB >= 1 && (4 * P) % (kB * kSlots) == 0, "a batch must tile the entries");
    __shared__ int2 ent[kWarps][kItems][4 * kStride];  // (row element offset | -1, weight)

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    static_assert(kSlots % 4 == 0, "a warp instruction covers whole samples");

    // phase-1 role: sample j of the round's item `seg`
    const int seg = lane / P;
    const int j = lane % P;
    const bool jact = j < LK;
    const int lvl = jact ? j / K : 0;
    const int H = p.lv.H[lvl], W = p.lv.W[lvl], start = p.lv.start[lvl];

    // phase-2 role: 16-byte chunk `chunk` of the rows in slot `slot`
    const int slot = lane / R;
    const int chunk = lane % R;
    const bool chunk_ok = chunk < p.nchunks;
    // lanes past the last chunk of a row re-read chunk 0; their sums are discarded
    const int lane_elem = (chunk_ok ? chunk : 0) * EPL;

    const int64_t stride = (int64_t)gridDim.x * kWarps * kItems;
    int64_t item0 = ((int64_t)blockIdx.x * kWarps + warp) * kItems;

    // inputs of this lane's sample in the round starting at item0
    float pa = 0.f, pb = 0.f, pc = 0.f;
    auto fetch = [&](int64_t i0) {
        const int64_t item = i0 + seg;
        pa = pb = pc = 0.f;
        if (jact && item < p.items) {
            const int64_t si = item * LK + j;                               // per head
            const int64_t sl = msda_loc_item(item, p.dM, p.G, p.dHg) * LK + j;  // per group
            if constexpr (kFused) {
                pa = __ldcs(p.logits + si);
                const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sl);
                pb = o.x;
                pc = o.y;
            } else {
                const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sl);
                pb = t.x;
                pc = t.y;
                pa = __ldcs(p.attn + si);
            }
        }
    };
    if (MSDA_FWD_PREFETCH) fetch(item0);

    for (; item0 < p.items; item0 += stride) {
        if (!MSDA_FWD_PREFETCH) fetch(item0);
        // ---- phase 1 -------------------------------------------------------
        const int64_t item = item0 + seg;
        const bool act = jact && item < p.items;
        const int64_t si = item * LK + j;
        float lx, ly, a;
        if constexpr (kFused) {
            a = seg_softmax<P>(pa, act);  // joint over the item's L*K logits
            lx = ly = 0.f;
            if (act) {
                const float2 loc = msda_fused_location(p.ref, p.ref_dim, (int64_t)fastdiv(p.dM, (unsigned)item), pb, pc, H, W);
                lx = loc.x;
                ly = loc.y;
                if (p.loc_out && msda_group_first(item, p.dM, p.dHg))  // group's first head
                    __stcs(reinterpret_cast<float2 *>(p.loc_out) +
                               msda_loc_item(item, p.dM, p.G, p.dHg) * LK + j,
                           make_float2(lx, ly));
                if (p.attn_out) __stcs(p.attn_out + si, a);
            }
        } else {
            lx = pb;
            ly = pc;
            a = pa;
        }
        if (MSDA_FWD_PREFETCH) fetch(item0 + stride);  // loads while this round gathers
        {
            int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
            float x, y, fx, fy;
            int x0, y0;
            if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = msda_row(start, H, W, y0 + (c >> 1), x0 + (c & 1));
                    if (r >= 0) e[c] = make_int2(r * MD, __float_as_int(w[c] * a));
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) ent[warp][seg][c * kStride + j] = e[c];
        }
        __syncwarp();

        // ---- phase 2: gather, item by item --------------------------------
#pragma unroll 1
        for (int it = 0; it < kItems; ++it) {
            const int64_t itm = item0 + it;
            if (itm >= p.items) break;  // uniform
            const ItemIdx ix = msda_item_idx(itm, p.dM, p.dLq);
            const int m = ix.m;
            const int64_t nq = ix.nq;
            const int64_t n = ix.n;
            const int64_t vbe = (n * p.S * M + m) * (int64_t)D + lane_elem;
            const VT *vb = static_cast<const VT *>(p.value) + vbe;
            const int2 *en = ent[warp][it];
            float2 acc[kNP];
#pragma unroll
            for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
            // pair t = (sample t/4, corner t%4); slot s takes corner s%4 of sample
            // s/4 + kSlots/4 * (instruction), so its entries sit at one lane base
            const int2 *enl = en + (slot & 3) * kStride + (slot >> 2);
            for (int s0 = 0; s0 < LK; s0 += kB * (kSlots / 4)) {
                int2 e[kB];
                typename LL::Raw raw[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    e[b] = enl[s0 + b * (kSlots / 4)];
                    if (e[b].x >= 0 && !msda_in_map(p.check, p.check_limit, vbe + e[b].x, EPL))
                        e[b].x = -1;  // bounds-checked build: skipped, reads as zero
                    if (e[b].x >= 0) raw[b] = LL::load(vb + e[b].x);
                }
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    if (e[b].x >= 0) {
                        float2 v[kNP];
                        LL::widen(raw[b], v);
                        const float wb = __int_as_float(e[b].y);
                        const float2 w2 = make_float2(wb, wb);
#pragma unroll
                        for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(w2, v[i], acc[i]);
                    }
                }
            }
            store_row<R, EPL>(acc, lane, chunk, chunk_ok, p.out + nq * (int64_t)MD + m * D);
        }
        __syncwarp();  // the next round overwrites this warp's entries
    }
}

// ---------------------------------------------------------------------------
// Items of more than 32 samples (32 < L*K <= kMaxLK), any row width.
//
// One warp per item and round.  The fused softmax comes first: lane j holds
// the logits of samples j, j + 32, ... in registers and the warp forms the
// joint statistics (long_softmax).  The samples are then taken in blocks of
// 32, lane j owning sample blk*32 + j: phase 1 writes the block's corner
// entries, phase 2 gathers them into the same accumulators, and the item's
// output is stored once after its last block.
// ---------------------------------------------------------------------------
template <typename VT, int EPL, int R, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, 3)
    fwd_kernel_long(const __grid_constant__ FwdParams p)
{
    using LL = LaneLoad<VT, EPL>;
    constexpr int kSlots = 32 / R;  // (sample, corner) pairs per warp instruction
    constexpr int kStride = 34;     // = 2 mod 8: conflict-free entries
    constexpr int kNP = EPL / 2;
    constexpr int kB = MSDA_FWD_BATCH;
    constexpr int kNB = kMaxLK / 32;
    static_assert(128 % (kB * kSlots) == 0, "a batch must tile a block's entries");
    __shared__ int2 ent[kWarps][4 * kStride];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int nblk = (LK + 31) / 32;
    const int slot = lane / R;
    const int chunk = lane % R;
    // rows of more than R 16-byte chunks (R = 32: over 512 bytes) take passes
    // of R chunks, each a unit of work of its own; pass 0 stores the sampling
    // locations and weights
    const int npass = R == 32 ? (p.nchunks + R - 1) / R : 1;  // narrower rows: one pass
    const int64_t units = p.items * npass;

    for (int64_t u = (int64_t)blockIdx.x * kWarps + warp; u < units;
         u += (int64_t)gridDim.x * kWarps) {
        const int64_t item = npass == 1 ? u : u / npass;
        const int pass = (int)(u - item * npass);
        const int ck = pass * R + chunk;  // this lane's chunk of the row
        const bool chunk_ok = ck < p.nchunks;
        const int64_t lane_elem = (int64_t)(chunk_ok ? ck : 0) * EPL;
        const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
        const int m = ix.m;
        const int64_t nq = ix.nq;
        const int64_t n = ix.n;
        const int64_t vbe = (n * p.S * M + m) * (int64_t)D + lane_elem;
        const VT *vb = static_cast<const VT *>(p.value) + vbe;
        const int64_t litem = msda_loc_item(item, p.dM, p.G, p.dHg);
        const bool first_head = msda_group_first_m(m, p.dHg);
        float z[kNB];
        float sum = 1.f;
        if constexpr (kFused) {
#pragma unroll
            for (int b = 0; b < kNB; ++b) {
                const int s = b * 32 + lane;
                z[b] = s < LK ? __ldcs(p.logits + item * LK + s) : -INFINITY;
            }
            sum = long_softmax<kNB>(z);
        }
        float2 acc[kNP];
#pragma unroll
        for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);

#pragma unroll 1
        for (int blk = 0; blk < nblk; ++blk) {
            // ---- phase 1: sample blk*32 + lane --------------------------------
            {
                const int s = blk * 32 + lane;
                const bool act = s < LK;
                const int64_t si = item * LK + s;    // per head
                const int64_t sl = litem * LK + s;   // per group
                const int l = act ? s / K : 0;
                const int H = p.lv.H[l], W = p.lv.W[l], start = p.lv.start[l];
                float lx = 0.f, ly = 0.f, a = 0.f;
                if (act) {
                    if constexpr (kFused) {
                        a = __fdiv_rn(pick<kNB>(z, blk), sum);
                        const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sl);
                        const float2 loc = msda_fused_location(p.ref, p.ref_dim, nq, o.x, o.y, H, W);
                        lx = loc.x;
                        ly = loc.y;
                        if (p.loc_out && first_head && pass == 0)
                            __stcs(reinterpret_cast<float2 *>(p.loc_out) + sl, make_float2(lx, ly));
                        if (p.attn_out && pass == 0) __stcs(p.attn_out + si, a);
                    } else {
                        const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sl);
                        lx = t.x;
                        ly = t.y;
                        a = __ldcs(p.attn + si);
                    }
                }
                int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
                float x, y, fx, fy;
                int x0, y0;
                if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = msda_row(start, H, W, y0 + (c >> 1), x0 + (c & 1));
                        if (r >= 0) e[c] = make_int2(r * MD, __float_as_int(w[c] * a));
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) ent[warp][c * kStride + lane] = e[c];
            }
            __syncwarp();

            // ---- phase 2: the block's (sample, corner) pairs ------------------
            const int rem = LK - blk * 32;
            const int npairs = 4 * (rem < 32 ? rem : 32);
            for (int t0 = 0; t0 < npairs; t0 += kB * kSlots) {
                int2 e[kB];
                typename LL::Raw raw[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int t = t0 + b * kSlots + slot;  // < 128: entries past L*K hold -1
                    e[b] = ent[warp][(t & 3) * kStride + (t >> 2)];
                    if (e[b].x >= 0 && !msda_in_map(p.check, p.check_limit, vbe + e[b].x, EPL))
                        e[b].x = -1;  // bounds-checked build: skipped, reads as zero
                    if (e[b].x >= 0) raw[b] = LL::load(vb + e[b].x);
                }
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    if (e[b].x >= 0) {
                        float2 v[kNP];
                        LL::widen(raw[b], v);
                        const float wb = __int_as_float(e[b].y);
                        const float2 w2 = make_float2(wb, wb);
#pragma unroll
                        for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(w2, v[i], acc[i]);
                    }
                }
            }
            __syncwarp();  // the next block overwrites the entries
        }
#pragma unroll
        for (int o = R; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < kNP; ++i) {
                acc[i].x += __shfl_xor_sync(kFull, acc[i].x, o);
                acc[i].y += __shfl_xor_sync(kFull, acc[i].y, o);
            }
        if (slot == 0 && chunk_ok) {
            float4 *dst =
                reinterpret_cast<float4 *>(p.out + nq * (int64_t)MD + m * D + (int64_t)ck * EPL);
#pragma unroll
            for (int i = 0; i < kNP / 2; ++i)
                __stcs(dst + i, make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x,
                                            acc[2 * i + 1].y));
        }
    }
}

template <typename VT, int EPL, bool kFused>
cudaError_t launch_long(FwdParams p, cudaStream_t stream)
{
    const int lanes = (p.D + EPL - 1) / EPL;  // D*size is a multiple of 16 bytes
    p.nchunks = lanes;
    const dim3 block(kWarps * 32);
    const int64_t units = p.items * ((lanes + 31) / 32);  // (item, pass of 32 lanes) pairs
    auto go = [&](auto kern) {
        const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, units, kWarps);
        kern<<<(unsigned)ctas, block, 0, stream>>>(p);
        return cudaGetLastError();
    };
    if (lanes <= 1) return go(fwd_kernel_long<VT, EPL, 1, kFused>);
    if (lanes <= 2) return go(fwd_kernel_long<VT, EPL, 2, kFused>);
    if (lanes <= 4) return go(fwd_kernel_long<VT, EPL, 4, kFused>);
    if (lanes <= 8) return go(fwd_kernel_long<VT, EPL, 8, kFused>);
    if (lanes <= 16) return go(fwd_kernel_long<VT, EPL, 16, kFused>);
    return go(fwd_kernel_long<VT, EPL, 32, kFused>);
}

// ---------------------------------------------------------------------------
// Items of 17..32 samples, rows of at most 8 lanes: one warp per item and a
// grid over all items (no persistent loop), two corner-row groups in flight,
// so the kernel needs few registers and the GPU keeps 48 (fp32) or 64 (bf16)
// warps per SM in flight.  On B200 that beats the fast kernel for these items
// (stress workload, bf16: 2.06 ms against 2.53 ms; fp32 L*K = 32: 6-7%
// faster), while for items of at most 16 samples the fast kernel's batching
// wins (encoder: 181 us against 218 us).
// ---------------------------------------------------------------------------
#ifndef MSDA_FWD_ITEM_BATCH
#define MSDA_FWD_ITEM_BATCH 2  // corner-row groups loaded before the first is used
#endif

// Resident CTAs of 8 warps per SM: bf16 at 32 registers (64 warps per SM),
// fp32 at 40 (48 warps), the best of the measured shapes.
template <typename VT>
constexpr int item_min_ctas()
{
    return sizeof(VT) == 2 ? 8 : 6;
}

template <typename VT, int EPL, int R, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, item_min_ctas<VT>())
    fwd_kernel_item(const __grid_constant__ FwdParams p)
{
    using LL = LaneLoad<VT, EPL>;
    constexpr int kSlots = 32 / R;  // (sample, corner) pairs per warp instruction
    constexpr int kNP = EPL / 2;
    constexpr int kStride = 34;     // corner-major entries, conflict-free
    __shared__ int2 ent[kWarps][4 * kStride];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * kWarps + warp;
    if (item >= p.items) return;  // whole warp; no block-wide barrier follows
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
    const int m = ix.m;
    const int64_t nq = ix.nq;
    const int64_t n = ix.n;

    // ---- phase 1: sample `lane` -------------------------------------------
    {
        const bool act = lane < LK;
        const int64_t si = item * LK + lane;                               // per head
        const int64_t sl = msda_loc_item(item, p.dM, p.G, p.dHg) * LK + lane;  // per group
        const int l = act ? lane / K : 0;
        const int H = p.lv.H[l], W = p.lv.W[l], start = p.lv.start[l];
        float lx = 0.f, ly = 0.f, a = 0.f;
        if constexpr (kFused) {
            a = seg_softmax<32>(act ? __ldcs(p.logits + si) : 0.f, act);
            if (act) {
                const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sl);
                const float2 loc = msda_fused_location(p.ref, p.ref_dim, nq, o.x, o.y, H, W);
                lx = loc.x;
                ly = loc.y;
                if (p.loc_out && (msda_group_first_m(m, p.dHg)))  // the group's first head
                    __stcs(reinterpret_cast<float2 *>(p.loc_out) + sl, make_float2(lx, ly));
                if (p.attn_out) __stcs(p.attn_out + si, a);
            }
        } else if (act) {
            const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sl);
            lx = t.x;
            ly = t.y;
            a = __ldcs(p.attn + si);
        }
        int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
        float x, y, fx, fy;
        int x0, y0;
        if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
            const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
            const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int r = msda_row(start, H, W, y0 + (c >> 1), x0 + (c & 1));
                if (r >= 0) e[c] = make_int2(r * MD, __float_as_int(w[c] * a));
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) ent[warp][c * kStride + lane] = e[c];
    }
    __syncwarp();

    // ---- phase 2: the item's (sample, corner) pairs, four loads in flight ----
    const int slot = lane / R;
    const int chunk = lane % R;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_elem = (chunk_ok ? chunk : 0) * EPL;
    const int64_t vbe = (n * p.S * M + m) * (int64_t)D + lane_elem;
    const VT *vb = static_cast<const VT *>(p.value) + vbe;
    float2 acc[kNP];
#pragma unroll
    for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
    constexpr int kB = MSDA_FWD_ITEM_BATCH;
    static_assert(128 % (kB * kSlots) == 0, "a batch must tile the entries");
    static_assert(kSlots % 4 == 0, "a warp instruction covers whole samples");
    // slot s takes corner s%4 of samples s/4, s/4 + kSlots/4, ... (entries
    // past L*K hold -1)
    const int2 *enl = ent[warp] + (slot & 3) * kStride + (slot >> 2);
    for (int s0 = 0; s0 < LK; s0 += kB * (kSlots / 4)) {
        int2 e[kB];
        typename LL::Raw raw[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            e[b] = enl[s0 + b * (kSlots / 4)];
            if (e[b].x >= 0 && !msda_in_map(p.check, p.check_limit, vbe + e[b].x, EPL))
                e[b].x = -1;  // bounds-checked build: skipped, reads as zero
            if (e[b].x >= 0) raw[b] = LL::load(vb + e[b].x);
        }
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            if (e[b].x >= 0) {
                float2 v[kNP];
                LL::widen(raw[b], v);
                const float wb = __int_as_float(e[b].y);
                const float2 w2 = make_float2(wb, wb);
#pragma unroll
                for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(w2, v[i], acc[i]);
            }
        }
    }
    store_row<R, EPL>(acc, lane, chunk, chunk_ok, p.out + nq * (int64_t)MD + m * D);
}

template <typename VT, int EPL, int R, bool kFused>
cudaError_t launch_item(const FwdParams &p, cudaStream_t stream)
{
    const dim3 grid((unsigned)((p.items + kWarps - 1) / kWarps));
    fwd_kernel_item<VT, EPL, R, kFused><<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename VT, int EPL, int R, int P, bool kFused>
cudaError_t launch_fast(FwdParams p, cudaStream_t stream)
{
    constexpr int kRound = kWarps * (32 / P);  // items per CTA round
    auto kern = fwd_kernel<VT, EPL, R, P, kFused>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kRound);
    fwd_kernel<VT, EPL, R, P, kFused><<<(unsigned)ctas, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

#ifndef MSDA_FWD_ITEM_MIN_LK
#define MSDA_FWD_ITEM_MIN_LK 17  // items of at least this many samples: fwd_kernel_item
#endif

template <typename VT, int EPL, int R, bool kFused>
cudaError_t launch_fast_r(const FwdParams &p, cudaStream_t stream)
{
    // P: a power of two >= L*K, >= 8 (conflict-free entry stride) and >= the
    // 8/R samples one warp instruction gathers
    const int LK = p.L * p.K;
    if (LK <= 8) return launch_fast<VT, EPL, R, 8, kFused>(p, stream);
    if (LK <= 16 && !one_item_rounds((const void *)fwd_kernel<VT, EPL, R, 16, kFused>,
                                     (const void *)fwd_kernel<VT, EPL, R, 32, kFused>, kWarps,
                                     p.items))
        return launch_fast<VT, EPL, R, 16, kFused>(p, stream);
    return launch_fast<VT, EPL, R, 32, kFused>(p, stream);
}

// Items of up to this many samples take the fast path; larger ones the wide
// kernel's one-warp-per-item loop.
#ifndef MSDA_FWD_FAST_MAX_LK
#define MSDA_FWD_FAST_MAX_LK 32
#endif

template <typename VT, int EPL, bool kFused>
cudaError_t launch_item_r(FwdParams p, int lanes, cudaStream_t stream)
{
    p.nchunks = lanes;
    if (lanes <= 1) return launch_item<VT, EPL, 1, kFused>(p, stream);
    if (lanes <= 2) return launch_item<VT, EPL, 2, kFused>(p, stream);
    if (lanes <= 4) return launch_item<VT, EPL, 4, kFused>(p, stream);
    return launch_item<VT, EPL, 8, kFused>(p, stream);
}

template <typename VT, int EPL, bool kFused>
cudaError_t launch_fast_lanes(FwdParams p, int lanes, cudaStream_t stream)
{
    p.nchunks = lanes;
    if (lanes <= 1) return launch_fast_r<VT, EPL, 1, kFused>(p, stream);
    if (lanes <= 2) return launch_fast_r<VT, EPL, 2, kFused>(p, stream);
    if (lanes <= 4) return launch_fast_r<VT, EPL, 4, kFused>(p, stream);
    return launch_fast_r<VT, EPL, 8, kFused>(p, stream);
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
    constexpr int E16 = 16 / (int)sizeof(VT);  // elements of a 16-byte lane
    const int LK = p.L * p.K;
    if (LK > kLaneLK) return launch_long<VT, E16, kFused>(p, stream);
    // items of 17..32 samples, rows of at most eight 16-byte lanes
    if (LK >= MSDA_FWD_ITEM_MIN_LK && p.D % E16 == 0 && p.D / E16 <= 8)
        return launch_item_r<VT, E16, kFused>(p, p.D / E16, stream);
    // fast path: bf16 rows of 32 elements take four 16-byte lanes (with the
    // one-element-per-lane reduce-scatter: encoder bf16 forward 174 -> 166 us
    // against 8-byte lanes); otherwise lanes of four elements where a row
    // needs at most eight of them, else 16-byte lanes
    if (LK <= MSDA_FWD_FAST_MAX_LK) {
        if constexpr (E16 == 4) {
            // fp32 rows of 32 elements in four 32-byte lanes (256-bit loads)
            // where the map is 32-byte aligned: encoder forward 163.8 -> 160.6 us
            // (compass 172.0 -> 167.9 us) against eight 16-byte lanes
            if (p.D == 32 && (reinterpret_cast<uintptr_t>(p.value) & 31) == 0) {
                FwdParams q = p;
                q.nchunks = 4;
                return launch_fast_r<VT, 8, 4, kFused>(q, stream);
            }
        }
        if (E16 == 8 && p.D == 32) return launch_fast_lanes<VT, E16, kFused>(p, 4, stream);
        if (p.D % 4 == 0 && p.D / 4 <= 8) return launch_fast_lanes<VT, 4, kFused>(p, p.D / 4, stream);
        if (E16 != 4 && p.D % E16 == 0 && p.D / E16 <= 8)
            return launch_fast_lanes<VT, E16, kFused>(p, p.D / E16, stream);
    }
    const bool exact = p.nchunks % R == 0;  // every lane holds a chunk in every pass
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
