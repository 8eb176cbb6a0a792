// msda_bwd.cu -- backward kernel of the MSDeformAttn core (sm_100a).
//
// Gradients flow through the bilinear interpolation to the value map, the
// sampling locations and the attention weights ("Deformable DETR" wiki
// page, "Deformable attention module"; "Deformable Attention" glossary
// page, the interpolation passes gradients on).  Per sample, with
// g = grad_out[n,q,m,:], corner weights w_j(fx, fy) and t_j = <v_j, g>:
//   dA        = sum_j w_j t_j
//   dloc_x    = A * W * sum_j (dw_j/dfx) t_j,  dloc_y = A * H * sum_j (dw_j/dfy) t_j
//   dvalue_j += A * w_j * g            (scatter; corners inside the level)
//
// Two kernels:
//   * bwd_kernel (value rows of at most 128 bytes): a group of R lanes owns
//     whole samples and sums their four corners inside each lane, so only
//     the R chunk lanes need combining (see its comment).  Persistent CTAs
//     whose warps take rounds of items grid-stride.
//   * bwd_kernel_wide (rows wider than 128 bytes): one warp per item; lane j
//     finds sample j's cell and stores per-corner (row offset, w, dw/dfx,
//     dw/dfy) in shared memory; min(32, 4R) lanes work on one sample, and the
//     per-sample partial sums are reduced every 8 samples with a butterfly
//     reduce-scatter.
// Both scatter A w_j g with one vector `red.global.add.v4.f32` per 16 bytes.
#include "msda_common.cuh"
#include "msda_internal.h"
#include "msda_rows.cuh"

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

// Generic path (any row width): one warp per item, partial sums of 32 lanes
// reduced every 8 samples.  Used for rows wider than 128 bytes.  The item's
// samples are taken in blocks of 32 (one per lane in phase 1), so any L*K up
// to kMaxLK works.
template <typename VT, int R, bool kFused>
__global__ void __launch_bounds__(kWarps * 32)
    bwd_kernel_wide(const __grid_constant__ BwdParams p)
{
    constexpr int kVec = Chunk<VT>::kVec;
    constexpr int kSpan = (4 * R < 32) ? 4 * R : 32;  // lanes per sample
    constexpr int kGroups = 32 / kSpan;               // samples in flight per warp
    constexpr int kCornerSlots = kSpan / R;           // 4, 2 or 1
    constexpr int kCpl = 4 / kCornerSlots;            // corners per lane
    constexpr int kPer = kNV / kSpan;                 // finished sums per lane
    constexpr int kNB = kMaxLK / 32;

    __shared__ CornerB corners[kWarps][32 * 4];
    __shared__ float sA[kWarps][32];
    __shared__ int sH[kMaxLevels], sW[kMaxLevels], sStart[kMaxLevels];
    // fused: every sample's weight and its gradient, and the block's offsets
    __shared__ float sAll[kWarps][kFused ? kMaxLK : 1];
    __shared__ float sdA[kWarps][kFused ? kMaxLK : 1];
    __shared__ float2 sOff[kWarps][kFused ? 32 : 1];

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
    const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
    const int m = ix.m;
    const int64_t nq = ix.nq;
    const int64_t n = ix.n;

    const int grp = lane / kSpan;
    const int lin = lane % kSpan;
    const int cslot = lin / R;
    const int chunk = lin % R;
    const bool chunk_ok = chunk < p.nchunks;
    // rows of more than R 16-byte chunks (R = 32: over 512 bytes) take passes
    // of R chunks; pass 0 keeps its grad_out chunk in registers
    const int npass = R == 32 ? (p.nchunks + R - 1) / R : 1;  // narrower rows: one pass

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

    const int64_t litem = msda_loc_item(item, p.dM, p.G, p.dHg);
    const bool shared_loc = p.Hg > 1;

    float2 bwh = make_float2(0.f, 0.f);       // fused, box reference: (w, h)
    float rx = 0.f, ry = 0.f, rw = 0.f, rh = 0.f;  // fused: this lane's reference-point terms
    if constexpr (kFused) {
        // the joint softmax over all L*K logits, as the fused forward forms it
        float z[kNB];
#pragma unroll
        for (int b = 0; b < kNB; ++b) {
            const int s = b * 32 + lane;
            z[b] = s < LK ? __ldcs(p.logits + item * LK + s) : -INFINITY;
        }
        const float sum = long_softmax<kNB>(z);
#pragma unroll
        for (int b = 0; b < kNB; ++b) {
            const int s = b * 32 + lane;
            if (s < LK) sAll[warp][s] = __fdiv_rn(z[b], sum);
        }
        if (p.ref_dim == 4) bwh = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
        __syncwarp();
    }

    for (int blk0 = 0; blk0 < LK; blk0 += 32) {
        const int nb = LK - blk0 < 32 ? LK - blk0 : 32;  // samples in this block
        const int64_t sbase = item * LK + blk0;   // per head
        const int64_t lbase = litem * LK + blk0;  // per group
        // ---- phase 1: cell and corner derivatives of sample blk0 + lane -------
        if (lane < nb) {
            const int l = (blk0 + lane) / K;
            const int H = sH[l], W = sW[l], start = sStart[l];
            float2 t;
            if constexpr (kFused) {
                const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + lbase + lane);
                t = msda_fused_location(p.ref, p.ref_dim, nq, o.x, o.y, H, W);
                sA[warp][lane] = sAll[warp][blk0 + lane];
                sOff[warp][lane] = o;
            } else {
                t = __ldg(reinterpret_cast<const float2 *>(p.loc) + lbase + lane);
                sA[warp][lane] = __ldg(p.attn + sbase + lane);
            }
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

        // ---- phase 2/3 ---------------------------------------------------
        const int per_batch = kBatch * kGroups;
        for (int b0 = 0; b0 < nb; b0 += per_batch) {
            float v[kNV];
#pragma unroll
            for (int i = 0; i < kNV; ++i) v[i] = 0.f;
#pragma unroll
            for (int it = 0; it < kBatch; ++it) {
                const int s = b0 + it * kGroups + grp;
                if (s < nb) {
                    const float a = sA[warp][s];
#pragma unroll
                    for (int ci = 0; ci < kCpl; ++ci) {
                        const CornerB e = corners[warp][s * 4 + cslot * kCpl + ci];
                        float t = 0.f;
                        if (e.off >= 0 && chunk_ok &&
                            msda_in_map(p.check, p.check_limit, rowbase + e.off, kVec)) {
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
                        for (int ps = 1; ps < npass && e.off >= 0; ++ps) {
                            const int ck = ps * R + chunk;
                            if (ck >= p.nchunks) break;
                            const int64_t eo = e.off + (int64_t)ps * R * kVec;
                            if (!msda_in_map(p.check, p.check_limit, rowbase + eo, kVec))
                                continue;
                            float gp[kVec], x[kVec];
                            const float4 *gq = reinterpret_cast<const float4 *>(
                                p.grad_out + nq * (int64_t)(M * D) + m * D + (int64_t)ck * kVec);
#pragma unroll
                            for (int i = 0; i < kVec / 4; ++i) {
                                const float4 q4 = __ldg(gq + i);
                                gp[4 * i] = q4.x;
                                gp[4 * i + 1] = q4.y;
                                gp[4 * i + 2] = q4.z;
                                gp[4 * i + 3] = q4.w;
                            }
                            Chunk<VT>::load(vbase + eo, x);
#pragma unroll
                            for (int i = 0; i < kVec; ++i) t = fmaf(x[i], gp[i], t);
                            const float aw = a * e.w;
                            float *dst = gvbase + eo;
#pragma unroll
                            for (int i = 0; i < kVec; i += 4)
                                red_add_v4(dst + i, aw * gp[i], aw * gp[i + 1], aw * gp[i + 2],
                                           aw * gp[i + 3]);
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
                if (qty < 3 && s < nb) {
                    const int64_t si = sbase + s;
                    const float a = sA[warp][s];
                    if (qty == 0) {
                        if constexpr (kFused)
                            sdA[warp][blk0 + s] = v[i];
                        else if (p.grad_attn)
                            p.grad_attn[si] = v[i];
                        continue;
                    }
                    const int l = (blk0 + s) / K;
                    const float scale = (qty == 1) ? (float)sW[l] : (float)sH[l];
                    const float gl = a * (scale * v[i]);  // d loc
                    float go = gl;                        // the value written per location
                    float *base = p.grad_loc;
                    if constexpr (kFused) {
                        base = p.grad_off;
                        if (p.ref_dim == 2) {
                            go = a * v[i];  // loc = ref + off / W_l: d off = d loc / W_l
                        } else {
                            const float2 o = sOff[warp][s];
                            go = gl * (qty == 1 ? bwh.x : bwh.y);  // loc = c + off * (w, h)
                            if (qty == 1)
                                rw = fmaf(gl, o.x, rw);
                            else
                                rh = fmaf(gl, o.y, rh);
                        }
                        if (qty == 1)
                            rx += gl;
                        else
                            ry += gl;
                    }
                    if (base) {
                        float *dst = base + 2 * (lbase + s) + (qty - 1);
                        if (shared_loc)
                            atomicAdd(dst, go);  // the group's heads add into one location
                        else
                            *dst = go;
                    }
                }
            }
        }
        __syncwarp();  // the next block overwrites corners and weights
    }

    if constexpr (kFused) {
        // softmax Jacobian over all L*K samples: d z_s = A_s (dA_s - sum_j A_j dA_j)
        float dpart = 0.f;
        for (int s = lane; s < LK; s += 32) dpart = fmaf(sAll[warp][s], sdA[warp][s], dpart);
        const float dot = warp_sum(dpart);
        if (p.grad_logits)
            for (int s = lane; s < LK; s += 32)
                __stcs(p.grad_logits + item * LK + s, sAll[warp][s] * (sdA[warp][s] - dot));
        // reference point: sum over this head's samples, then add over heads
        rx = warp_sum(rx);
        ry = warp_sum(ry);
        if (p.ref_dim == 4) {
            rw = warp_sum(rw);
            rh = warp_sum(rh);
        }
        if (lane == 0 && p.grad_ref) {
            float *gr = p.grad_ref + nq * p.ref_dim;
            atomicAdd(gr, rx);
            atomicAdd(gr + 1, ry);
            if (p.ref_dim == 4) {
                atomicAdd(gr + 2, rw);
                atomicAdd(gr + 3, rh);
            }
        }
    }
}

// Fast path for D <= 32 (R = D/4 <= 8 lanes per row, four elements per lane).
//
// The scatter into grad_value is bound by the L2's atomic throughput (a flat
// cost per 128-byte row), the gathers by how many rows the L2 returns per
// second; both want many warps per SM, so the footprint stays small:
//   * a warp loops over rounds of 32/P items; lane j of an item's P-lane
//     segment owns sample j (level metadata in registers for the whole
//     kernel) and loads the next round's location and weight while the
//     current round gathers;
//   * phase 1 stores, per corner, an 8-byte (row offset | -1, A*w) entry
//     (corner-major, stride P + 2: no bank conflicts) and, per sample,
//     (fx, fy, A*W, A*H);
//   * phase 2 takes R instructions at a time (each gathers 32/R corner rows,
//     16 bytes per lane), forms t = <v_chunk, g_chunk>, scatters A*w*g_chunk
//     with a vector reduction, reduces t over the R chunk lanes with a
//     butterfly reduce-scatter, weights it with (w, dw/dfx, dw/dfy) of its
//     corner and sums the four corner lanes with two xor steps.
#ifndef MSDA_BWD_MIN_CTAS
#define MSDA_BWD_MIN_CTAS 3
#endif
#ifndef MSDA_BWD_MIN_CTAS_F32
#define MSDA_BWD_MIN_CTAS_F32 2
#endif

// Resident CTAs of 8 warps per SM.  fp32 rows of eight lanes (D = 32) run at
// 2 CTAs (128 registers, no spills; encoder backward 471 -> 448 us, fused
// 556 -> 529 us on B200); bf16, whose value chunks take half the registers,
// and narrower rows, which need fewer, are fastest at 3.
template <typename VT, int R>
constexpr int bwd_min_ctas()
{
    return (sizeof(VT) == 4 && R == 8) ? MSDA_BWD_MIN_CTAS_F32 : MSDA_BWD_MIN_CTAS;
}

template <typename VT, int R, int P, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, bwd_min_ctas<VT, R>())
    bwd_kernel(const __grid_constant__ BwdParams p)
{
    static_assert(R <= 8, "fast path: at least four pairs per warp instruction");
    constexpr int kVec = 4;                // value elements per lane
    using Raw = typename Lane4<VT>::Raw;
    constexpr int kSlots = 32 / R;         // pairs per warp instruction
    constexpr int kSG = kSlots / 4;        // samples per warp instruction
    constexpr int kB = R;                  // instructions per batch: one t per lane after stage A
    constexpr int kBS = kB * kSG;          // samples per batch (= 8)
    constexpr int kItems = 32 / P;
    constexpr int kStride = P + 2;
    static_assert(kBS <= P && P % kBS == 0, "a batch must stay inside the P sample slots");
    constexpr int kNB = P / kBS;           // batches per item, at most
    __shared__ int2 ent[kWarps][kItems][4 * kStride];  // (row element offset | -1, A*w)
    __shared__ float4 smp[kWarps][kItems][P];          // (fx, fy, A*W, A*H)
    __shared__ float4 smq[kWarps][kItems][kFused ? P : 1];  // fused: (A, off_x, off_y, dA)
    __shared__ float2 sdl[kWarps][kItems][kFused ? P : 1];  // fused: d loc per sample

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;

    const int seg = lane / P;
    const int j = lane % P;
    const bool jact = j < LK;
    const int lvl = jact ? j / K : 0;
    const int H = p.lv.H[lvl], W = p.lv.W[lvl], start = p.lv.start[lvl];

    const int slot = lane / R;
    const int chunk = lane % R;
    const int corner = slot & 3;
    const int sg = slot >> 2;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_elem = (chunk_ok ? chunk : 0) * kVec;
    const bool cx = corner & 1, cy = corner >> 1;

    const int64_t stride = (int64_t)gridDim.x * kWarps * kItems;
    int64_t item0 = ((int64_t)blockIdx.x * kWarps + warp) * kItems;

    // this lane's sample inputs: (loc.x, loc.y, A), or fused (off.x, off.y, logit)
    float pl_x = 0.f, pl_y = 0.f, pa = 0.f;
    auto fetch = [&](int64_t i0) {
        const int64_t item = i0 + seg;
        pl_x = pl_y = pa = 0.f;
        if (jact && item < p.items) {
            const int64_t si = item * LK + j;                               // per head
            const int64_t sl = msda_loc_item(item, p.dM, p.G, p.dHg) * LK + j;  // per group
            if constexpr (kFused) {
                const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + sl);
                pl_x = o.x;
                pl_y = o.y;
                pa = __ldcs(p.logits + si);
            } else {
                const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + sl);
                pl_x = t.x;
                pl_y = t.y;
                pa = __ldcs(p.attn + si);
            }
        }
    };
    fetch(item0);

    for (; item0 < p.items; item0 += stride) {
        // ---- phase 1 -------------------------------------------------------
        {
            const int64_t item = item0 + seg;
            const bool act = jact && item < p.items;
            float lx = pl_x, ly = pl_y, a = pa;
            if constexpr (kFused) {
                // the fused forward's softmax and location map, bit for bit
                const float ox = pl_x, oy = pl_y;
                a = seg_softmax<P>(pa, act);
                lx = ly = 0.f;
                if (act) {
                    const float2 loc = msda_fused_location(p.ref, p.ref_dim, (int64_t)fastdiv(p.dM, (unsigned)item), ox, oy, H, W);
                    lx = loc.x;
                    ly = loc.y;
                }
                smq[warp][seg][j] = make_float4(act ? a : 0.f, ox, oy, 0.f);
            }
            fetch(item0 + stride);
            int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
            float4 rec = make_float4(0.f, 0.f, 0.f, 0.f);
            float x, y, fx, fy;
            int x0, y0;
            if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = msda_row(start, H, W, y0 + (c >> 1), x0 + (c & 1));
                    if (r >= 0) e[c] = make_int2(r * MD, __float_as_int(a * w[c]));
                }
                rec = make_float4(fx, fy, a * (float)W, a * (float)H);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) ent[warp][seg][c * kStride + j] = e[c];
            smp[warp][seg][j] = rec;
        }
        __syncwarp();

        // ---- phase 2 -------------------------------------------------------
#pragma unroll 1
        for (int it = 0; it < kItems; ++it) {
            const int64_t itm = item0 + it;
            if (itm >= p.items) break;  // uniform
            const ItemIdx ix = msda_item_idx(itm, p.dM, p.dLq);
            const int m = ix.m;
            const int64_t nq = ix.nq;
            const int64_t n = ix.n;
            const int64_t sbase = itm * LK;                                 // per head
            const int64_t lbase = msda_loc_item(itm, p.dM, p.G, p.dHg) * LK;    // per group
            const int64_t mapoff = (n * p.S * M + m) * (int64_t)D;
            const int64_t vbe = mapoff + lane_elem;
            const VT *vb = static_cast<const VT *>(p.value) + vbe;
            float *gvb = p.grad_value + mapoff + chunk * kVec;
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
            const int2 *en = ent[warp][it] + corner * kStride + sg;
            float2 bwh = make_float2(0.f, 0.f);  // fused box reference: (w, h)
            if constexpr (kFused) {
                if (p.ref_dim == 4) bwh = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
            }
#pragma unroll
            for (int bi = 0; bi < kNB; ++bi) {
                const int s0 = bi * kBS;
                if (s0 >= LK) break;  // uniform
                int2 e[kB];
                Raw raw[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    e[b] = en[s0 + b * kSG];  // sample s0 + b*kSG + sg, this lane's corner
                    // bounds-checked build: a skipped corner reads zeros and scatters nothing
                    if (e[b].x >= 0 && !msda_in_map(p.check, p.check_limit, vbe + e[b].x, kVec))
                        e[b].x = -1;
                    if (e[b].x >= 0) raw[b] = Lane4<VT>::load(vb + e[b].x);
                }
                float t[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    t[b] = 0.f;
                    if (e[b].x >= 0) {
                        float v[kVec];
                        Lane4<VT>::widen(raw[b], v);
#pragma unroll
                        for (int i = 0; i < kVec; ++i) t[b] = fmaf(v[i], gv[i], t[b]);
                        if (chunk_ok) {
                            const float aw = __int_as_float(e[b].y);
                            float *dst = gvb + e[b].x;
#pragma unroll
                            for (int i = 0; i < kVec; i += 4)
                                red_add_v4(dst + i, aw * gv[i], aw * gv[i + 1], aw * gv[i + 2],
                                           aw * gv[i + 3]);
                        }
                    }
                }
                // stage A: sum t over the R chunk lanes; this lane keeps instruction b = chunk
                reduce_scatter_n<R, kB, kB>(t, lane);
                const int s = s0 + chunk * kSG + sg;
                const float4 rec = smp[warp][it][s < P ? s : 0];
                const float fx = rec.x, fy = rec.y;
                const float wxc = cx ? fx : __fsub_rn(1.f, fx);
                const float wyc = cy ? fy : __fsub_rn(1.f, fy);
                float q0 = (wyc * wxc) * t[0];                 // w t
                float q1 = (cx ? wyc : -wyc) * t[0];           // dw/dfx t
                float q2 = (cy ? wxc : -wxc) * t[0];           // dw/dfy t
                // stage B: sum over the four corner lanes of the sample
#pragma unroll
                for (int o = R; o < 4 * R; o <<= 1) {
                    q0 += __shfl_xor_sync(kFull, q0, o);
                    q1 += __shfl_xor_sync(kFull, q1, o);
                    q2 += __shfl_xor_sync(kFull, q2, o);
                }
                if (corner == 0 && s < LK) {
                    const int64_t si = sbase + s;
                    const float dlx = rec.z * q1, dly = rec.w * q2;  // d loc
                    if constexpr (!kFused) {
                        if (p.grad_attn) __stcs(p.grad_attn + si, q0);
                        if (p.grad_loc) msda_put_loc_grad(p.grad_loc, lbase + s, dlx, dly, p.Hg > 1);
                    } else {
                        const float4 r2 = smq[warp][it][s];  // (A, off_x, off_y, -)
                        float2 goff;
                        if (p.ref_dim == 2) {
                            // loc = ref + off / W_l: d off = d loc / W_l = A * (sum dw t)
                            goff = make_float2(r2.x * q1, r2.x * q2);
                        } else {
                            // loc = c + off * (w, h)
                            goff = make_float2(dlx * bwh.x, dly * bwh.y);
                        }
                        if (p.grad_off)
                            msda_put_loc_grad(p.grad_off, lbase + s, goff.x, goff.y, p.Hg > 1);
                        smq[warp][it][s].w = q0;                 // dA, for the softmax Jacobian
                        sdl[warp][it][s] = make_float2(dlx, dly);  // for the reference gradient
                    }
                }
            }
        }
        if constexpr (kFused) {
            // Per item of the round, in the phase-1 layout (lane = seg * P + j
            // holds sample j of item seg), segment sums over the item's samples:
            //   softmax Jacobian  d z_j = A_j (dA_j - sum_i A_i dA_i)
            //   reference point   d ref = sum_j d loc_j (box: also sum_j d loc_j * off_j)
            __syncwarp();
            const int64_t item = item0 + seg;
            const bool act = jact && item < p.items;
            const float4 ad = act ? smq[warp][seg][j] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float2 dl = act ? sdl[warp][seg][j] : make_float2(0.f, 0.f);
            const float dot = seg_sum<P>(ad.x * ad.w);
            if (act && p.grad_logits) __stcs(p.grad_logits + item * LK + j, ad.x * (ad.w - dot));
            const float rx = seg_sum<P>(dl.x), ry = seg_sum<P>(dl.y);
            float rw = 0.f, rh = 0.f;
            if (p.ref_dim == 4) {
                rw = seg_sum<P>(dl.x * ad.y);
                rh = seg_sum<P>(dl.y * ad.z);
            }
            // summed over the item's samples here, over its heads by the atomics
            if (j == 0 && item < p.items && p.grad_ref) {
                float *gr = p.grad_ref + (int64_t)fastdiv(p.dM, (unsigned)item) * p.ref_dim;
                atomicAdd(gr, rx);
                atomicAdd(gr + 1, ry);
                if (p.ref_dim == 4) {
                    atomicAdd(gr + 2, rw);
                    atomicAdd(gr + 3, rh);
                }
            }
        }
        __syncwarp();
    }
}

// Items of more than 32 samples (32 < L*K <= kMaxLK) with rows of at most
// eight 4-element lanes.  The lane layout, entries and two-stage reduction are
// bwd_kernel's with one item per warp and round; the item's samples are taken
// in blocks of 32 (lane j of phase 1 owns sample blk*32 + j).  The fused
// variant forms the joint softmax first (long_softmax, as the forward does)
// and keeps every sample's (A, dA) in shared memory until the softmax
// Jacobian's sum over all blocks is known.
template <typename VT, int R, bool kFused>
__global__ void __launch_bounds__(kWarps * 32, MSDA_BWD_MIN_CTAS)
    bwd_kernel_long(const __grid_constant__ BwdParams p)
{
    static_assert(R <= 8, "at least four pairs per warp instruction");
    constexpr int kVec = 4;
    using Raw = typename Lane4<VT>::Raw;
    constexpr int kSlots = 32 / R;
    constexpr int kSG = kSlots / 4;  // samples per warp instruction
    constexpr int kB = R;            // instructions per batch
    constexpr int kBS = kB * kSG;    // samples per batch (= 8)
    constexpr int kStride = 34;
    constexpr int kNBt = 32 / kBS;   // batches per block
    constexpr int kNB = kMaxLK / 32;
    __shared__ int2 ent[kWarps][4 * kStride];                // (row offset | -1, A*w)
    __shared__ float4 smp[kWarps][32];                       // (fx, fy, A*W, A*H)
    __shared__ float4 smq[kWarps][kFused ? 32 : 1];          // fused: (A, off_x, off_y, -)
    __shared__ float2 smd[kWarps][kFused ? kMaxLK : 1];      // fused: (A, dA) per sample

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int nblk = (LK + 31) / 32;

    const int slot = lane / R;
    const int chunk = lane % R;
    const int corner = slot & 3;
    const int sg = slot >> 2;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_elem = (chunk_ok ? chunk : 0) * kVec;
    const bool cx = corner & 1, cy = corner >> 1;

    for (int64_t item = (int64_t)blockIdx.x * kWarps + warp; item < p.items;
         item += (int64_t)gridDim.x * kWarps) {
        const ItemIdx ix = msda_item_idx(item, p.dM, p.dLq);
        const int m = ix.m;
        const int64_t nq = ix.nq;
        const int64_t n = ix.n;
        const int64_t mapoff = (n * p.S * M + m) * (int64_t)D;
        const int64_t vbe = mapoff + lane_elem;
        const VT *vb = static_cast<const VT *>(p.value) + vbe;
        float *gvb = p.grad_value + mapoff + chunk * kVec;
        const int64_t lbase = msda_loc_item(item, p.dM, p.G, p.dHg) * LK;  // per group
        float gv[kVec];
        if (chunk_ok) {
            const float4 t = __ldcs(reinterpret_cast<const float4 *>(
                p.grad_out + nq * (int64_t)MD + m * D + chunk * kVec));
            gv[0] = t.x;
            gv[1] = t.y;
            gv[2] = t.z;
            gv[3] = t.w;
        } else {
            gv[0] = gv[1] = gv[2] = gv[3] = 0.f;
        }
        float z[kNB];
        float sum = 1.f;
        float2 bwh = make_float2(0.f, 0.f);
        if constexpr (kFused) {
#pragma unroll
            for (int b = 0; b < kNB; ++b) {
                const int s = b * 32 + lane;
                z[b] = s < LK ? __ldcs(p.logits + item * LK + s) : -INFINITY;
            }
            sum = long_softmax<kNB>(z);
            if (p.ref_dim == 4) bwh = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
        }
        float dpart = 0.f, rx = 0.f, ry = 0.f, rw = 0.f, rh = 0.f;

#pragma unroll 1
        for (int blk = 0; blk < nblk; ++blk) {
            // ---- phase 1: sample blk*32 + lane ---------------------------------
            {
                const int s = blk * 32 + lane;
                const bool act = s < LK;
                const int64_t si = item * LK + s;  // per head
                const int l = act ? s / K : 0;
                const int H = p.lv.H[l], W = p.lv.W[l], start = p.lv.start[l];
                float lx = 0.f, ly = 0.f, a = 0.f;
                if constexpr (kFused) {
                    float ox = 0.f, oy = 0.f;
                    if (act) {
                        a = __fdiv_rn(pick<kNB>(z, blk), sum);
                        const float2 o =
                            __ldcs(reinterpret_cast<const float2 *>(p.off) + lbase + s);
                        ox = o.x;
                        oy = o.y;
                        const float2 loc = msda_fused_location(p.ref, p.ref_dim, nq, ox, oy, H, W);
                        lx = loc.x;
                        ly = loc.y;
                    }
                    smq[warp][lane] = make_float4(a, ox, oy, 0.f);
                } else if (act) {
                    const float2 t = __ldcs(reinterpret_cast<const float2 *>(p.loc) + lbase + s);
                    lx = t.x;
                    ly = t.y;
                    a = __ldcs(p.attn + si);
                }
                int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
                float4 rec = make_float4(0.f, 0.f, 0.f, 0.f);
                float x, y, fx, fy;
                int x0, y0;
                if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = msda_row(start, H, W, y0 + (c >> 1), x0 + (c & 1));
                        if (r >= 0) e[c] = make_int2(r * MD, __float_as_int(a * w[c]));
                    }
                    rec = make_float4(fx, fy, a * (float)W, a * (float)H);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) ent[warp][c * kStride + lane] = e[c];
                smp[warp][lane] = rec;
            }
            __syncwarp();

            // ---- phase 2: batches of 8 samples ----------------------------------
            const int2 *en = ent[warp] + corner * kStride + sg;
#pragma unroll
            for (int bi = 0; bi < kNBt; ++bi) {
                const int s0 = bi * kBS;
                if (blk * 32 + s0 >= LK) break;  // uniform
                int2 e[kB];
                Raw raw[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    e[b] = en[s0 + b * kSG];
                    if (e[b].x >= 0 && !msda_in_map(p.check, p.check_limit, vbe + e[b].x, kVec))
                        e[b].x = -1;  // bounds-checked build: reads zeros, scatters nothing
                    if (e[b].x >= 0) raw[b] = Lane4<VT>::load(vb + e[b].x);
                }
                float t[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    t[b] = 0.f;
                    if (e[b].x >= 0) {
                        float v[kVec];
                        Lane4<VT>::widen(raw[b], v);
#pragma unroll
                        for (int i = 0; i < kVec; ++i) t[b] = fmaf(v[i], gv[i], t[b]);
                        if (chunk_ok) {
                            const float aw = __int_as_float(e[b].y);
                            red_add_v4(gvb + e[b].x, aw * gv[0], aw * gv[1], aw * gv[2],
                                       aw * gv[3]);
                        }
                    }
                }
                reduce_scatter_n<R, kB, kB>(t, lane);
                const int s = s0 + chunk * kSG + sg;  // sample within the block, < 32
                const int sgl = blk * 32 + s;
                const float4 rec = smp[warp][s];
                const float fx = rec.x, fy = rec.y;
                const float wxc = cx ? fx : __fsub_rn(1.f, fx);
                const float wyc = cy ? fy : __fsub_rn(1.f, fy);
                float q0 = (wyc * wxc) * t[0];
                float q1 = (cx ? wyc : -wyc) * t[0];
                float q2 = (cy ? wxc : -wxc) * t[0];
#pragma unroll
                for (int o = R; o < 4 * R; o <<= 1) {
                    q0 += __shfl_xor_sync(kFull, q0, o);
                    q1 += __shfl_xor_sync(kFull, q1, o);
                    q2 += __shfl_xor_sync(kFull, q2, o);
                }
                if (corner == 0 && sgl < LK) {
                    const int64_t si = item * LK + sgl;
                    const float dlx = rec.z * q1, dly = rec.w * q2;
                    if constexpr (!kFused) {
                        if (p.grad_attn) __stcs(p.grad_attn + si, q0);
                        if (p.grad_loc)
                            msda_put_loc_grad(p.grad_loc, lbase + sgl, dlx, dly, p.Hg > 1);
                    } else {
                        const float4 r2 = smq[warp][s];  // (A, off_x, off_y, -)
                        float2 goff;
                        if (p.ref_dim == 2) {
                            goff = make_float2(r2.x * q1, r2.x * q2);
                        } else {
                            goff = make_float2(dlx * bwh.x, dly * bwh.y);
                            rw = fmaf(dlx, r2.y, rw);
                            rh = fmaf(dly, r2.z, rh);
                        }
                        if (p.grad_off)
                            msda_put_loc_grad(p.grad_off, lbase + sgl, goff.x, goff.y, p.Hg > 1);
                        rx += dlx;
                        ry += dly;
                        dpart = fmaf(r2.x, q0, dpart);
                        smd[warp][sgl] = make_float2(r2.x, q0);
                    }
                }
            }
            __syncwarp();  // the next block overwrites the entries and records
        }
        if constexpr (kFused) {
            // softmax Jacobian over all L*K samples: d z_s = A_s (dA_s - sum_j A_j dA_j)
            const float dot = warp_sum(dpart);
            for (int s = lane; s < LK; s += 32) {
                const float2 ad = smd[warp][s];
                if (p.grad_logits) __stcs(p.grad_logits + item * LK + s, ad.x * (ad.y - dot));
            }
            rx = warp_sum(rx);
            ry = warp_sum(ry);
            if (p.ref_dim == 4) {
                rw = warp_sum(rw);
                rh = warp_sum(rh);
            }
            if (lane == 0 && p.grad_ref) {
                float *gr = p.grad_ref + nq * p.ref_dim;
                atomicAdd(gr, rx);
                atomicAdd(gr + 1, ry);
                if (p.ref_dim == 4) {
                    atomicAdd(gr + 2, rw);
                    atomicAdd(gr + 3, rh);
                }
            }
            __syncwarp();  // the next item overwrites smd
        }
    }
}

template <typename VT, bool kFused>
cudaError_t launch_long(const BwdParams &p, cudaStream_t stream)
{
    const int r4 = p.D / 4;  // D % 4 == 0 and r4 <= 8 checked by the caller
    BwdParams q = p;
    q.nchunks = r4;
    auto go = [&](auto kern) {
        const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, q.items, kWarps);
        kern<<<(unsigned)ctas, kWarps * 32, 0, stream>>>(q);
        return cudaGetLastError();
    };
    if (r4 <= 1) return go(bwd_kernel_long<VT, 1, kFused>);
    if (r4 <= 2) return go(bwd_kernel_long<VT, 2, kFused>);
    if (r4 <= 4) return go(bwd_kernel_long<VT, 4, kFused>);
    return go(bwd_kernel_long<VT, 8, kFused>);
}

template <typename VT, int R, int P, bool kFused>
cudaError_t launch_fast(const BwdParams &p, cudaStream_t stream)
{
    constexpr int kRound = kWarps * (32 / P);
    auto kern = bwd_kernel<VT, R, P, kFused>;
    const int64_t ctas = persistent_ctas((const void *)kern, kWarps * 32, p.items, kRound);
    bwd_kernel<VT, R, P, kFused><<<(unsigned)ctas, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename VT, int R, bool kFused = false>
cudaError_t launch_fast_r(const BwdParams &p, cudaStream_t stream)
{
    // P: a power of two >= L*K and >= the 8 samples of one batch
    const int LK = p.L * p.K;
    if (LK <= 8) return launch_fast<VT, R, 8, kFused>(p, stream);
    if (LK <= 16 && !one_item_rounds((const void *)bwd_kernel<VT, R, 16, kFused>,
                                     (const void *)bwd_kernel<VT, R, 32, kFused>, kWarps,
                                     p.items))
        return launch_fast<VT, R, 16, kFused>(p, stream);
    return launch_fast<VT, R, 32, kFused>(p, stream);
}

// Rows wider than the fast path's eight 4-element lanes (or not a multiple
// of 4 elements): one warp per item, R lanes of 16 bytes per row.
template <typename VT, bool kFused>
cudaError_t launch_wide(const BwdParams &p, int R, cudaStream_t stream)
{
    const dim3 block(kWarps * 32);
    const dim3 grid((unsigned)((p.items + kWarps - 1) / kWarps));
    switch (R) {
    case 1: bwd_kernel_wide<VT, 1, kFused><<<grid, block, 0, stream>>>(p); break;
    case 2: bwd_kernel_wide<VT, 2, kFused><<<grid, block, 0, stream>>>(p); break;
    case 4: bwd_kernel_wide<VT, 4, kFused><<<grid, block, 0, stream>>>(p); break;
    case 8: bwd_kernel_wide<VT, 8, kFused><<<grid, block, 0, stream>>>(p); break;
    case 16: bwd_kernel_wide<VT, 16, kFused><<<grid, block, 0, stream>>>(p); break;
    case 32: bwd_kernel_wide<VT, 32, kFused><<<grid, block, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename VT>
cudaError_t launch_bwd_fused_vt(const BwdParams &p, int R, cudaStream_t stream)
{
    const int r4 = p.D / 4;
    if (p.D % 4 != 0 || r4 > 8) return launch_wide<VT, true>(p, R, stream);
    if (p.L * p.K > kLaneLK) return launch_long<VT, true>(p, stream);
    BwdParams q = p;
    q.nchunks = r4;
    if (r4 <= 1) return launch_fast_r<VT, 1, true>(q, stream);
    if (r4 <= 2) return launch_fast_r<VT, 2, true>(q, stream);
    if (r4 <= 4) return launch_fast_r<VT, 4, true>(q, stream);
    return launch_fast_r<VT, 8, true>(q, stream);
}

template <typename VT>
cudaError_t launch_bwd_vt(const BwdParams &p, int R, cudaStream_t stream)
{
    // fast path: four elements per lane, R4 = D/4 lanes per (fp32) gradient row
    const int r4 = p.D / 4;
    if (p.D % 4 == 0 && r4 <= 8 && p.L * p.K > kLaneLK) return launch_long<VT, false>(p, stream);
    if (p.D % 4 == 0 && r4 <= 8) {
        BwdParams q = p;
        q.nchunks = r4;
        if (r4 <= 1) return launch_fast_r<VT, 1>(q, stream);
        if (r4 <= 2) return launch_fast_r<VT, 2>(q, stream);
        if (r4 <= 4) return launch_fast_r<VT, 4>(q, stream);
        return launch_fast_r<VT, 8>(q, stream);
    }
    return launch_wide<VT, false>(p, R, stream);
}

}  // namespace

cudaError_t launch_backward_fused(const BwdParams &p, bool bf16, int lanes_per_row,
                                  cudaStream_t stream)
{
    if (p.items == 0) return cudaSuccess;
    return bf16 ? launch_bwd_fused_vt<__nv_bfloat16>(p, lanes_per_row, stream)
                : launch_bwd_fused_vt<float>(p, lanes_per_row, stream);
}

cudaError_t launch_backward(const BwdParams &p, bool bf16, int lanes_per_row,
                            cudaStream_t stream)
{
    if (p.items == 0) return cudaSuccess;
    return bf16 ? launch_bwd_vt<__nv_bfloat16>(p, lanes_per_row, stream)
                : launch_bwd_vt<float>(p, lanes_per_row, stream);
}

}  // namespace msda
