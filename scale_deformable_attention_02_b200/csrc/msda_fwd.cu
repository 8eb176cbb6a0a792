// msda_fwd.cu -- forward kernels of the MSDeformAttn core (sm_100a).
//
// Computes, per batch entry n, query q and head m ("Deformable DETR" wiki
// page, "Multi-scale deformable attention" equation):
//   out[n,q,m,:] = sum_{l,k} A[n,q,m,l,k] * bilinear(value[n, level l, m, :], loc)
//
// Work decomposition (one warp per (n, q, m)):
//   1. Lane j < L*K owns sample j.  It reads the sample's location and weight
//      (fused: forms them from the reference point, the pixel offset and the
//      logit; the softmax runs across the lanes with shuffles), finds the cell
//      and writes four (row offset, weight) corner entries to shared memory.
//      The attention weight is folded into the corner weights.
//   2. The warp walks the 4*L*K (sample, corner) pairs.  A value row of one
//      head (D elements) is split into 16-byte chunks: R lanes cover a row and
//      32/R rows are gathered per warp instruction, so every corner read is a
//      coalesced 16-byte-per-lane load of a whole row (fp32 D = 32: 8 lanes x
//      16 B, four corners per instruction; bf16 D = 32: 4 lanes, two samples
//      per instruction).  Each lane accumulates its chunk in fp32 registers.
//   3. The 32/R partial sums of a chunk are combined with xor shuffles and
//      lanes 0..R-1 store the head's D outputs.
// The gather is the whole cost ("Deformable DETR" wiki page, "Limitations":
// deformable sampling means unordered memory access); there is no dense
// contraction, so no tensor-core path.
#include "msda_common.cuh"
#include "msda_internal.h"

namespace msda {
namespace {

constexpr int kWarps = 8;  // warps (items) per CTA

struct __align__(8) Corner {
    int off;  // element offset of the corner row inside the (n, m) map; -1 = outside
    float w;  // bilinear weight times the attention weight
};

template <typename VT, int R, bool kFused>
__global__ void __launch_bounds__(kWarps * 32)
    fwd_kernel(const __grid_constant__ FwdParams p)
{
    constexpr int kVec = Chunk<VT>::kVec;
    constexpr int kSlots = 32 / R;  // (sample, corner) pairs per warp instruction
    __shared__ Corner corners[kWarps][kMaxLK * 4];
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
    if (item >= p.items) return;  // whole warp leaves together

    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int m = (int)(item % M);
    const int64_t nq = item / M;  // n * Lq + q
    const int64_t n = nq / p.Lq;
    const int64_t sbase = item * LK;  // first sample of this (n, q, m)
    const bool act = lane < LK;
    const int l = act ? lane / K : 0;

    // ---- phase 1: location and weight of sample `lane` --------------------
    float lx = 0.f, ly = 0.f, a = 0.f;
    if constexpr (kFused) {
        // Joint softmax over the L*K logits of this head, max-subtracted.
        const float z = act ? __ldg(p.logits + sbase + lane) : -INFINITY;
        const float mx = warp_max(z);
        const float e = act ? expf(__fsub_rn(z, mx)) : 0.f;
        const float s = warp_sum(e);
        a = __fdiv_rn(e, s);
        if (act) {
            const float2 o = __ldg(reinterpret_cast<const float2 *>(p.off) + sbase + lane);
            if (p.ref_dim == 2) {
                // point reference: offsets are level-l pixels -> divide by the level size
                const float2 r = __ldg(reinterpret_cast<const float2 *>(p.ref) + nq);
                lx = __fadd_rn(r.x, __fdiv_rn(o.x, (float)sW[l]));
                ly = __fadd_rn(r.y, __fdiv_rn(o.y, (float)sH[l]));
            } else {
                // box reference (cx, cy, w, h): offsets are in box units
                const float2 c = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq);
                const float2 s2 = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
                lx = __fadd_rn(c.x, __fmul_rn(o.x, s2.x));
                ly = __fadd_rn(c.y, __fmul_rn(o.y, s2.y));
            }
            if (p.loc_out)
                reinterpret_cast<float2 *>(p.loc_out)[sbase + lane] = make_float2(lx, ly);
            if (p.attn_out) p.attn_out[sbase + lane] = a;
        }
    } else {
        if (act) {
            const float2 t = __ldg(reinterpret_cast<const float2 *>(p.loc) + sbase + lane);
            lx = t.x;
            ly = t.y;
            a = __ldg(p.attn + sbase + lane);
        }
    }
    if (act) {
        const int H = sH[l], W = sW[l], start = sStart[l];
        Corner c[4] = {{-1, 0.f}, {-1, 0.f}, {-1, 0.f}, {-1, 0.f}};
        float x, y, fx, fy;
        int x0, y0;
        if (msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
            const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
            const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
            const int MD = M * D;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = msda_row(start, H, W, y0 + (j >> 1), x0 + (j & 1));
                c[j].off = r < 0 ? -1 : r * MD;
                c[j].w = w[j] * a;
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) corners[warp][lane * 4 + j] = c[j];
    }
    __syncwarp();

    // ---- phase 2: gather the corner rows ---------------------------------
    const int slot = lane / R;
    const int chunk = lane % R;
    const bool chunk_ok = chunk < p.nchunks;
    const VT *vbase = static_cast<const VT *>(p.value) + (n * p.S * M + m) * (int64_t)D +
                      chunk * kVec;
    float acc[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) acc[i] = 0.f;
    const int npairs = 4 * LK;
#pragma unroll 4
    for (int t = slot; t < npairs; t += kSlots) {
        const Corner e = corners[warp][t];
        if (e.off >= 0 && chunk_ok) {
            float v[kVec];
            Chunk<VT>::load(vbase + e.off, v);
#pragma unroll
            for (int i = 0; i < kVec; ++i) acc[i] = fmaf(e.w, v[i], acc[i]);
        }
    }

    // ---- phase 3: combine the slots, store the head's output --------------
#pragma unroll
    for (int o = R; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < kVec; ++i) acc[i] += __shfl_xor_sync(kFull, acc[i], o);
    if (slot == 0 && chunk_ok) {
        float4 *dst = reinterpret_cast<float4 *>(p.out + nq * (int64_t)(M * D) + m * D +
                                                 chunk * kVec);
#pragma unroll
        for (int i = 0; i < kVec / 4; ++i)
            dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    }
}

template <typename VT, bool kFused>
cudaError_t launch_fwd_vt(const FwdParams &p, int R, cudaStream_t stream)
{
    const dim3 block(kWarps * 32);
    const dim3 grid((unsigned)((p.items + kWarps - 1) / kWarps));
    switch (R) {
    case 1: fwd_kernel<VT, 1, kFused><<<grid, block, 0, stream>>>(p); break;
    case 2: fwd_kernel<VT, 2, kFused><<<grid, block, 0, stream>>>(p); break;
    case 4: fwd_kernel<VT, 4, kFused><<<grid, block, 0, stream>>>(p); break;
    case 8: fwd_kernel<VT, 8, kFused><<<grid, block, 0, stream>>>(p); break;
    case 16: fwd_kernel<VT, 16, kFused><<<grid, block, 0, stream>>>(p); break;
    case 32: fwd_kernel<VT, 32, kFused><<<grid, block, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
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
