// msda_fwd_tiled.cu -- the tiled forward kernel (sm_100a): the same result as
// fwd_kernel, scheduled cell by cell with the value windows in shared memory.
//
// Per batch entry n, query q and head m ("Deformable DETR" wiki page,
// "Multi-scale deformable attention" equation):
//   out[n,q,m,:] = sum_{l,k} A[n,q,m,l,k] * bilinear(value[n, level l, m, :], loc)
// Each query samples around its own reference point on every level, so the
// queries of one cell of the tile plan read overlapping parts of each level
// ("Limitations": the method's cost is unordered memory access).  A work
// unit is one (batch entry n, cell c, head m):
//   * one thread arms an mbarrier and issues one tensor copy per level: the
//     head's window of the value map around the cell (the cell's pixels plus
//     the halo and one corner on every side) lands in shared memory, and
//     pixels outside the level read as zero, which is the zero padding of
//     the method;
//   * the warps then sweep the cell's queries in rounds, exactly as
//     fwd_kernel does (lane j of an item's P-lane segment forms sample j's
//     weight, location and cell; four corner entries per sample; the warp
//     gathers the entries' rows and reduces the slot sums), except that a
//     corner entry whose sample lies inside its level's window names a
//     shared-memory row, and only samples outside it read global memory;
//   * before the next unit's copies overwrite the windows, every warp has
//     passed a CTA barrier.
// Two or three CTAs share an SM, so one CTA's copies overlap another's
// gathers.  Each sample's arithmetic (softmax, location, cell, corner
// weights) is fwd_kernel's and an item's corner terms are summed in
// fwd_kernel's order; a window corner outside the level adds w * 0.
#include "msda_common.cuh"
#include "msda_internal.h"
#include "msda_rows.cuh"
#include "msda_tile.cuh"
#include "msda_tma.cuh"

namespace msda {
namespace {

constexpr int kWarps = 8;

constexpr int kQueueQ = 512;  // queries of a cell taken per chunk (their order in shared memory)


template <typename VT, int EPL, int R, int P, bool kFused, int kMinCtas>
__global__ void __launch_bounds__(kWarps * 32, kMinCtas)
    fwd_tiled_kernel(const __grid_constant__ FwdTiledParams tp)
{
    using LL = LaneLoad<VT, EPL>;
    using Raw = typename LL::Raw;
    const FwdParams &p = tp.f;
    const TileView &t = tp.t;
    constexpr int kSlots = 32 / R;   // (sample, corner) pairs per warp instruction
    constexpr int kItems = 32 / P;   // items per warp round
    constexpr int kNP = EPL / 2;
    __shared__ int4 srec[kWarps][kItems][P];  // one record per sample
    __shared__ int squeue[kQueueQ];           // the chunk's queries
    __shared__ __align__(8) uint64_t bar;
    extern __shared__ __align__(128) unsigned char win_raw[];
    // tensor copies land on 128-byte boundaries (the launch adds 128 bytes)
    unsigned char *const win = win_raw + ((128u - (smem_addr(win_raw) & 127u)) & 127u);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int rowb = D * (int)sizeof(VT);  // bytes of a window row

    // phase-1 role: sample j of the round's item `seg`; its level is fixed
    const int seg = lane / P;
    const int j = lane % P;
    const bool jact = j < LK;
    const int lvl = jact ? j / K : 0;
    const int H = p.lv.H[lvl], W = p.lv.W[lvl];
    const int ww = t.ww[lvl], wh = t.wh[lvl];
    const int soff = t.soff[lvl];

    // phase-2 role: 16-byte chunk `chunk` of the rows in slot `slot`
    const int slot = lane / R;
    const int chunk = lane % R;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_elem = (chunk_ok ? chunk : 0) * EPL;
    const unsigned char *wlane = win + lane_elem * (int)sizeof(VT);

    if (threadIdx.x == 0) mbar_init(&bar, 1);
    __syncthreads();

    uint32_t parity = 0;
    for (int u = blockIdx.x; u < t.units; u += gridDim.x) {
        const unsigned ncell = fastdiv(p.dM, (unsigned)u);
        const int m = u - (int)(ncell * (unsigned)M);
        const unsigned n = fastdiv(t.dG, ncell);
        const int c = (int)(ncell - n * (unsigned)t.G);
        const int *cs = t.cell_start + (int64_t)n * (t.G + 1);
        // plan entries are clamped into range: a stale plan is slow, never out of bounds
        const int q0 = min(max(__ldg(cs + c), 0), p.Lq);
        const int q1 = min(max(__ldg(cs + c + 1), q0), p.Lq);
        if (q1 == q0) continue;  // the same for every thread of the CTA
        const int cy = c / t.gx, cx = c - cy * t.gx;

        // this lane's level window (its origin; the extent test below)
        const int wx0 = ww ? window_origin(cx, t.gx, W, t.halo, ww) : 0;
        const int wy0 = ww ? window_origin(cy, t.gy, H, t.halo, wh) : 0;
        const int count = q1 - q0;
        const int *pl = t.perm + (int64_t)n * p.Lq + q0;
        const int64_t nbase = (int64_t)n * p.Lq;
        const int64_t vbe = ((int64_t)n * p.S * M + m) * (int64_t)D + lane_elem;
        const VT *vb = static_cast<const VT *>(p.value) + vbe;

        // this lane's sample inputs in the round starting at item i0 of the
        // chunk: (logit, off) fused, (attn, loc) unfused
        float pa = 0.f, pb = 0.f, pc = 0.f;
        auto fetch = [&](int i0, int ccount) {
            const int ii = i0 + seg;
            pa = pb = pc = 0.f;
            if (jact && ii < ccount) {
                const int64_t si = ((nbase + squeue[ii]) * M + m) * LK + j;
                if constexpr (kFused) {
                    pa = __ldcs(p.logits + si);
                    const float2 o = __ldcs(reinterpret_cast<const float2 *>(p.off) + si);
                    pb = o.x;
                    pc = o.y;
                } else {
                    const float2 tl = __ldcs(reinterpret_cast<const float2 *>(p.loc) + si);
                    pb = tl.x;
                    pc = tl.y;
                    pa = __ldcs(p.attn + si);
                }
            }
        };

        for (int cb = 0; cb < count; cb += kQueueQ) {
            const int ccount = min(kQueueQ, count - cb);
            const bool first = cb == 0;
            fence_proxy_async_smem();  // this thread's window reads before the next copies
            __syncthreads();  // every warp is done with the windows and the queue
            if (first && threadIdx.x == 0) {
                mbar_arrive_expect_tx(&bar, t.window_tx);
                for (int l = 0; l < p.L; ++l) {
                    if (t.ww[l] == 0) continue;
                    const int ox = window_origin(cx, t.gx, p.lv.W[l], t.halo, t.ww[l]);
                    const int oy = window_origin(cy, t.gy, p.lv.H[l], t.halo, t.wh[l]);
                    tma_load_5d(win + t.soff[l], &tp.maps[l], 0, m, ox, oy, (int)n, &bar);
                }
            }
            // the chunk's queries, clamped: a stale plan is slow, never out of bounds
            for (int i = threadIdx.x; i < ccount; i += kWarps * 32)
                squeue[i] = min(max(__ldg(pl + cb + i), 0), p.Lq - 1);
            __syncthreads();
            fetch(warp * kItems, ccount);  // in flight while the windows arrive
            if (first) {
                const bool ok = mbar_wait(&bar, parity);
                parity ^= 1u;
                if (__syncthreads_or(!ok)) {
                    // never expected: record it, give the copies a second bound, stop
                    if (threadIdx.x == 0 && t.stall) atomicAdd(t.stall, 1u);
                    mbar_wait(&bar, parity ^ 1u);
                    return;
                }
            }

        for (int i0 = warp * kItems; i0 < ccount; i0 += kWarps * kItems) {
            // ---- phase 1: sample j of item i0 + seg ------------------------
            const int ii = i0 + seg;
            const bool iact = ii < ccount;
            const bool act = jact && iact;
            const int q = iact ? squeue[ii] : 0;
            const int64_t nq = nbase + q;
            const int64_t item = nq * M + m;
            const int64_t si = item * LK + j;
            float lx = 0.f, ly = 0.f, a = 0.f;
            if constexpr (kFused) {
                a = seg_softmax<P>(pa, act);
                if (act) {
                    const float2 loc = msda_fused_location(p.ref, p.ref_dim, nq, pb, pc, H, W);
                    lx = loc.x;
                    ly = loc.y;
                    if (p.loc_out)
                        __stcs(reinterpret_cast<float2 *>(p.loc_out) + si, make_float2(lx, ly));
                    if (p.attn_out) __stcs(p.attn_out + si, a);
                }
            } else if (act) {
                lx = pb;
                ly = pc;
                a = pa;
            }
            fetch(i0 + kWarps * kItems, ccount);  // loads while this round gathers
            {
                // one record per sample: (window row offset and row step, or the
                // cell for a global read, or none; A; fx; fy)
                int4 rc = make_int4(-1, 0, 0, 0);
                float x, y, fx, fy;
                int x0, y0;
                if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                    const int ux = x0 - wx0, uy = y0 - wy0;
                    int code;
                    if (ux >= 0 && ux <= ww - 2 && uy >= 0 && uy <= wh - 2)
                        // all four corners in the window (corners outside the
                        // level read its zero fill)
                        code = window_record(soff + (uy * ww + ux) * rowb, ww * rowb);
                    else
                        code = global_record(x0, y0, W);
                    rc = make_int4(code, __float_as_int(a), __float_as_int(fx), __float_as_int(fy));
                }
                srec[warp][seg][j] = rc;
            }
            __syncwarp();

            // ---- phase 2: gather, item by item ----------------------------
            // slot s walks samples s, s + kSlots, ...; for each it reads the
            // sample's record once and its four corner rows (16 bytes a lane)
#pragma unroll 1
            for (int it = 0; it < kItems; ++it) {
                const int qi = __shfl_sync(kFull, q, it * P);
                if (i0 + it >= ccount) break;  // uniform
                float2 acc[kNP];
#pragma unroll
                for (int i = 0; i < kNP; ++i) acc[i] = make_float2(0.f, 0.f);
                const int4 *rs = srec[warp][it];
#pragma unroll 2
                for (int smp = slot; smp < LK; smp += kSlots) {
                    const int4 rc = rs[smp];
                    if (rc.x == -1) continue;
                    const float a = __int_as_float(rc.y);
                    const float fx = __int_as_float(rc.z), fy = __int_as_float(rc.w);
                    const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                    const float w[4] = {(hy * hx) * a, (hy * fx) * a, (fy * hx) * a, (fy * fx) * a};
                    Raw raw[4];
                    bool has[4] = {true, true, true, true};
                    if (rc.x >= 0) {
                        const unsigned char *pb = wlane + (rc.x & kRecOffMask);
                        const int step = (rc.x >> kRecOffBits) << 4;
                        raw[0] = *reinterpret_cast<const Raw *>(pb);
                        raw[1] = *reinterpret_cast<const Raw *>(pb + rowb);
                        raw[2] = *reinterpret_cast<const Raw *>(pb + step);
                        raw[3] = *reinterpret_cast<const Raw *>(pb + step + rowb);
                    } else {
                        // outside the window: this sample's level, its cell, global rows
                        const int l = smp / K;
                        const int Hl = p.lv.H[l], Wl = p.lv.W[l];
                        const int cell = -2 - rc.x;
                        const int cy0 = cell / (Wl + 1) - 1, cx0 = cell % (Wl + 1) - 1;
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const int r = msda_row(p.lv.start[l], Hl, Wl, cy0 + (cc >> 1),
                                                   cx0 + (cc & 1));
                            has[cc] = r >= 0 && msda_in_map(p.check, p.check_limit,
                                                            vbe + (int64_t)r * MD, EPL);
                            if (has[cc]) raw[cc] = LL::load(vb + (int64_t)r * MD);
                        }
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        if (!has[cc]) continue;
                        float2 v[kNP];
                        LL::widen(raw[cc], v);
                        const float2 w2 = make_float2(w[cc], w[cc]);
#pragma unroll
                        for (int i = 0; i < kNP; ++i) acc[i] = __ffma2_rn(w2, v[i], acc[i]);
                    }
                }
                store_row<R, EPL>(acc, lane, chunk, chunk_ok,
                                  p.out + (nbase + qi) * (int64_t)MD + m * D);
            }
            __syncwarp();  // the next round overwrites this warp's entries
        }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_inval(&bar);
}

template <typename VT, int EPL, int R, int P, bool kFused>
cudaError_t launch_p(const FwdTiledParams &p, int ctas_per_sm, int dyn_smem, cudaStream_t s)
{
    auto go = [&](auto kern) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             dyn_smem);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        int64_t ctas = (int64_t)sms * ctas_per_sm;
        if (ctas > p.t.units) ctas = p.t.units;
        if (ctas < 1) ctas = 1;
        kern<<<(unsigned)ctas, kWarps * 32, dyn_smem, s>>>(p);
        return cudaGetLastError();
    };
    if (ctas_per_sm >= 3) return go(fwd_tiled_kernel<VT, EPL, R, P, kFused, 3>);
    if (ctas_per_sm == 2) return go(fwd_tiled_kernel<VT, EPL, R, P, kFused, 2>);
    return go(fwd_tiled_kernel<VT, EPL, R, P, kFused, 1>);
}

template <typename VT, int EPL, int R, bool kFused>
cudaError_t launch_r(const FwdTiledParams &p, int cps, int smem, cudaStream_t s)
{
    const int LK = p.f.L * p.f.K;
    if (LK <= 8) return launch_p<VT, EPL, R, 8, kFused>(p, cps, smem, s);
    if (LK <= 16) return launch_p<VT, EPL, R, 16, kFused>(p, cps, smem, s);
    return launch_p<VT, EPL, R, 32, kFused>(p, cps, smem, s);
}

// Lanes per row as fwd_kernel takes them: 16-byte lanes for bf16 rows of 32
// elements, else four-element lanes (rows of at most eight of them).
template <typename VT, bool kFused>
cudaError_t launch_vt(FwdTiledParams p, int cps, int smem, cudaStream_t s)
{
    constexpr int E16 = 16 / (int)sizeof(VT);
    const int D = p.f.D;
    if (E16 == 8 && D == 32) {
        p.f.nchunks = 4;
        return launch_r<VT, E16, 4, kFused>(p, cps, smem, s);
    }
    if (D % 4 == 0 && D / 4 <= 8) {
        const int lanes = D / 4;
        p.f.nchunks = lanes;
        if (lanes <= 1) return launch_r<VT, 4, 1, kFused>(p, cps, smem, s);
        if (lanes <= 2) return launch_r<VT, 4, 2, kFused>(p, cps, smem, s);
        if (lanes <= 4) return launch_r<VT, 4, 4, kFused>(p, cps, smem, s);
        return launch_r<VT, 4, 8, kFused>(p, cps, smem, s);
    }
    if constexpr (E16 == 8) {  // bf16 rows of 16-byte lanes (D = 40, 48, 56, 64)
        const int lanes = D / E16;
        p.f.nchunks = lanes;
        return launch_r<VT, E16, 8, kFused>(p, cps, smem, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_forward_tiled(const FwdTiledParams &p, bool bf16, bool fused,
                                 int ctas_per_sm, int dyn_smem, cudaStream_t stream)
{
    if (p.f.items == 0) return cudaSuccess;
    if (bf16)
        return fused ? launch_vt<__nv_bfloat16, true>(p, ctas_per_sm, dyn_smem, stream)
                     : launch_vt<__nv_bfloat16, false>(p, ctas_per_sm, dyn_smem, stream);
    return fused ? launch_vt<float, true>(p, ctas_per_sm, dyn_smem, stream)
                 : launch_vt<float, false>(p, ctas_per_sm, dyn_smem, stream);
}

}  // namespace msda
