// msda_bwd_tiled.cu -- the tiled backward kernel (sm_100a): the gradients of
// bwd_kernel, scheduled cell by cell, with the value windows in shared memory
// and each window row's value gradient summed on the chip.
//
// Gradients flow through the bilinear interpolation to the value map, the
// sampling locations and the attention weights ("Deformable DETR" wiki page,
// "Deformable attention module"; "Deformable Attention" glossary page: the
// interpolation passes gradients on).  Per sample, with g = grad_out[n,q,m,:],
// corner weights w_j(fx, fy) and t_j = <v_j, g>:
//   dA = sum_j w_j t_j,  dloc = A * (W, H) * sum_j (dw_j/dfx, dw_j/dfy) t_j,
//   dvalue_j += A w_j g.
// The queries of one cell of the tile plan sample overlapping windows of
// every level, so most of their corners fall on a few hundred pixels per
// level.  A work unit is one (batch entry n, cell c, head m); its queries are
// taken in chunks of up to T:
//   1. one thread copies the head's value window of every level into shared
//      memory (tensor copies on an mbarrier, once per unit; pixels outside
//      the level read zero); the chunk's grad_out rows are loaded beside them;
//   2. phase A: the warps sweep the chunk's queries as bwd_kernel does (lane
//      j of an item's segment forms sample j's weight, location, cell and
//      corner entries; R lanes per row form <v_j, g> and reduce it in two
//      stages) and write dA and dloc.  A sample whose four corners lie in its
//      level's window reads them from shared memory and leaves a record
//      (window pixel of its first corner, query, A, fx, fy), counted per
//      pixel; any other sample reads global memory and adds A w_j g to
//      grad_value directly, as bwd_kernel does;
//   3. a counting sort orders the contributions A w_j g by target pixel:
//      phase A counted one per corner inside its level; after a prefix sum of
//      the counts, one pass places a (query, A w_j) entry per corner, in the
//      shared memory of the windows, which the chunk no longer reads;
//   4. phase B: R lanes take one window pixel, walk its run of entries, sum
//      A w_j g in registers and add the row to grad_value with one vector
//      reduction per 16 bytes.  Each touched pixel is reduced into L2 once
//      per chunk instead of once per (sample, corner).  The next chunk (of
//      the same cell, or of the next one) copies the windows in again.
// No shared-memory atomics touch floating point: the only shared atomics
// are the integer counts and placements of the sort.
#include "msda_common.cuh"
#include "msda_internal.h"
#include "msda_rows.cuh"
#include "msda_tile.cuh"
#include "msda_tma.cuh"

namespace msda {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;

// Exclusive prefix sum over a[0, n) by the whole CTA, with a[n] = the total.
// Every thread must call it; it ends with a CTA barrier.
__device__ void cta_exclusive_scan(int *a, int n, int *warp_tot)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kThreads - 1) / kThreads;
    const int c0 = min(tid * per, n), c1 = min(c0 + per, n);
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += a[c];
    int v = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kWarps ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += t;
        }
        if (lane < kWarps) warp_tot[lane] = w;
    }
    __syncthreads();
    int run = v - sum + (warp > 0 ? warp_tot[warp - 1] : 0);
    for (int c = c0; c < c1; ++c) {
        const int k = a[c];
        a[c] = run;
        run += k;
    }
    if (tid == kThreads - 1) a[n] = run;
    __syncthreads();
}

template <typename VT, int R, int P, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tiled_kernel(const __grid_constant__ BwdTiledParams tp)
{
    static_assert(R <= 8, "at least four (sample, corner) pairs per warp instruction");
    const BwdParams &p = tp.b;
    const TileView &t = tp.t;
    constexpr int kVec = 4;  // value elements per lane
    using Raw = typename Lane4<VT>::Raw;
    constexpr int kSlots = 32 / R;
    constexpr int kSG = kSlots / 4;  // samples per warp instruction
    constexpr int kB = R;            // instructions per batch: one t per lane after stage A
    constexpr int kBS = kB * kSG;    // samples per batch (= 8)
    constexpr int kItems = 32 / P;
    constexpr int kStride = P + 2;
    static_assert(kBS <= P && P % kBS == 0, "a batch must stay inside the P sample slots");
    constexpr int kNB = P / kBS;
    __shared__ int2 ent[kWarps][kItems][4 * kStride];        // (row offset, A*w)
    __shared__ float4 smp[kWarps][kItems][P];                // (fx, fy, A*W, A*H)
    __shared__ float4 smq[kWarps][kItems][kFused ? P : 1];   // fused: (A, off_x, off_y, dA)
    __shared__ float2 sdl[kWarps][kItems][kFused ? P : 1];   // fused: d loc per sample
    __shared__ int warp_tot[kWarps];
    __shared__ __align__(8) uint64_t bar;
    extern __shared__ __align__(128) unsigned char dyn_raw[];
    unsigned char *const win = dyn_raw + ((128u - (smem_addr(dyn_raw) & 127u)) & 127u);
    float *const sgo = reinterpret_cast<float *>(win + tp.off_g);        // [T][D] grad_out rows
    int4 *const rec = reinterpret_cast<int4 *>(win + tp.off_rec);        // [T][L*K] records
    int *const kstart = reinterpret_cast<int *>(win + tp.off_start);     // [keys + 1]
    int *const kcur = reinterpret_cast<int *>(win + tp.off_cursor);      // [keys]
    int *const squeue = reinterpret_cast<int *>(win + tp.off_queue);     // [T] the chunk's queries

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int M = p.M, D = p.D, K = p.K;
    const int LK = p.L * K;
    const int MD = M * D;
    const int rowb = D * (int)sizeof(VT);

    // phase-1 role: sample j of the round's item `seg`
    const int seg = lane / P;
    const int j = lane % P;
    const bool jact = j < LK;
    const int lvl = jact ? j / K : 0;
    const int H = p.lv.H[lvl], W = p.lv.W[lvl], start = p.lv.start[lvl];
    const int ww = t.ww[lvl], wh = t.wh[lvl];
    const int soff = t.soff[lvl];
    const int kbase = tp.roff[lvl];

    // phase-2 role: chunk `chunk` of the rows of slot `slot` (corner slot & 3)
    const int slot = lane / R;
    const int chunk = lane % R;
    const int corner = slot & 3;
    const int sgi = slot >> 2;
    const bool chunk_ok = chunk < p.nchunks;
    const int lane_elem = (chunk_ok ? chunk : 0) * kVec;
    const bool cx = corner & 1, cy = corner >> 1;
    const unsigned char *wlane = win + lane_elem * (int)sizeof(VT);

    if (tid == 0) mbar_init(&bar, 1);
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
        const int ccy = c / t.gx, ccx = c - ccy * t.gx;
        const int wx0 = ww ? window_origin(ccx, t.gx, W, t.halo, ww) : 0;
        const int wy0 = ww ? window_origin(ccy, t.gy, H, t.halo, wh) : 0;
        const int64_t nbase = (int64_t)n * p.Lq;
        const int64_t mapoff = ((int64_t)n * p.S * M + m) * (int64_t)D;
        const int64_t vbe = mapoff + lane_elem;
        const VT *vb = static_cast<const VT *>(p.value) + vbe;
        float *gvb = p.grad_value + mapoff + chunk * kVec;
        const int *pl = t.perm + nbase;

        for (int cb = q0; cb < q1; cb += tp.T) {
            const int cnt = min(tp.T, q1 - cb);
            // the previous chunk is done with shared memory; its entries (written
            // through the generic proxy) are ordered before the tensor copies
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {  // every chunk: the previous chunk's entries overwrote the windows
                mbar_arrive_expect_tx(&bar, t.window_tx);
                for (int l = 0; l < p.L; ++l) {
                    if (t.ww[l] == 0) continue;
                    const int ox = window_origin(ccx, t.gx, p.lv.W[l], t.halo, t.ww[l]);
                    const int oy = window_origin(ccy, t.gy, p.lv.H[l], t.halo, t.wh[l]);
                    tma_load_5d(win + t.soff[l], &tp.maps[l], 0, m, ox, oy, (int)n, &bar);
                }
            }
            // the chunk's queries (clamped: a stale plan is slow, never out of
            // bounds) and grad_out rows, and zero pixel counts
            for (int i = tid / R; i < cnt; i += kThreads / R) {
                const int q = min(max(__ldg(pl + cb + i), 0), p.Lq - 1);
                if (chunk == 0) squeue[i] = q;
                if (!chunk_ok) continue;
                const float4 gq = __ldcs(reinterpret_cast<const float4 *>(
                    p.grad_out + (nbase + q) * MD + m * D + chunk * kVec));
                *reinterpret_cast<float4 *>(sgo + i * D + chunk * kVec) = gq;
            }
            for (int k = tid; k <= tp.keys; k += kThreads) kstart[k] = 0;
            {
                const bool ok = mbar_wait(&bar, parity);
                parity ^= 1u;
                if (__syncthreads_or(!ok)) {
                    // never expected: record it, give the copies a second bound, stop
                    if (tid == 0 && t.stall) atomicAdd(t.stall, 1u);
                    mbar_wait(&bar, parity ^ 1u);
                    return;
                }
            }

            // ---- phase A: dA, dloc; records of the in-window samples --------
            // this lane's sample inputs in the round starting at item i0:
            // (logit, off) fused, (attn, loc) unfused
            float pa = 0.f, pb = 0.f, pc = 0.f;
            auto fetch = [&](int i0) {
                const int ii = i0 + seg;
                pa = pb = pc = 0.f;
                if (jact && ii < cnt) {
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
            fetch(warp * kItems);
            for (int i0 = warp * kItems; i0 < cnt; i0 += kWarps * kItems) {
                const int ii = i0 + seg;
                const bool iact = ii < cnt;
                const bool act = jact && iact;
                const int q = iact ? squeue[ii] : 0;
                {
                    const int64_t nq = nbase + q;
                    float lx = 0.f, ly = 0.f, a = 0.f;
                    if constexpr (kFused) {
                        // the fused forward's softmax and location map, bit for bit
                        a = seg_softmax<P>(pa, act);
                        if (act) {
                            const float2 loc =
                                msda_fused_location(p.ref, p.ref_dim, nq, pb, pc, H, W);
                            lx = loc.x;
                            ly = loc.y;
                        }
                        smq[warp][seg][j] = make_float4(act ? a : 0.f, act ? pb : 0.f,
                                                        act ? pc : 0.f, 0.f);
                    } else if (act) {
                        lx = pb;
                        ly = pc;
                        a = pa;
                    }
                    fetch(i0 + kWarps * kItems);  // loads while this round gathers
                    int2 e[4] = {{-1, 0}, {-1, 0}, {-1, 0}, {-1, 0}};
                    float4 sr = make_float4(0.f, 0.f, 0.f, 0.f);
                    int4 pr = make_int4(-1, 0, 0, 0);
                    float x, y, fx, fy;
                    int x0, y0;
                    if (act && msda_cell(lx, ly, H, W, x, y, x0, y0, fx, fy)) {
                        const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                        const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
                        const int ux = x0 - wx0, uy = y0 - wy0;
                        if (ux >= 0 && ux <= ww - 2 && uy >= 0 && uy <= wh - 2) {
                            const int b = soff + (uy * ww + ux) * rowb;
                            const int step[4] = {0, rowb, ww * rowb, (ww + 1) * rowb};
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc)
                                e[cc] = make_int2(shared_entry(b + step[cc]),
                                                  __float_as_int(a * w[cc]));
                            const int key = kbase + uy * ww + ux;
                            pr = make_int4(key | (ii << 16), __float_as_int(a),
                                           __float_as_int(fx), __float_as_int(fy));
                            // one value-gradient contribution per corner inside the level
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) {
                                const int xx = x0 + (cc & 1), yy = y0 + (cc >> 1);
                                if (xx >= 0 && xx < W && yy >= 0 && yy < H)
                                    atomicAdd(&kstart[key + (cc >> 1) * ww + (cc & 1)], 1);
                            }
                        } else {
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) {
                                const int r = msda_row(start, H, W, y0 + (cc >> 1), x0 + (cc & 1));
                                if (r >= 0) e[cc] = make_int2(r * MD, __float_as_int(a * w[cc]));
                            }
                        }
                        sr = make_float4(fx, fy, a * (float)W, a * (float)H);
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) ent[warp][seg][cc * kStride + j] = e[cc];
                    smp[warp][seg][j] = sr;
                    if (iact && jact) rec[ii * LK + j] = pr;
                }
                __syncwarp();

#pragma unroll 1
                for (int it = 0; it < kItems; ++it) {
                    const int qi = __shfl_sync(kFull, q, it * P);
                    const int iti = i0 + it;
                    if (iti >= cnt) break;  // uniform
                    const int64_t nq = nbase + qi;
                    const int64_t sbase = (nq * M + m) * LK;
                    float gv[kVec];
                    if (chunk_ok) {
                        const float4 g4 = *reinterpret_cast<const float4 *>(sgo + iti * D +
                                                                            chunk * kVec);
                        gv[0] = g4.x;
                        gv[1] = g4.y;
                        gv[2] = g4.z;
                        gv[3] = g4.w;
                    } else {
#pragma unroll
                        for (int i = 0; i < kVec; ++i) gv[i] = 0.f;
                    }
                    const int2 *en = ent[warp][it] + corner * kStride + sgi;
                    float2 bwh = make_float2(0.f, 0.f);  // fused box reference: (w, h)
                    if constexpr (kFused) {
                        if (p.ref_dim == 4)
                            bwh = __ldg(reinterpret_cast<const float2 *>(p.ref) + 2 * nq + 1);
                    }
#pragma unroll
                    for (int bi = 0; bi < kNB; ++bi) {
                        const int s0 = bi * kBS;
                        if (s0 >= LK) break;  // uniform
                        int2 e[kB];
                        Raw raw[kB];
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            e[b] = en[s0 + b * kSG];  // sample s0 + b*kSG + sgi, this lane's corner
                            if (e[b].x <= -2) {
                                raw[b] = *reinterpret_cast<const Raw *>(wlane + (-2 - e[b].x));
                            } else if (e[b].x >= 0) {
                                // bounds-checked build: a skipped corner reads zeros, adds nothing
                                if (!msda_in_map(p.check, p.check_limit, vbe + e[b].x, kVec))
                                    e[b].x = -1;
                                else
                                    raw[b] = Lane4<VT>::load(vb + e[b].x);
                            }
                        }
                        float tt[kB];
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            tt[b] = 0.f;
                            if (e[b].x != -1) {
                                float v[kVec];
                                Lane4<VT>::widen(raw[b], v);
#pragma unroll
                                for (int i = 0; i < kVec; ++i) tt[b] = fmaf(v[i], gv[i], tt[b]);
                                if (e[b].x >= 0 && chunk_ok) {  // outside the window: direct
                                    const float aw = __int_as_float(e[b].y);
                                    red_add_v4(gvb + e[b].x, aw * gv[0], aw * gv[1], aw * gv[2],
                                               aw * gv[3]);
                                }
                            }
                        }
                        // stage A: sum t over the R chunk lanes; this lane keeps b = chunk
                        reduce_scatter_n<R, kB, kB>(tt, lane);
                        const int s = s0 + chunk * kSG + sgi;
                        const float4 sr = smp[warp][it][s < P ? s : 0];
                        const float fx = sr.x, fy = sr.y;
                        const float wxc = cx ? fx : __fsub_rn(1.f, fx);
                        const float wyc = cy ? fy : __fsub_rn(1.f, fy);
                        float g0 = (wyc * wxc) * tt[0];        // w t
                        float g1 = (cx ? wyc : -wyc) * tt[0];  // dw/dfx t
                        float g2 = (cy ? wxc : -wxc) * tt[0];  // dw/dfy t
                        // stage B: sum over the four corner lanes of the sample
#pragma unroll
                        for (int o = R; o < 4 * R; o <<= 1) {
                            g0 += __shfl_xor_sync(kFull, g0, o);
                            g1 += __shfl_xor_sync(kFull, g1, o);
                            g2 += __shfl_xor_sync(kFull, g2, o);
                        }
                        if (corner == 0 && s < LK) {
                            const int64_t si = sbase + s;
                            const float dlx = sr.z * g1, dly = sr.w * g2;  // d loc
                            if constexpr (!kFused) {
                                if (p.grad_attn) __stcs(p.grad_attn + si, g0);
                                if (p.grad_loc)
                                    __stcs(reinterpret_cast<float2 *>(p.grad_loc) + si,
                                           make_float2(dlx, dly));
                            } else {
                                const float4 r2 = smq[warp][it][s];  // (A, off_x, off_y, -)
                                float2 goff;
                                if (p.ref_dim == 2)  // d off = d loc / W_l = A * (sum dw t)
                                    goff = make_float2(r2.x * g1, r2.x * g2);
                                else  // loc = c + off * (w, h)
                                    goff = make_float2(dlx * bwh.x, dly * bwh.y);
                                if (p.grad_off)
                                    __stcs(reinterpret_cast<float2 *>(p.grad_off) + si, goff);
                                smq[warp][it][s].w = g0;                 // dA
                                sdl[warp][it][s] = make_float2(dlx, dly);  // d loc
                            }
                        }
                    }
                }
                if constexpr (kFused) {
                    // the item's segment sums, as bwd_kernel: softmax Jacobian
                    // d z_j = A_j (dA_j - sum_i A_i dA_i) and the reference point
                    __syncwarp();
                    const int64_t nq = nbase + q;
                    const int64_t item = nq * M + m;
                    const float4 ad = act ? smq[warp][seg][j] : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float2 dl = act ? sdl[warp][seg][j] : make_float2(0.f, 0.f);
                    const float dot = seg_sum<P>(ad.x * ad.w);
                    if (act && p.grad_logits)
                        __stcs(p.grad_logits + item * LK + j, ad.x * (ad.w - dot));
                    const float rx = seg_sum<P>(dl.x), ry = seg_sum<P>(dl.y);
                    float rw = 0.f, rh = 0.f;
                    if (p.ref_dim == 4) {
                        rw = seg_sum<P>(dl.x * ad.y);
                        rh = seg_sum<P>(dl.y * ad.z);
                    }
                    if (j == 0 && iact && p.grad_ref) {
                        float *gr = p.grad_ref + nq * p.ref_dim;
                        atomicAdd(gr, rx);
                        atomicAdd(gr + 1, ry);
                        if (p.ref_dim == 4) {
                            atomicAdd(gr + 2, rw);
                            atomicAdd(gr + 3, rh);
                        }
                    }
                }
                __syncwarp();  // the next round overwrites this warp's entries
            }
            __syncthreads();

            // ---- counting sort of the contributions by window pixel --------
            // Each in-window sample adds A w_j g to the pixel of each corner j
            // inside its level.  The windows are no longer read in this chunk,
            // so the sorted (query, A w_j) entries take their place.
            cta_exclusive_scan(kstart, tp.keys, warp_tot);
            for (int k = tid; k < tp.keys; k += kThreads) kcur[k] = kstart[k];
            __syncthreads();
            int2 *const cent = reinterpret_cast<int2 *>(win);
            for (int r = tid; r < cnt * LK; r += kThreads) {
                const int4 rr = rec[r];
                if (rr.x < 0) continue;
                const int key = rr.x & 0xffff, ii = rr.x >> 16;
                int l = 0;
                while (l + 1 < p.L && key >= tp.roff[l + 1]) ++l;
                const int wwl = t.ww[l];
                const int loc = key - tp.roff[l];
                const int uy = loc / wwl, ux = loc - uy * wwl;
                const int x0 = window_origin(ccx, t.gx, p.lv.W[l], t.halo, wwl) + ux;
                const int y0 = window_origin(ccy, t.gy, p.lv.H[l], t.halo, t.wh[l]) + uy;
                const float a = __int_as_float(rr.y);
                const float fx = __int_as_float(rr.z), fy = __int_as_float(rr.w);
                const float hx = __fsub_rn(1.f, fx), hy = __fsub_rn(1.f, fy);
                const float w[4] = {hy * hx, hy * fx, fy * hx, fy * fx};
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int xx = x0 + (cc & 1), yy = y0 + (cc >> 1);
                    if (xx < 0 || xx >= p.lv.W[l] || yy < 0 || yy >= p.lv.H[l]) continue;
                    const int pos = atomicAdd(&kcur[key + (cc >> 1) * wwl + (cc & 1)], 1);
                    cent[pos] = make_int2(ii, __float_as_int(a * w[cc]));
                }
            }
            __syncthreads();

            // ---- phase B: one vector reduction per touched window pixel ----
            for (int pix = tid / R; pix < tp.keys; pix += kThreads / R) {
                const int r0 = kstart[pix], r1 = kstart[pix + 1];
                if (r0 == r1 || !chunk_ok) continue;
                float acc[kVec] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int idx = r0; idx < r1; ++idx) {
                    const int2 e = cent[idx];
                    const float coef = __int_as_float(e.y);
                    const float4 g4 =
                        *reinterpret_cast<const float4 *>(sgo + e.x * D + lane_elem);
                    acc[0] = fmaf(coef, g4.x, acc[0]);
                    acc[1] = fmaf(coef, g4.y, acc[1]);
                    acc[2] = fmaf(coef, g4.z, acc[2]);
                    acc[3] = fmaf(coef, g4.w, acc[3]);
                }
                int l = 0;
                while (l + 1 < p.L && pix >= tp.roff[l + 1]) ++l;
                const int wwl = t.ww[l], Wl = p.lv.W[l];
                const int loc = pix - tp.roff[l];
                const int py = loc / wwl, px = loc - py * wwl;
                const int gx = window_origin(ccx, t.gx, Wl, t.halo, wwl) + px;
                const int gy = window_origin(ccy, t.gy, p.lv.H[l], t.halo, t.wh[l]) + py;
                // gx, gy lie inside the level: only corners inside it were placed
                const int64_t off = (int64_t)(p.lv.start[l] + gy * Wl + gx) * MD;
                if (!msda_in_map(p.check, p.check_limit, mapoff + off + chunk * kVec, kVec))
                    continue;  // bounds-checked build: dropped and reported
                red_add_v4(gvb + off, acc[0], acc[1], acc[2], acc[3]);
            }
        }
    }
    __syncthreads();
    if (tid == 0) mbar_inval(&bar);
}

template <typename VT, int R, int P, bool kFused>
cudaError_t launch_p(const BwdTiledParams &p, int dyn_smem, cudaStream_t s)
{
    auto kern = bwd_tiled_kernel<VT, R, P, kFused>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dyn_smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t ctas = sms;
    if (ctas > p.t.units) ctas = p.t.units;
    if (ctas < 1) ctas = 1;
    kern<<<(unsigned)ctas, kThreads, dyn_smem, s>>>(p);
    return cudaGetLastError();
}

template <typename VT, int R, bool kFused>
cudaError_t launch_r(const BwdTiledParams &p, int smem, cudaStream_t s)
{
    const int LK = p.b.L * p.b.K;
    if (LK <= 8) return launch_p<VT, R, 8, kFused>(p, smem, s);
    if (LK <= 16) return launch_p<VT, R, 16, kFused>(p, smem, s);
    return launch_p<VT, R, 32, kFused>(p, smem, s);
}

template <typename VT, bool kFused>
cudaError_t launch_vt(BwdTiledParams p, int smem, cudaStream_t s)
{
    // four elements per lane: R = D/4 lanes cover a row of the fp32 gradient
    const int lanes = p.b.D / 4;
    p.b.nchunks = lanes;
    if (lanes <= 1) return launch_r<VT, 1, kFused>(p, smem, s);
    if (lanes <= 2) return launch_r<VT, 2, kFused>(p, smem, s);
    if (lanes <= 4) return launch_r<VT, 4, kFused>(p, smem, s);
    return launch_r<VT, 8, kFused>(p, smem, s);
}

// Static shared memory of the kernel that a launch of these dims takes.
template <typename VT, bool kFused>
int static_smem_vt(int D, int LK)
{
    auto pick = [&](auto kern) {
        cudaFuncAttributes a;
        return cudaFuncGetAttributes(&a, kern) == cudaSuccess ? (int)a.sharedSizeBytes : -1;
    };
    const int lanes = D / 4;
    const int R = lanes <= 1 ? 1 : lanes <= 2 ? 2 : lanes <= 4 ? 4 : 8;
    const int P = LK <= 8 ? 8 : LK <= 16 ? 16 : 32;
#define MSDA_PICK(RR)                                                                  \
    if (R == RR) {                                                                     \
        if (P == 8) return pick(bwd_tiled_kernel<VT, RR, 8, kFused>);                  \
        if (P == 16) return pick(bwd_tiled_kernel<VT, RR, 16, kFused>);                \
        return pick(bwd_tiled_kernel<VT, RR, 32, kFused>);                             \
    }
    MSDA_PICK(1)
    MSDA_PICK(2)
    MSDA_PICK(4)
    MSDA_PICK(8)
#undef MSDA_PICK
    return -1;
}

}  // namespace

int backward_tiled_static_smem(bool bf16, bool fused, int D, int LK)
{
    if (bf16)
        return fused ? static_smem_vt<__nv_bfloat16, true>(D, LK)
                     : static_smem_vt<__nv_bfloat16, false>(D, LK);
    return fused ? static_smem_vt<float, true>(D, LK) : static_smem_vt<float, false>(D, LK);
}

cudaError_t launch_backward_tiled(const BwdTiledParams &p, bool bf16, bool fused, int dyn_smem,
                                  cudaStream_t stream)
{
    if (p.b.items == 0) return cudaSuccess;
    if (bf16)
        return fused ? launch_vt<__nv_bfloat16, true>(p, dyn_smem, stream)
                     : launch_vt<__nv_bfloat16, false>(p, dyn_smem, stream);
    return fused ? launch_vt<float, true>(p, dyn_smem, stream)
                 : launch_vt<float, false>(p, dyn_smem, stream);
}

}  // namespace msda
