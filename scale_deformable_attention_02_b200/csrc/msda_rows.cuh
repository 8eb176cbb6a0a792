// msda_rows.cuh -- per-lane value-row loads, the output-row store and the
// lane reductions shared by the forward kernels (msda_fwd.cu,
// msda_fwd_tiled.cu) and the backward kernels (msda_bwd.cu,
// msda_bwd_tiled.cu).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "msda_common.cuh"

namespace msda {

// EPL consecutive value elements of one lane (32, 16 or 8 bytes), widened to
// float pairs when consumed.
template <typename VT, int EPL>
struct LaneLoad;

template <>
struct LaneLoad<float, 4> {
    using Raw = uint4;
    __device__ __forceinline__ static Raw load(const float *p)
    {
        return __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ static void widen(const Raw &r, float2 (&v)[2])
    {
        v[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
        v[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
    }
};

// Eight fp32 elements (32 bytes) of one lane with one 256-bit load (sm_100).
// The address must be 32-byte aligned: the launcher takes these lanes only
// for rows of 32 elements (128 bytes) in a value map whose base is 32-byte
// aligned.
struct Raw8 {
    uint32_t w[8];
};

template <>
struct LaneLoad<float, 8> {
    using Raw = Raw8;
    __device__ __forceinline__ static Raw load(const float *p)
    {
        Raw r;
        asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                       "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
                     : "l"(p));
        return r;
    }
    __device__ __forceinline__ static void widen(const Raw &r, float2 (&v)[4])
    {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = make_float2(__uint_as_float(r.w[2 * i]), __uint_as_float(r.w[2 * i + 1]));
    }
};

template <>
struct LaneLoad<__nv_bfloat16, 8> {
    using Raw = uint4;
    __device__ __forceinline__ static Raw load(const __nv_bfloat16 *p)
    {
        return __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ static void widen(const Raw &r, float2 (&v)[4])
    {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)  // exact widening: bf16 bits become the high half
            v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    }
};

template <>
struct LaneLoad<__nv_bfloat16, 4> {
    using Raw = uint2;
    __device__ __forceinline__ static Raw load(const __nv_bfloat16 *p)
    {
        return __ldg(reinterpret_cast<const uint2 *>(p));
    }
    __device__ __forceinline__ static void widen(const Raw &r, float2 (&v)[2])
    {
        v[0] = make_float2(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u));
        v[1] = make_float2(__uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
    }
};

// Sums each chunk's accumulators over the 32/R slot lanes that hold it and
// stores the item's output row (evict-first).  Where the lanes hold 32
// elements in all (R * EPL == 32) this is a butterfly reduce-scatter: at xor
// distance o a lane keeps one half of its values (the upper half if bit o of
// its lane is set) and adds the partner's copy of that half, so after
// log2(32/R) steps it holds one finished element, idx, of its chunk, and the
// warp stores the row with one coalesced instruction (3 shuffles for
// 4-element lanes, 7 for 8, against 8 and 24 for a full xor reduction).
// Other widths take the full xor reduction, and the slot-0 lanes store.
template <int R, int EPL>
__device__ __forceinline__ void store_row(float2 (&acc)[EPL / 2], int lane, int chunk,
                                          bool chunk_ok, float *row)
{
    constexpr int kNP = EPL / 2;
    if constexpr (R * EPL == 32) {
        float v[EPL];
#pragma unroll
        for (int i = 0; i < kNP; ++i) {
            v[2 * i] = acc[i].x;
            v[2 * i + 1] = acc[i].y;
        }
        int idx = 0;
#pragma unroll
        for (int o = 16, n = EPL; o >= R; o >>= 1, n >>= 1) {
            const int half = n / 2;
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = up ? v[i] : v[i + half];
                const float keep = up ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(kFull, send, o);
            }
            if (up) idx += half;
        }
        if (chunk_ok) __stcs(row + chunk * EPL + idx, v[0]);
    } else {
#pragma unroll
        for (int o = R; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < kNP; ++i) {
                acc[i].x += __shfl_xor_sync(kFull, acc[i].x, o);
                acc[i].y += __shfl_xor_sync(kFull, acc[i].y, o);
            }
        if (lane < R && chunk_ok) {  // slot 0
            float4 *dst = reinterpret_cast<float4 *>(row + chunk * EPL);
#pragma unroll
            for (int i = 0; i < kNP / 2; ++i)
                __stcs(dst + i, make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x,
                                            acc[2 * i + 1].y));
        }
    }
}

// Four consecutive value elements of one lane, widened to fp32: a 16-byte
// load for fp32, an 8-byte load for bf16.  The backward's fast path gives
// every lane four elements so that R = D/4 lanes cover a row of the fp32
// gradient and one vector reduction instruction updates whole 128-byte
// gradient rows, whatever the value dtype.
template <typename VT>
struct Lane4;

template <>
struct Lane4<float> {
    using Raw = uint4;
    __device__ __forceinline__ static Raw load(const float *p)
    {
        return __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ static void widen(const Raw &r, float (&v)[4])
    {
        v[0] = __uint_as_float(r.x);
        v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z);
        v[3] = __uint_as_float(r.w);
    }
};

template <>
struct Lane4<__nv_bfloat16> {
    using Raw = uint2;
    __device__ __forceinline__ static Raw load(const __nv_bfloat16 *p)
    {
        return __ldg(reinterpret_cast<const uint2 *>(p));
    }
    __device__ __forceinline__ static void widen(const Raw &r, float (&v)[4])
    {
        v[0] = __uint_as_float(r.x << 16);
        v[1] = __uint_as_float(r.x & 0xffff0000u);
        v[2] = __uint_as_float(r.y << 16);
        v[3] = __uint_as_float(r.y & 0xffff0000u);
    }
};

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

}  // namespace msda
