// msda_types.h -- plain types shared by host and device code.
#pragma once

#if defined(__CUDACC__)
#define MSDA_HD __host__ __device__
#else
#define MSDA_HD
#endif

namespace msda {

constexpr int kMaxLK = 128;     // samples per (query, head): up to four per lane
constexpr int kLaneLK = 32;     // items of up to 32 samples: one sample per lane
constexpr int kMaxLevels = 32;  // L <= 32

// Per-level metadata, copied by value into every launch.
struct Levels {
    int H[kMaxLevels];
    int W[kMaxLevels];
    int start[kMaxLevels];  // first value row of the level
};

// Unsigned 32-bit division by a divisor d >= 1 that is fixed for a launch,
// as one multiply-high, a subtract, an add and two shifts.  The method is
// Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication" (PLDI 1994), section 4, Figure 4.1, with N = 32:
//   l  = ceil(log2 d)                 (so 2^(l-1) < d <= 2^l)
//   m' = floor(2^32 (2^l - d) / d) + 1, which fits in 32 bits
//   t  = floor(m' n / 2^32)
//   n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0)   for every n < 2^32.
// The host rejects problems of 2^31 or more items (n, q, m), so 32 bits hold
// every dividend.
struct FastDiv {
    unsigned d;   // the divisor
    unsigned m;   // m'
    int s1, s2;   // min(l, 1), max(l - 1, 0)
};

inline FastDiv make_fastdiv(unsigned d)
{
    int l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    const unsigned long long m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
    FastDiv f;
    f.d = d;
    f.m = (unsigned)m;
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

MSDA_HD inline unsigned fastdiv(const FastDiv &f, unsigned n)
{
#if defined(__CUDA_ARCH__)
    const unsigned t = __umulhi(f.m, n);
#else
    const unsigned t = (unsigned)(((unsigned long long)f.m * n) >> 32);
#endif
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

}  // namespace msda
