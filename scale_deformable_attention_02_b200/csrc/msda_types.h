// msda_types.h -- plain types shared by host and device code.
#pragma once

namespace msda {

constexpr int kMaxLK = 32;      // samples per (query, head): one per lane
constexpr int kMaxLevels = 32;  // L <= L*K <= 32

// Per-level metadata, copied by value into every launch.
struct Levels {
    int H[kMaxLevels];
    int W[kMaxLevels];
    int start[kMaxLevels];  // first value row of the level
};

}  // namespace msda
