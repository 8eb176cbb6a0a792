// msda_types.h -- plain types shared by host and device code.
#pragma once

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

}  // namespace msda
