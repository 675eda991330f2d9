// mxq_grids.h -- the 8-bit block-scale grids, decoded from their bit fields (host side).
//
//  E4M3  (FN) 4 exponent bits, bias 7, 3 mantissa bits; codes 0..126 (127 is NaN)
//  UE4M4 unsigned, 4 exponent bits, bias 7, 4 mantissa bits; codes 0..255, all finite
//  UE5M3 unsigned, 5 exponent bits, bias 15, 3 mantissa bits; codes 0..255, all finite
//  UE8M0 2^(code - 127), codes 0..254 (255 is NaN)
// (qwantize "Results", sections "MXFP4 (UE8M0 power-of-2 scales)" and "Exotic Scales";
// "Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1.)
#pragma once

#include <cmath>

namespace mxq {

enum ScaleFmt { kScaleE4M3 = 0, kScaleUE4M4 = 1, kScaleUE5M3 = 2, kScaleUE8M0 = 3 };

struct GridInfo {
  int ncodes;  // codes 0 .. ncodes - 1 are finite
  int first;   // the first candidate code of a search (the grids with a zero skip it)
};

inline bool grid_known(int sfmt) { return sfmt >= kScaleE4M3 && sfmt <= kScaleUE8M0; }

inline GridInfo grid_info(int sfmt) {
  switch (sfmt) {
    case kScaleUE4M4: return {256, 1};
    case kScaleUE5M3: return {256, 1};
    case kScaleUE8M0: return {255, 0};
    default: return {127, 1};
  }
}

// Exact value of a finite code (every value is a float32 and a double).
inline double grid_value(int sfmt, int code) {
  switch (sfmt) {
    case kScaleUE4M4: {
      const int e = (code >> 4) & 15, m = code & 15;
      return e == 0 ? std::ldexp(m / 16.0, -6) : std::ldexp(1.0 + m / 16.0, e - 7);
    }
    case kScaleUE5M3: {
      const int e = (code >> 3) & 31, m = code & 7;
      return e == 0 ? std::ldexp(m / 8.0, -14) : std::ldexp(1.0 + m / 8.0, e - 15);
    }
    case kScaleUE8M0:
      return std::ldexp(1.0, code - 127);
    default: {
      const int e = (code >> 3) & 15, m = code & 7;
      return e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
    }
  }
}

// True when s is a positive value of the grid.
inline bool grid_has_value(int sfmt, float s) {
  const GridInfo g = grid_info(sfmt);
  for (int c = 1; c < g.ncodes; ++c)
    if (grid_value(sfmt, c) == (double)s) return true;
  return sfmt == kScaleUE8M0 && (double)s == grid_value(sfmt, 0);
}

}  // namespace mxq
