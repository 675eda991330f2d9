// mxq_gridk.cuh -- device-side scale-grid tables and the element steps shared by the
// grid searches (mxq_quant_grid.cu) and the GPTQ sweep (mxq_gptq_full.cu).
#pragma once

#include "mxq_common.cuh"
#include "mxq_grids.h"

#include <cuda_runtime.h>

namespace mxq {

enum { kElemE2M1 = 0, kElemInt4 = 1 };

// Per code: {s, r_hi, r_lo, 0} with r_hi + r_lo = 1/s to ~2^-48 (zero scale: all 0).
struct GridTable {
  float4 c[256];
  int ncodes, first, sfmt;
};

__device__ __forceinline__ float2 quot2(float2 a, float4 t) {
  return __ffma2_rn(a, make_float2(t.y, t.y), __fmul2_rn(a, make_float2(t.z, t.z)));
}

// Grid values g (as floats) of the element codes of two non-negative quotients.
template <int ELEM>
__device__ __forceinline__ float2 elem_values(float2 x) {
  if constexpr (ELEM == kElemE2M1) {
    float v0, v1;
    asm("{\n\t.reg .b8 q;\n\t.reg .b32 v;\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %3, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 v, q;\n\t"
        "mov.b32 {h0, h1}, v;\n\t"
        "cvt.f32.f16 %0, h0;\n\t"
        "cvt.f32.f16 %1, h1;\n\t}"
        : "=f"(v0), "=f"(v1)
        : "f"(x.x), "f"(x.y));
    return make_float2(v0, v1);
  } else {
    // min(x, 7) rounded to an integer, ties to even: adding 2^23 leaves an integer for
    // 0 <= x < 2^23, subtracting it again is exact.
    const float2 m = make_float2(8388608.f, 8388608.f);
    const float2 t = __fadd2_rn(make_float2(fminf(x.x, 7.f), fminf(x.y, 7.f)), m);
    return __fadd2_rn(t, make_float2(-8388608.f, -8388608.f));
  }
}

// Index of the table value nearest to z >= 0 (values ascending from 0); equidistant values
// go to the even code; z at or above the last value saturates.
__device__ __forceinline__ int grid_nearest(const float4* tab, int n, float z) {
  if (!(z > 0.0f)) return 0;
  if (z >= tab[n - 1].x) return n - 1;
  int lo = 0, hi = n - 1;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tab[mid].x <= z) lo = mid;
    else hi = mid;
  }
  const double dlo = (double)z - (double)tab[lo].x, dhi = (double)tab[hi].x - (double)z;
  if (dlo < dhi) return lo;
  if (dhi < dlo) return hi;
  return (lo & 1) ? hi : lo;
}

// floor(log2 x) of a positive finite float (normal or subnormal), exactly.
__device__ __forceinline__ int floor_log2(float x) {
  const uint32_t b = __float_as_uint(x);
  const int e = (int)((b >> 23) & 0xffu);
  return e ? e - 127 : (31 - __clz((int)b)) - 149;
}

// The naive code: UE8M0 2^(floor(log2 amax) - 2) clamped to 0..254 (0 for amax = 0);
// otherwise the grid's nearest value to fl32(amax / qmax).
template <int ELEM>
__device__ __forceinline__ int naive_code(float amax, const float4* tab, int ncodes, int sfmt) {
  if (sfmt == kScaleUE8M0) {
    if (!(amax > 0.0f)) return 0;
    return min(max(floor_log2(amax) - 2 + 127, 0), 254);
  }
  const float z = __fdiv_rn(amax, ELEM == kElemE2M1 ? 6.0f : 7.0f);
  if (sfmt == kScaleE4M3) return e4m3_rn_code(z);
  return grid_nearest(tab, ncodes, z);
}

// Candidate range of the definition: every candidate code, or a window of codes around
// the naive code c0 ([1, max(w, 1)] when c0 is a zero scale).
__device__ __forceinline__ void grid_window(const float4* tab, int ncodes, int first, int c0,
                                            int window, int& lo, int& hi) {
  lo = first;
  hi = ncodes - 1;
  if (window >= 0) {
    lo = max(first, c0 - window);
    hi = min(ncodes - 1, c0 + window);
    if (tab[c0].x == 0.0f) { lo = 1; hi = max(1, window); }
  }
}

// Smallest code whose value is >= v (ncodes if none).
__device__ __forceinline__ int grid_ceil(const float4* tab, int ncodes, float v) {
  int lo = 0, hi = ncodes;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (tab[mid].x >= v) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

inline GridTable make_grid_table(int sfmt) {
  GridTable t;
  const GridInfo g = grid_info(sfmt);
  t.ncodes = g.ncodes;
  t.first = g.first;
  t.sfmt = sfmt;
  for (int c = 0; c < 256; ++c) {
    if (c >= g.ncodes || grid_value(sfmt, c) == 0.0) {
      t.c[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const double v = grid_value(sfmt, c);
    const double r = 1.0 / v;
    const float rhi = (float)r;
    const float rlo = (float)(r - (double)rhi);
    t.c[c] = make_float4((float)v, rhi, rlo, 0.f);
  }
  return t;
}

}  // namespace mxq
