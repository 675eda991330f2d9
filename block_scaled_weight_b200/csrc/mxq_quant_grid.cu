// mxq_quant_grid.cu -- scale search + quantize for E2M1 or INT4 elements on any 8-bit
// block-scale grid: MXFP4 (E2M1 on UE8M0 powers of two), NVINT4 (INT4 on E4M3), and the
// UE4M4 / UE5M3 grids (qwantize "Results", sections "MXFP4 (UE8M0 power-of-2 scales)",
// "Exotic Scales", and the NVINT4 rows of "GPTQ Quantization"; "Is Finer Better? The
// Limits of Microscaling Formats in LLMs", sec. 2.1).
//
// Definitions as for NVFP4 (see mxq_quant.cu): candidate scale s from the grid's table,
// q_j = RNE_grid(fl32(|w_j| / s)) (E2M1 codebook, or the integers 0..7), w^_j = fl32(s q_j),
// error sum_j c_j (w_j - w^_j)^2 (c = 1 for SSE, h for H-optimal), ties to the lowest code.
//
// Exactness. Every grid value has at most 5 significant bits (UE4M4; 4 for E4M3 and UE5M3,
// 1 for UE8M0). A quotient |w| / s that is not a float32 is then at least 2^-30 (relative)
// away from every float32 rounding boundary (its distance to a midpoint, scaled to the
// 24-bit significand, is a nonzero multiple of 1 / (2 S) with S < 32), so the split-
// reciprocal quotient fma(a, r_hi, a r_lo) (error ~2^-46) rounds exactly like the IEEE
// quotient; for powers of two (r_lo = 0) it is the same product. Quotients below 2^-126
// round to code 0 either way. The dequantised product s g has at most 8 significant bits,
// so a - s g is one fma with a single rounding, as the definition's difference.
// Ranking, lower bounds, range cuts and flagging are those of the NVFP4 search; flagged
// blocks (bit 7 of the scale byte) are re-scored exactly by k_grid_fixup.
#include "mxq_block.cuh"
#include "mxq_common.cuh"
#include "mxq_grids.h"
#include "mxq_internal.h"

#include <cmath>

namespace mxq {

namespace {

constexpr int kThreads = 256;
enum { kElemE2M1 = 0, kElemInt4 = 1 };

// Per code: {s, r_hi, r_lo, 0} with r_hi + r_lo = 1/s to ~2^-48 (zero scale: all 0).
struct GridTable {
  float4 c[256];
  int ncodes, first, sfmt;
};

struct GridParams {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* h;
  int window;
  uint8_t* codes;
  uint8_t* scales;
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

// Float32 error of one candidate: sum_j c_j (a_j - s g_j)^2.
template <int B, int ELEM, bool HOPT>
__device__ __forceinline__ float grid_eval(const float2 (&a)[B / 2], const float2 (&c)[B / 2],
                                           float4 t) {
  const float2 ns = make_float2(-t.x, -t.x);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 d = __ffma2_rn(elem_values<ELEM>(quot2(a[p], t)), ns, a[p]);
    float2& acc = (p & 1) ? acc1 : acc0;
    if constexpr (HOPT) acc = __ffma2_rn(__fmul2_rn(c[p], d), d, acc);
    else acc = __ffma2_rn(d, d, acc);
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// Float32 error of the two bound elements at one candidate.
template <int ELEM>
__device__ __forceinline__ float grid_lb(float2 at, float2 ct, float4 t) {
  const float2 d = __ffma2_rn(elem_values<ELEM>(quot2(at, t)), make_float2(-t.x, -t.x), at);
  const float2 v = __fmul2_rn(__fmul2_rn(ct, d), d);
  return v.x + v.y;
}

// Double error of one candidate in the definition's order: e += c_j * (d * d),
// d = (double)|w_j| - (double)fl32(s g_j).
template <int B, int ELEM, bool HOPT>
__device__ double grid_exact(const float2 (&a)[B / 2], const float2 (&c)[B / 2], float4 t) {
  double e = 0.0;
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 g = elem_values<ELEM>(quot2(a[p], t));
    const double d0 = (double)a[p].x - (double)__fmul_rn(t.x, g.x);
    const double d1 = (double)a[p].y - (double)__fmul_rn(t.x, g.y);
    const double c0 = HOPT ? (double)c[p].x : 1.0;
    const double c1 = HOPT ? (double)c[p].y : 1.0;
    e = __dadd_rn(e, __dmul_rn(c0, __dmul_rn(d0, d0)));
    e = __dadd_rn(e, __dmul_rn(c1, __dmul_rn(d1, d1)));
  }
  return e;
}

// Packed codes of one block at table entry t: E2M1 nibbles sign << 3 | code, INT4 nibbles
// the two's complement of the signed code; element 2i in the low nibble.
template <int B, int ELEM>
__device__ __forceinline__ void grid_emit(const float2 (&a)[B / 2], uint32_t sgn, float4 t,
                                          uint8_t* dst) {
  const bool zero = t.x == 0.0f;
  uint32_t wds[B / 8];
#pragma unroll
  for (int i = 0; i < B / 8; ++i) wds[i] = 0;
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const uint32_t n0 = (sgn >> (2 * p)) & 1u, n1 = (sgn >> (2 * p + 1)) & 1u;
    uint32_t byte;
    if constexpr (ELEM == kElemE2M1) {
      const float2 x = quot2(a[p], t);
      byte = zero ? 0u : (e2m1x2_rn(x.x, x.y) & 0x77u);
      byte |= (n0 << 3) | (n1 << 7);
    } else {
      int q0 = 0, q1 = 0;
      if (!zero) {
        const float2 g = elem_values<ELEM>(quot2(a[p], t));
        q0 = (int)g.x;
        q1 = (int)g.y;
      }
      byte = (uint32_t)((n0 ? -q0 : q0) & 15) | ((uint32_t)((n1 ? -q1 : q1) & 15) << 4);
    }
    wds[p / 4] |= byte << (8 * (p % 4));
  }
  if constexpr (B == 16) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(wds[0], wds[1]);
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
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

}  // namespace
}  // namespace mxq

namespace mxq {
namespace {

// Search + quantize, one thread per block. Naive mode emits the naive code directly.
// The float32 winner is emitted when it is separated from every other candidate by the
// error band; otherwise the block is flagged (bit 7 of the scale byte) for k_grid_fixup.
// Lower bounds (as for NVFP4): the two elements with the largest c w^2 bound every
// candidate from below; single elements cut the range -- below max_j (a_j - sqrt(T/c_j))
// / qmax the saturated element alone costs more than the seed's upper bound T, and from
// min {a_j / zthr : c_j a_j^2 > T} on an element rounds to 0 (zthr = 1/4 for E2M1, 1/2
// for INT4) and alone costs more than T.
template <int B, bool BF16, int ELEM, int MODE>
__global__ void __launch_bounds__(kThreads, 2)
k_grid_search(GridParams P, GridTable T) {
  __shared__ float4 tab[256];
  for (int i = threadIdx.x; i < 256; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  constexpr bool HOPT = MODE == 2;
  constexpr float kQmax = ELEM == kElemE2M1 ? 6.0f : 7.0f;
  constexpr float kZero = ELEM == kElemE2M1 ? 4.0f : 2.0f;   // s >= kZero a: element -> 0
  const int ncodes = T.ncodes, first = T.first, sfmt = T.sfmt;
  const int64_t kb = P.k / B, nblocks = P.n * kb;
  const int elsz = BF16 ? 2 : 4;
  const float gam = (float)(B + 8) * 5.9604645e-8f;  // (B + 8) 2^-24
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;                // 2^-130: underflow slack
  const float inf = __int_as_float(0x7f800000);
  for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * kThreads) {
    const int64_t row = b / kb, jb = b - row * kb;
    float2 a[B / 2], c[B / 2];
    uint32_t sgn;
    load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
    if constexpr (HOPT) load_h<B>(P.h + jb * B, c);
    else {
#pragma unroll
      for (int p = 0; p < B / 2; ++p) c[p] = make_float2(1.f, 1.f);
    }
    const int c0 = naive_code<ELEM>(block_amax<B>(a), tab, ncodes, sfmt);
    uint8_t* dst = P.codes + row * (P.k / 2) + jb * (B / 2);
    if constexpr (MODE == 0) {
      grid_emit<B, ELEM>(a, sgn, tab[c0], dst);
      P.scales[b] = (uint8_t)c0;
      continue;
    }
    int lo, hi;
    grid_window(tab, ncodes, first, c0, P.window, lo, hi);
    float m1 = inf, m2 = inf;
    int i1 = lo;
    const int cs = min(max(c0, lo), hi);
    track(grid_eval<B, ELEM, HOPT>(a, c, tab[cs]), cs, m1, m2, i1);
    float upper = fmaf(m1, hi_f, slack);
    float2 at, ct;
    float s_cut = 0.f, s_hi = inf;
    {
      const float sqt = sqrtf(upper) * 1.00001f;
      float v1 = -1.f, a1 = 0.f, c1 = 0.f, v2 = -1.f, a2 = 0.f, c2 = 0.f;
      auto visit = [&](float aj, float cj) {
        const float v = cj * aj * aj;
        if (v > v1) { v2 = v1; a2 = a1; c2 = c1; v1 = v; a1 = aj; c1 = cj; }
        else if (v > v2) { v2 = v; a2 = aj; c2 = cj; }
        if (cj > 0.f) {
          s_cut = fmaxf(s_cut, (aj - sqt * rsqrtf(cj)) * (1.0f / kQmax) * 0.99999f);
          if (v * 0.99999f - slack > upper) s_hi = fminf(s_hi, kZero * aj);
        }
      };
#pragma unroll
      for (int p = 0; p < B / 2; ++p) {
        visit(a[p].x, c[p].x);
        visit(a[p].y, c[p].y);
      }
      at = make_float2(a1, a2);
      ct = make_float2(c1, c2);
    }
    if (s_cut > 0.f) lo = max(lo, grid_ceil(tab, ncodes, s_cut));
    if (s_hi < inf) hi = min(hi, grid_ceil(tab, ncodes, s_hi) - 1);
    const float lb_f = 1.0f - 8.0f * 5.9604645e-8f;
    for (int cc = lo; cc <= hi; ++cc) {
      if (cc == cs) continue;
      const float4 t = tab[cc];
      if (grid_lb<ELEM>(at, ct, t) * lb_f - slack > upper) continue;
      track(grid_eval<B, ELEM, HOPT>(a, c, t), cc, m1, m2, i1);
      upper = fmaf(m1, hi_f, slack);
    }
    if (!(m2 * lo_f - slack > upper)) {
      P.scales[b] = (uint8_t)(0x80 | i1);
    } else {
      grid_emit<B, ELEM>(a, sgn, tab[i1], dst);
      P.scales[b] = (uint8_t)i1;
    }
  }
}

// Exact pass over the flagged blocks (as k_fp4_fixup): a warp per flagged block, lanes
// evaluate candidates lo + lane + 32 t in float32, the warp minimum bounds the band, the
// candidates inside it are re-scored in double in the definition's order, and the warp
// arg-min (lowest code on equal doubles) is emitted.
template <int B, bool BF16, int ELEM, bool HOPT>
__global__ void __launch_bounds__(kThreads)
k_grid_fixup(GridParams P, GridTable T) {
  __shared__ float4 tab[256];
  for (int i = threadIdx.x; i < 256; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int ncodes = T.ncodes, first = T.first, sfmt = T.sfmt;
  const int64_t kb = P.k / B, nblocks = P.n * kb;
  const int elsz = BF16 ? 2 : 4;
  const float gam = (float)(B + 8) * 5.9604645e-8f;
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;
  const float inf = __int_as_float(0x7f800000);
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  for (int64_t base = gw * 32; base < nblocks; base += nw * 32) {
    const int64_t mine = base + lane;
    const bool flagged = mine < nblocks && (P.scales[mine] & 0x80);
    unsigned todo = __ballot_sync(kFull, flagged);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const int64_t b = base + src;
      const int64_t row = b / kb, jb = b - row * kb;
      float2 a[B / 2], c[B / 2];
      uint32_t sgn;
      load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
      if constexpr (HOPT) load_h<B>(P.h + jb * B, c);
      else {
#pragma unroll
        for (int p = 0; p < B / 2; ++p) c[p] = make_float2(1.f, 1.f);
      }
      const int c0 = naive_code<ELEM>(block_amax<B>(a), tab, ncodes, sfmt);
      int lo, hi;
      grid_window(tab, ncodes, first, c0, P.window, lo, hi);
      float ef[8];
      float mloc = inf;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int cc = lo + lane + 32 * t;
        ef[t] = cc <= hi ? grid_eval<B, ELEM, HOPT>(a, c, tab[cc]) : inf;
        mloc = fminf(mloc, ef[t]);
      }
      const float m1 = warp_min(mloc);
      const float upper = fmaf(m1, hi_f, slack);
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bi = 0x7fffffff;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int cc = lo + lane + 32 * t;
        if (cc <= hi && !(ef[t] * lo_f - slack > upper)) {
          const double ed = grid_exact<B, ELEM, HOPT>(a, c, tab[cc]);
          if (ed < best || (ed == best && cc < bi)) { best = ed; bi = cc; }
        }
      }
      warp_argmin(best, bi);
      if (bi > hi) bi = lo;  // every candidate NaN (non-finite input): keep the first
      if (lane == 0) {
        grid_emit<B, ELEM>(a, sgn, tab[bi], P.codes + row * (P.k / 2) + jb * (B / 2));
        P.scales[b] = (uint8_t)bi;
      }
    }
  }
}

GridTable make_grid_table(int sfmt) {
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

template <int B, bool BF16, int ELEM>
cudaError_t grid_dispatch(const QuantArgs& a, cudaStream_t st) {
  static const GridTable tables[4] = {make_grid_table(0), make_grid_table(1),
                                      make_grid_table(2), make_grid_table(3)};
  const GridTable& T = tables[a.scale_fmt];
  GridParams P{(const char*)a.W, a.n, a.k, a.ld * (BF16 ? 2 : 4), a.h, a.window,
               (uint8_t*)a.codes, (uint8_t*)a.scales};
  const int64_t nblocks = a.n * (a.k / B);
  const int64_t want = (nblocks + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sm_count() * 16;
  const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  if (a.mode == 0) {
    k_grid_search<B, BF16, ELEM, 0><<<grid, kThreads, 0, st>>>(P, T);
    return cudaGetLastError();
  }
  if (a.mode == 1) k_grid_search<B, BF16, ELEM, 1><<<grid, kThreads, 0, st>>>(P, T);
  else k_grid_search<B, BF16, ELEM, 2><<<grid, kThreads, 0, st>>>(P, T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t fwant = (nblocks + 32 * 8 - 1) / (32 * 8);
  const int fgrid = (int)(fwant < (int64_t)sm_count() * 8 ? fwant : (int64_t)sm_count() * 8);
  if (a.mode == 1) k_grid_fixup<B, BF16, ELEM, false><<<fgrid, kThreads, 0, st>>>(P, T);
  else k_grid_fixup<B, BF16, ELEM, true><<<fgrid, kThreads, 0, st>>>(P, T);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_grid(const QuantArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == 1;
  if (a.fmt == 0) {
    if (a.block == 16)
      return bf ? grid_dispatch<16, true, kElemE2M1>(a, st) : grid_dispatch<16, false, kElemE2M1>(a, st);
    return bf ? grid_dispatch<32, true, kElemE2M1>(a, st) : grid_dispatch<32, false, kElemE2M1>(a, st);
  }
  if (a.block == 16)
    return bf ? grid_dispatch<16, true, kElemInt4>(a, st) : grid_dispatch<16, false, kElemInt4>(a, st);
  return bf ? grid_dispatch<32, true, kElemInt4>(a, st) : grid_dispatch<32, false, kElemInt4>(a, st);
}

}  // namespace mxq
