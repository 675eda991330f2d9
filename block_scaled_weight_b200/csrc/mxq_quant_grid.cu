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
#include "mxq_gridk.cuh"
#include "mxq_internal.h"

#include <cmath>

namespace mxq {

namespace {

constexpr int kThreads = 256;

struct GridParams {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* h;
  int window;
  uint8_t* codes;
  uint8_t* scales;
};

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

// ---------------------------------------------------------------------------------------
// Block-Hessian objective: candidate error d^T G_b d with the block's Gram matrix G_b
// ("quantization_algorithms.txt", sec. 1: the exact output-error objective of a block).
// A CTA owns one column block b (G_b staged in shared memory) and 256 consecutive rows;
// thread t quantizes row t's block. Per candidate: signed differences d (as in the grid
// search), t = G_b d with packed FMAs, e = d . t in float32.
// Bracket: |e_f - e| <= (B + 4) u sum_ij |G_ij| |d_i| |d_j| (float32 roundings of d, of the
// B-term products and of the final dot), and sum_ij |G_ij| |d_i||d_j| <= kappa
// (sum_i sqrt(G_ii) |d_i|)^2 with kappa = max(1, max_ij |G_ij| / sqrt(G_ii G_jj)) computed
// per block (1 for any Gram matrix; infinite when a diagonal entry is not positive, which
// sends every block to the exact pass). Flagged blocks are re-scored exactly by
// k_gram_fixup in the definition's order (e += G_ij * (d_i * d_j), i then j, in double).
// ---------------------------------------------------------------------------------------
struct GramSearchParams {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* G;  // [k/B][B][B]
  int window;
  uint8_t* codes;
  uint8_t* scales;
};

// kappa of one B x B block (see above); +inf when some G_ii <= 0 or a value is not finite.
template <int B>
__device__ float gram_kappa(const float* g) {
  float kap = 1.0f;
  for (int i = 0; i < B; ++i) {
    const float gi = g[i * B + i];
    if (!(gi > 0.0f) || !(gi < __int_as_float(0x7f800000))) return __int_as_float(0x7f800000);
    for (int j = 0; j < B; ++j) {
      const float gj = g[j * B + j];
      if (!(gj > 0.0f)) return __int_as_float(0x7f800000);
      const float r = fabsf(g[i * B + j]) / sqrtf(gi * gj);
      if (!(r <= 1e30f)) return __int_as_float(0x7f800000);
      kap = fmaxf(kap, r);
    }
  }
  return kap * 1.0001f;  // covers the roundings of this estimate
}

// Signed differences d_j = w_j - sign(w_j) fl32(s g_j) of one candidate, in pairs.
template <int B, int ELEM>
__device__ __forceinline__ void gram_diffs(const float2 (&a)[B / 2], uint32_t sgn, float4 t,
                                           float2 (&d)[B / 2]) {
  const float2 ns = make_float2(-t.x, -t.x);
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 dd = __ffma2_rn(elem_values<ELEM>(quot2(a[p], t)), ns, a[p]);
    d[p].x = __uint_as_float(__float_as_uint(dd.x) ^ (((sgn >> (2 * p)) & 1u) << 31));
    d[p].y = __uint_as_float(__float_as_uint(dd.y) ^ (((sgn >> (2 * p + 1)) & 1u) << 31));
  }
}

// A 16-byte shared-memory load the compiler may not hoist out of the candidate loop (G
// is loop-invariant; kept in registers it would not fit).
__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Float32 d^T G d and the bracket's sum_i sqrt(G_ii) |d_i| (g: G_b in shared memory,
// sq: sqrt(G_ii)).
template <int B>
__device__ __forceinline__ float gram_form(const float2 (&d)[B / 2], const float* g,
                                           const float* sq, float& sd) {
  float e = 0.0f;
  float2 s2 = make_float2(0.f, 0.f);
  const uint32_t gbase = (uint32_t)__cvta_generic_to_shared(g);
#pragma unroll
  for (int i = 0; i < B; ++i) {
    float2 t0 = make_float2(0.f, 0.f), t1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < B / 4; ++q) {
      const float4 gv = lds4(gbase + (uint32_t)((i * B + 4 * q) * 4));
      t0 = __ffma2_rn(make_float2(gv.x, gv.y), d[2 * q], t0);
      t1 = __ffma2_rn(make_float2(gv.z, gv.w), d[2 * q + 1], t1);
    }
    const float ti = (t0.x + t0.y) + (t1.x + t1.y);
    const float di = (i & 1) ? d[i / 2].y : d[i / 2].x;
    e = fmaf(di, ti, e);
  }
#pragma unroll
  for (int p = 0; p < B / 2; p += 2) {
    const float4 q4 = lds4((uint32_t)__cvta_generic_to_shared(sq) + (uint32_t)(p * 8));
    s2 = __ffma2_rn(make_float2(q4.x, q4.y), make_float2(fabsf(d[p].x), fabsf(d[p].y)), s2);
    s2 = __ffma2_rn(make_float2(q4.z, q4.w), make_float2(fabsf(d[p + 1].x), fabsf(d[p + 1].y)), s2);
  }
  sd = s2.x + s2.y;
  return e;
}

// Double d^T G d in the definition's order.
template <int B, int ELEM>
__device__ double gram_exact(const float2 (&a)[B / 2], uint32_t sgn, float4 t, const float* g) {
  double d[B];
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 v = elem_values<ELEM>(quot2(a[p], t));
    const float w0 = ((sgn >> (2 * p)) & 1u) ? -a[p].x : a[p].x;
    const float w1 = ((sgn >> (2 * p + 1)) & 1u) ? -a[p].y : a[p].y;
    const float q0 = __fmul_rn(t.x, v.x), q1 = __fmul_rn(t.x, v.y);
    d[2 * p] = (double)w0 - (double)(((sgn >> (2 * p)) & 1u) ? -q0 : q0);
    d[2 * p + 1] = (double)w1 - (double)(((sgn >> (2 * p + 1)) & 1u) ? -q1 : q1);
  }
  double e = 0.0;
  for (int i = 0; i < B; ++i)
#pragma unroll
    for (int j = 0; j < B; ++j) e = __dadd_rn(e, __dmul_rn((double)g[i * B + j], __dmul_rn(d[i], d[j])));
  return e;
}

// Pruning (as the diagonal searches, with per-element weights that bound the quadratic
// form from below): d^T G d >= sum_i cg_i d_i^2 with the Gershgorin weights
// cg_i = G_ii - sum_{j != i} (|G_ij| + |G_ji|) / 2 (|G_ij d_i d_j| <= |G_ij| (d_i^2 + d_j^2)
// / 2). Bounds from a subset of elements (the range cuts, the two-element bound) need every
// cg_i >= 0, i.e. a diagonally dominant G (weakly correlated inputs); otherwise all cg are
// set to 0 and every candidate is evaluated. With U the smallest upper bracket seen (the
// seed's first), the saturation and zero range cuts and the two-element bound of
// k_grid_search apply with cg in place of c; a candidate whose bound exceeds U can neither
// win nor tie.
template <int B, bool BF16, int ELEM>
__global__ void __launch_bounds__(kThreads, 2)
k_gram_search(GramSearchParams P, GridTable T) {
  __shared__ float4 tab[256];
  __shared__ __align__(16) float g[B * B];
  __shared__ __align__(16) float sq[B];
  __shared__ float cg[B];
  __shared__ float kap_s;
  __shared__ int dominant;
  for (int i = threadIdx.x; i < 256; i += kThreads) tab[i] = T.c[i];
  const int64_t kb = P.k / B;
  const int64_t jb = blockIdx.x;
  for (int i = threadIdx.x; i < B * B; i += kThreads) g[i] = P.G[jb * B * B + i];
  if (threadIdx.x == 0) dominant = 1;
  __syncthreads();
  if (threadIdx.x < B) {
    const int i = threadIdx.x;
    sq[i] = sqrtf(fmaxf(g[i * (B + 1)], 0.0f));
    double off = 0.0;
    for (int j = 0; j < B; ++j)
      if (j != i) off += 0.5 * (fabs((double)g[i * B + j]) + fabs((double)g[j * B + i]));
    const double w = (double)g[i * (B + 1)] - off;
    const bool ok = w >= 0.0 && w < 1e38;
    cg[i] = ok ? __double2float_rd(w * (1.0 - 1e-12)) : 0.0f;
    if (!ok) dominant = 0;
  }
  if (threadIdx.x == 0) kap_s = gram_kappa<B>(g);
  __syncthreads();
  if (!dominant && threadIdx.x < B) cg[threadIdx.x] = 0.0f;
  __syncthreads();
  constexpr float kQmax = ELEM == kElemE2M1 ? 6.0f : 7.0f;
  constexpr float kZero = ELEM == kElemE2M1 ? 4.0f : 2.0f;
  const float kap = kap_s;
  const int ncodes = T.ncodes, first = T.first, sfmt = T.sfmt;
  const int elsz = BF16 ? 2 : 4;
  const float gam = (float)(B + 4) * 5.9604645e-8f * kap;
  const float slack = 7.3468396e-40f;
  const float inf = __int_as_float(0x7f800000);
  const float lb_f = 1.0f - 8.0f * 5.9604645e-8f;
  for (int64_t row = (int64_t)blockIdx.y * kThreads + threadIdx.x; row < P.n;
       row += (int64_t)gridDim.y * kThreads) {
    float2 a[B / 2];
    uint32_t sgn;
    load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
    const int c0 = naive_code<ELEM>(block_amax<B>(a), tab, ncodes, sfmt);
    int lo, hi;
    grid_window(tab, ncodes, first, c0, P.window, lo, hi);
    float m1 = inf, h1 = inf, l1 = inf, l2 = inf, U = inf;
    int i1 = lo, j1 = -1;
    auto visit = [&](int cc) {
      float2 d[B / 2];
      gram_diffs<B, ELEM>(a, sgn, tab[cc], d);
      float sd;
      const float e = gram_form<B>(d, g, sq, sd);
      const float w = fmaf(gam * sd, sd, slack);
      const float elo = e - w;
      if (e < m1) { m1 = e; i1 = cc; h1 = e + w; }
      if (elo < l1) { l2 = l1; l1 = elo; j1 = cc; }
      else if (elo < l2) l2 = elo;
      U = fminf(U, e + w);
    };
    const int cs = min(max(c0, lo), hi);
    visit(cs);
    float2 at = make_float2(0.f, 0.f), ct = make_float2(0.f, 0.f);
    if (U < inf) {
      const float sqt = sqrtf(fmaxf(U, 0.0f)) * 1.00001f;
      float s_cut = 0.f, s_hi = inf;
      float v1 = -1.f, a1 = 0.f, c1 = 0.f, v2 = -1.f, a2 = 0.f, c2 = 0.f;
#pragma unroll
      for (int p = 0; p < B; ++p) {
        const float aj = (p & 1) ? a[p / 2].y : a[p / 2].x, cj = cg[p];
        const float v = cj * aj * aj;
        if (v > v1) { v2 = v1; a2 = a1; c2 = c1; v1 = v; a1 = aj; c1 = cj; }
        else if (v > v2) { v2 = v; a2 = aj; c2 = cj; }
        if (cj > 0.f) {
          s_cut = fmaxf(s_cut, (aj - sqt * rsqrtf(cj)) * (1.0f / kQmax) * 0.99999f);
          if (v * 0.99999f - slack > U) s_hi = fminf(s_hi, kZero * aj);
        }
      }
      at = make_float2(a1, a2);
      ct = make_float2(c1, c2);
      if (s_cut > 0.f) lo = max(lo, grid_ceil(tab, ncodes, s_cut));
      if (s_hi < inf) hi = min(hi, grid_ceil(tab, ncodes, s_hi) - 1);
    }
    for (int cc = lo; cc <= hi; ++cc) {
      if (cc == cs) continue;
      if (grid_lb<ELEM>(at, ct, tab[cc]) * lb_f - slack > U) continue;
      visit(cc);
    }
    const bool flag = !((j1 == i1 ? l2 : l1) > h1);
    const int64_t b = row * kb + jb;
    grid_emit<B, ELEM>(a, sgn, tab[i1], P.codes + row * (P.k / 2) + jb * (B / 2));
    P.scales[b] = (uint8_t)(i1 | (flag ? 0x80 : 0));
  }
}

// Exact pass over flagged blocks: one warp per flagged block. The block's G is staged in
// the warp's slice of shared memory; lane l evaluates candidates lo + l + 32 t in float32
// with their brackets (as the search), and only the candidates whose bracket reaches the
// smallest upper end are scored in double in the definition's order (e += G_ij (d_i d_j),
// i then j); the warp arg-min (lowest code on equal values) wins.
template <int B, bool BF16, int ELEM>
__global__ void __launch_bounds__(kThreads)
k_gram_fixup(GramSearchParams P, GridTable T) {
  constexpr int kWarps = kThreads / 32;
  __shared__ float4 tab[256];
  __shared__ __align__(16) float gw_s[kWarps][B * B];
  __shared__ __align__(16) float sq_s[kWarps][B];
  for (int i = threadIdx.x; i < 256; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float* g = gw_s[wid];
  float* sq = sq_s[wid];
  const int ncodes = T.ncodes, first = T.first, sfmt = T.sfmt;
  const int64_t kb = P.k / B, nblocks = P.n * kb;
  const int elsz = BF16 ? 2 : 4;
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
      float2 a[B / 2];
      uint32_t sgn;
      load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
      const float* gb = P.G + jb * B * B;
      __syncwarp();
      for (int i = lane; i < B * B; i += 32) g[i] = gb[i];
      __syncwarp();
      // kappa of the block (as gram_kappa), one row per lane
      float kl = 1.0f;
      if (lane < B) {
        const float gi = g[lane * (B + 1)];
        sq[lane] = sqrtf(fmaxf(gi, 0.0f));
        if (!(gi > 0.0f) || !(gi < inf)) kl = inf;
        for (int j = 0; j < B && kl < inf; ++j) {
          const float gj = g[j * (B + 1)];
          const float r = (gj > 0.0f) ? fabsf(g[lane * B + j]) / sqrtf(gi * gj) : inf;
          kl = (r <= 1e30f) ? fmaxf(kl, r) : inf;
        }
      }
      const float kap = warp_max(kl) * 1.0001f;
      __syncwarp();
      const float gam = (float)(B + 4) * 5.9604645e-8f * kap;
      const int c0 = naive_code<ELEM>(block_amax<B>(a), tab, ncodes, sfmt);
      int lo, hi;
      grid_window(tab, ncodes, first, c0, P.window, lo, hi);
      float ef[8], wf[8];
      float up = inf;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int cc = lo + lane + 32 * t;
        ef[t] = inf;
        wf[t] = 0.f;
        if (cc <= hi) {
          float2 d[B / 2];
          gram_diffs<B, ELEM>(a, sgn, tab[cc], d);
          float sd;
          ef[t] = gram_form<B>(d, g, sq, sd);
          wf[t] = fmaf(gam * sd, sd, slack);
          up = fminf(up, ef[t] + wf[t]);
        }
      }
      up = warp_min(up);
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bi = 0x7fffffff;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int cc = lo + lane + 32 * t;
        if (cc <= hi && !(ef[t] - wf[t] > up)) {
          const double ed = gram_exact<B, ELEM>(a, sgn, tab[cc], gb);
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

template <int B, bool BF16, int ELEM>
cudaError_t gram_dispatch(const QuantArgs& a, cudaStream_t st) {
  static const GridTable tables[4] = {make_grid_table(0), make_grid_table(1),
                                      make_grid_table(2), make_grid_table(3)};
  const GridTable& T = tables[a.scale_fmt];
  GramSearchParams P{(const char*)a.W, a.n, a.k, a.ld * (BF16 ? 2 : 4), a.G, a.window,
                     (uint8_t*)a.codes, (uint8_t*)a.scales};
  const int64_t kb = a.k / B;
  int64_t ry = (a.n + kThreads - 1) / kThreads;
  const int64_t target = (int64_t)sm_count() * 8;
  if (ry * kb > target) ry = (target + kb - 1) / kb;
  if (ry < 1) ry = 1;
  if (ry > 65535) ry = 65535;
  k_gram_search<B, BF16, ELEM><<<dim3((unsigned)kb, (unsigned)ry), kThreads, 0, st>>>(P, T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nblocks = a.n * kb;
  const int64_t fwant = (nblocks + 32 * 8 - 1) / (32 * 8);
  const int fgrid = (int)(fwant < (int64_t)sm_count() * 8 ? fwant : (int64_t)sm_count() * 8);
  k_gram_fixup<B, BF16, ELEM><<<fgrid, kThreads, 0, st>>>(P, T);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_gram(const QuantArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == 1;
  if (a.fmt == 0) {
    if (a.block == 16)
      return bf ? gram_dispatch<16, true, kElemE2M1>(a, st) : gram_dispatch<16, false, kElemE2M1>(a, st);
    return bf ? gram_dispatch<32, true, kElemE2M1>(a, st) : gram_dispatch<32, false, kElemE2M1>(a, st);
  }
  if (a.block == 16)
    return bf ? gram_dispatch<16, true, kElemInt4>(a, st) : gram_dispatch<16, false, kElemInt4>(a, st);
  return bf ? gram_dispatch<32, true, kElemInt4>(a, st) : gram_dispatch<32, false, kElemInt4>(a, st);
}

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
