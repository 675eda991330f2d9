// mxq_quant.cu -- fused per-block scale search + quantize (naive / sse / hopt).
//
// Definitions ("Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1;
// qwantize "Results", INT8 and NVFP4 sections; "quantization_algorithms.txt", sec. 1):
//   naive  s0 = RNE_E4M3(amax / qmax)  (INT8: the stored amax RNE_E4M3(amax))
//   sse    argmin_s  sum_j (w_j - fl32(s q_j))^2
//   hopt   argmin_s  sum_j h_j (w_j - fl32(s q_j))^2,  q_j = RNE_grid(fl32(|w_j| / s))
// Candidate ties go to the smallest scale.
//
// Exactness. The element decisions use exactly the IEEE float32 quotient:
//  * NVFP4: an E4M3 scale has a significand of at most 4 bits, so |w| / s can never lie
//    within 2^-29 (relative) of a float32 rounding boundary without being a float32
//    itself. The quotient is formed as fma(a, r_hi, a * r_lo) with r_hi + r_lo = 1/s to
//    ~2^-48 (host-computed split of the reciprocal), whose error (~2^-46) is far inside
//    that gap: the result is the correctly rounded quotient, bit for bit.
//  * INT8 and E4M3 tiles rank candidates with the product |w| * fl32(1/s) instead, and
//    widen their error brackets by the largest change that a code differing from the
//    IEEE quotient's can make (see the INT8 and tile sections); emitted codes and exact
//    re-scores use __fdiv_rn, the IEEE-rounded division.
// Candidate errors are accumulated in float32 (packed f32x2 math); with every term
// non-negative the float32 sum is within gamma (relative) plus a tiny absolute underflow
// slack of the exact sum. Any candidate whose lower bound does not exceed the winner's
// upper bound is re-scored in double exactly as the plain definition orders it (element
// order, e += c_j * (d * d)), and the smallest double error (lowest index on ties) wins.
// So NVFP4 and INT8 picks equal the definition's, ties included. E4M3 tiles re-score in
// double in a fixed parallel order: picks equal the definition's wherever the two best
// tile errors differ by more than ~1e-12 relative.
#include "mxq_block.cuh"
#include "mxq_common.cuh"
#include "mxq_internal.h"

#include <cuda_fp16.h>

#include <cmath>
#include <cstring>

namespace mxq {

namespace {

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------------------
// Per-candidate constants for NVFP4: {s, r_hi, r_lo, s as fp16 bits}. Computed once on
// the host (double arithmetic), passed by value and staged in shared memory.
// ---------------------------------------------------------------------------------------
struct Fp4Table {
  float4 c[128];
  float2 sig[8];  // split reciprocals 8/S of the normal significands S = 8..15
};

struct Fp4Params {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* h;
  int window;
  uint8_t* codes;
  uint8_t* scales;
  double* err_partial;     // per-CTA error sums (search CTAs, then fixup CTAs), or null
  const float* h_err;      // h for the h-weighted sums of an SSE search, or null
  int fix_slot0;           // first partial slot of the fixup CTAs
};

// fl32(|w| / s) for an E4M3 scale s, from the split reciprocal (see the file header).
__device__ __forceinline__ float2 fp4_quot(float2 a, float2 rhi, float2 rlo) {
  return __ffma2_rn(a, rhi, __fmul2_rn(a, rlo));
}

// a - s * g for a pair of elements at one candidate: the E2M1 codes of the exact float32
// quotients x, decoded to halves, and one mixed-precision FMA each with the negated fp16
// scale (s g is exact; a single rounding of the difference). The E2M1 byte never leaves
// a .b8 register.
__device__ __forceinline__ float2 fp4_pair_diff(float2 a, float2 x, uint32_t s_neg_h) {
  float d0, d1;
  asm("{\n\t.reg .b8 q;\n\t.reg .b32 g;\n\t.reg .b16 g0, g1, sn, sx;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %3, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 g, q;\n\t"
      "mov.b32 {g0, g1}, g;\n\t"
      "mov.b32 {sn, sx}, %6;\n\t"
      "fma.rn.f32.f16 %0, g0, sn, %4;\n\t"
      "fma.rn.f32.f16 %1, g1, sn, %5;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(x.x), "f"(x.y), "f"(a.x), "f"(a.y), "r"(s_neg_h));
  return make_float2(d0, d1);
}

// Float32 error of one candidate: sum_j c_j (a_j - s g_j)^2 (c_j = 1 for SSE).
template <int B, bool HOPT>
__device__ __forceinline__ float fp4_eval(const float2 (&a)[B / 2], const float2 (&c)[B / 2],
                                          float4 t) {
  const float2 rhi = make_float2(t.y, t.y), rlo = make_float2(t.z, t.z);
  const uint32_t s_neg_h = __float_as_uint(t.w) ^ 0x8000u;
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 d = fp4_pair_diff(a[p], fp4_quot(a[p], rhi, rlo), s_neg_h);
    float2& acc = (p & 1) ? acc1 : acc0;
    if constexpr (HOPT) {
      acc = __ffma2_rn(__fmul2_rn(c[p], d), d, acc);
    } else {
      acc = __ffma2_rn(d, d, acc);
    }
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// Double error of one candidate, in the definition's order: e += c_j * (d * d),
// d = (double)|w_j| - (double)fl32(s g_j).
template <int B, bool HOPT>
__device__ double fp4_exact(const float2 (&a)[B / 2], const float2 (&c)[B / 2], float4 t) {
  const float2 rhi = make_float2(t.y, t.y), rlo = make_float2(t.z, t.z);
  double e = 0.0;
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 x = fp4_quot(a[p], rhi, rlo);
    const uint32_t g = e2m1x2_to_f16x2(e2m1x2_rn(x.x, x.y));
    const float g0 = __half2float(__ushort_as_half(lo16(g)));
    const float g1 = __half2float(__ushort_as_half(hi16(g)));
    const double d0 = (double)a[p].x - (double)__fmul_rn(t.x, g0);
    const double d1 = (double)a[p].y - (double)__fmul_rn(t.x, g1);
    const double c0 = HOPT ? (double)c[p].x : 1.0;
    const double c1 = HOPT ? (double)c[p].y : 1.0;
    e = __dadd_rn(e, __dmul_rn(c0, __dmul_rn(d0, d0)));
    e = __dadd_rn(e, __dmul_rn(c1, __dmul_rn(d1, d1)));
  }
  return e;
}

// Packed NVFP4 codes of one block at candidate table entry t (scale code != 0).
template <int B>
__device__ __forceinline__ void fp4_emit(const float2 (&a)[B / 2], uint32_t sgn, float4 t,
                                         bool zero, uint8_t* dst) {
  const float2 rhi = make_float2(t.y, t.y), rlo = make_float2(t.z, t.z);
  uint32_t wds[B / 8];
#pragma unroll
  for (int i = 0; i < B / 8; ++i) wds[i] = 0;
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    uint32_t byte = 0;
    if (!zero) {
      const float2 x = fp4_quot(a[p], rhi, rlo);
      byte = e2m1x2_rn(x.x, x.y);
    }
    byte |= ((sgn >> (2 * p)) & 1u) << 3;
    byte |= ((sgn >> (2 * p + 1)) & 1u) << 7;
    wds[p / 4] |= byte << (8 * (p % 4));
  }
  if constexpr (B == 16) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(wds[0], wds[1]);
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

// NVFP4, naive: one thread per block (HBM-bound).
template <int B, bool BF16>
__global__ void __launch_bounds__(kThreads)
k_fp4_naive(Fp4Params P, Fp4Table T) {
  __shared__ float4 tab[128];
  for (int i = threadIdx.x; i < 128; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int64_t kb = P.k / B, nblocks = P.n * kb;
  const int elsz = BF16 ? 2 : 4;
  for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * kThreads) {
    const int64_t row = b / kb, jb = b - row * kb;
    float2 a[B / 2];
    uint32_t sgn;
    load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
    const int c0 = e4m3_rn_code(__fdiv_rn(block_amax<B>(a), 6.0f));
    fp4_emit<B>(a, sgn, tab[c0], c0 == 0, P.codes + row * (P.k / 2) + jb * (B / 2));
    P.scales[b] = (uint8_t)c0;
  }
}

// Float32 error of the two bound elements (at, with weights ct) at one candidate.
__device__ __forceinline__ float fp4_lb(float2 at, float2 ct, float2 x, uint32_t s_neg_h) {
  const float2 d = fp4_pair_diff(at, x, s_neg_h);
  const float2 v = __fmul2_rn(__fmul2_rn(ct, d), d);
  return v.x + v.y;
}


// NVFP4, SSE / H-optimal search, compacted. A warp owns 32 blocks: one column block jb
// (so h is the same for every lane and stays in registers) in 32 consecutive rows, one block
// per lane. Every lane first scores, in full and in step with the other lanes, a window of
// codes around its naive code (naive - 1 .. naive + 5: the winner is usually there), then
// filters the codes the range cuts leave outside the window with exact lower bounds, writing
// the codes that survive into its own list in shared memory. The warp then scores the surviving (block, code) pairs 32 at a time -- every lane
// takes the next pair, whoever's block it is, reading that block's magnitudes from shared
// memory -- and each lane folds its own results back in code order. Blocks whose float32
// winner is not separated from the runner-up by the error bound are flagged (bit 7 of the
// scale byte) for k_fp4_fixup. With P.err_partial set, the kernel also adds each unflagged
// block's error sums at its winning scale (float32 over the block, double beyond) into
// per-CTA partials.
constexpr int kFp4WinLo = -1, kFp4WinHi = 5;   // codes every lane scores in full
constexpr int kFp4Queue = 128;       // scored pairs held per warp before the owners fold them
constexpr int kFp4List = 132;        // bytes per lane's code list (126 codes; rows offset by a bank)

template <int B>
struct Fp4WarpSmem {
  float a[32][B];                    // each lane's block magnitudes
  float res[kFp4Queue];              // scores of the current window of pairs
  int off[32];                       // first pair of each lane (exclusive prefix of counts)
  uint8_t list[32 * kFp4List];       // surviving codes of each lane, ascending
};

template <int B>
constexpr size_t fp4_search_smem() {
  return (size_t)(kThreads / 32) * sizeof(Fp4WarpSmem<B>);
}

// Error sums of one block at table entry t: sum d^2, sum a^2, sum c d^2, sum c a^2 (float32
// over the block, as the error pass does) added to acc in double.
template <int B, bool HAS_C>
__device__ __forceinline__ void fp4_block_sums(const float2 (&a)[B / 2], const float2 (&c)[B / 2],
                                               float4 t, double (&acc)[4]) {
  const float2 rhi = make_float2(t.y, t.y), rlo = make_float2(t.z, t.z);
  const uint32_t sn = __float_as_uint(t.w) ^ 0x8000u;
  float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
#pragma unroll
  for (int p = 0; p < B / 2; ++p) {
    const float2 d = fp4_pair_diff(a[p], fp4_quot(a[p], rhi, rlo), sn);
    const float2 d2 = __fmul2_rn(d, d), w2 = __fmul2_rn(a[p], a[p]);
    s0 = __fadd2_rn(s0, d2);
    s1 = __fadd2_rn(s1, w2);
    if constexpr (HAS_C) {
      s2 = __ffma2_rn(c[p], d2, s2);
      s3 = __ffma2_rn(c[p], w2, s3);
    }
  }
  acc[0] += (double)s0.x + (double)s0.y;
  acc[1] += (double)s1.x + (double)s1.y;
  if constexpr (HAS_C) {
    acc[2] += (double)s2.x + (double)s2.y;
    acc[3] += (double)s3.x + (double)s3.y;
  }
}

// Fixed-order sum of the CTA's per-thread sums into partial[slot][4].
__device__ void cta_sums(const double (&acc)[4], double* partial, int slot) {
  __shared__ double red[kThreads / 32][4];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double r = warp_sum(acc[i]);
    if (lane == 0) red[wid][i] = r;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += red[w][threadIdx.x];
    partial[(int64_t)slot * 4 + threadIdx.x] = s;
  }
}

template <int B, bool BF16, bool HOPT>
__global__ void __launch_bounds__(kThreads, B == 16 ? 3 : 2)
k_fp4_search(Fp4Params P, Fp4Table T) {
  __shared__ float4 tab[128];
  extern __shared__ __align__(16) unsigned char fp4_dyn[];
  Fp4WarpSmem<B>& S = reinterpret_cast<Fp4WarpSmem<B>*>(fp4_dyn)[threadIdx.x >> 5];
  for (int i = threadIdx.x; i < 128; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t kb = P.k / B, ntiles = (P.n + 31) / 32 * kb;
  const int elsz = BF16 ? 2 : 4;
  const float gam = (float)(B + 8) * 5.9604645e-8f;  // (B + 8) 2^-24
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;                // 2^-130: underflow slack
  const float lb_f = 1.0f - 8.0f * 5.9604645e-8f;
  const bool want_err = P.err_partial != nullptr;
  const bool err_h = HOPT || P.h_err != nullptr;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  uint8_t* my_list = S.list + lane * kFp4List;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  for (int64_t tile = gw; tile < ntiles; tile += nw) {
    const int64_t rg = tile / kb, jb = tile - rg * kb;
    const int64_t row = rg * 32 + lane;
    const bool valid = row < P.n;
    float2 a[B / 2], c[B / 2];
    uint32_t sgn = 0;
    if (valid) {
      load_block<B, BF16>(P.W + row * P.ld_bytes + jb * B * elsz, a, sgn);
    } else {
#pragma unroll
      for (int p = 0; p < B / 2; ++p) a[p] = make_float2(0.f, 0.f);
    }
    if constexpr (HOPT) load_h<B>(P.h + jb * B, c);
    const int c0 = e4m3_rn_code(__fdiv_rn(block_amax<B>(a), 6.0f));
    int lo = 1, hi = 126;
    if (P.window >= 0) {
      lo = max(1, c0 - P.window);
      hi = min(126, c0 + P.window);
      if (c0 == 0) { lo = 1; hi = max(1, P.window); }
    }
    if (!valid) hi = 0;                                // no candidates
    float m1 = __int_as_float(0x7f800000), m2 = m1;
    int i1 = lo;
    // a window of codes around the naive code (clipped to the candidate range), in full
    const int cs = min(max(c0, lo), max(hi, lo));
#pragma unroll
    for (int d = kFp4WinLo; d <= kFp4WinHi; ++d) {
      const int cc = cs + d;
      if (cc >= lo && cc <= hi) track(fp4_eval<B, HOPT>(a, c, tab[cc]), cc, m1, m2, i1);
    }
    int cnt = 0;
    if (valid) {
      // Lower bounds. A candidate's error is at least the error of any subset of elements;
      // the subset here is the two elements with the largest c w^2 (t1, t2). A candidate
      // whose bound, minus its float32 rounding margin, exceeds the upper bound T of the
      // best error so far can neither win nor tie, nor fall in the band that decides
      // flagging: it is never scored.
      //
      // Range cuts, from single elements j:
      //  * for s < a_j / 6, element j maps to 6 s, so the error is at least
      //    c_j (a_j - 6 s)^2, growing as s shrinks: every s below
      //    max_j (a_j - sqrt(T / c_j)) / 6 is out;
      //  * for s >= 4 a_j, element j's quotient is at most 0.25 and it maps to 0,
      //    contributing exactly c_j a_j^2: every s >= min {4 a_j : c_j a_j^2 > T} is out.
      // The margins (1e-5 relative) cover the float32 roundings of the approximate
      // reciprocal square root and products.
      const float upper = fmaf(m1, hi_f, slack);
      float2 at, ct;
      float s_cut = 0.f, s_hi = __int_as_float(0x7f800000);
      {
        const float sqt = sqrtf(upper) * 1.00001f;
        float v1 = -1.f, a1 = 0.f, c1 = 0.f, v2 = -1.f, a2 = 0.f, c2 = 0.f;
        auto visit = [&](float aj, float cj) {
          const float v = cj * aj * aj;
          if (v > v1) { v2 = v1; a2 = a1; c2 = c1; v1 = v; a1 = aj; c1 = cj; }
          else if (v > v2) { v2 = v; a2 = aj; c2 = cj; }
          if (cj > 0.f) {
            s_cut = fmaxf(s_cut, (aj - sqt * rsqrtf(cj)) * (1.0f / 6.0f) * 0.99999f);
            if (v * 0.99999f - slack > upper) s_hi = fminf(s_hi, 4.0f * aj);
          }
        };
#pragma unroll
        for (int p = 0; p < B / 2; ++p) {
          visit(a[p].x, HOPT ? c[p].x : 1.f);
          visit(a[p].y, HOPT ? c[p].y : 1.f);
        }
        at = make_float2(a1, a2);
        ct = make_float2(c1, c2);
      }
      int lo2 = lo, hi2 = hi;
      if (s_cut > 0.f) {
        int cl = e4m3_rn_code(s_cut);
        if (e4m3_pos(cl) < s_cut) ++cl;                 // smallest code with value >= s_cut
        lo2 = max(lo2, cl);
      }
      if (s_hi < 1e30f) {
        int ch = e4m3_rn_code(s_hi);
        if (!(e4m3_pos(ch) < s_hi)) --ch;               // largest code with value < s_hi
        hi2 = min(hi2, ch);
      }
      // the codes the cuts leave below and above the window, two at a time (independent)
      auto bound_range = [&](int c_lo, int c_hi) {
        for (int cc = c_lo; cc <= c_hi; cc += 2) {
          const int cd = min(cc + 1, c_hi);
          const float4 t0 = tab[cc], t1 = tab[cd];
          const float l0 = fp4_lb(at, ct, fp4_quot(at, make_float2(t0.y, t0.y),
                                                   make_float2(t0.z, t0.z)),
                                  __float_as_uint(t0.w) ^ 0x8000u);
          const float l1 = fp4_lb(at, ct, fp4_quot(at, make_float2(t1.y, t1.y),
                                                   make_float2(t1.z, t1.z)),
                                  __float_as_uint(t1.w) ^ 0x8000u);
          if (!(l0 * lb_f - slack > upper)) my_list[cnt++] = (uint8_t)cc;
          if (cd > cc && !(l1 * lb_f - slack > upper)) my_list[cnt++] = (uint8_t)cd;
        }
      };
      bound_range(lo2, min(hi2, cs + kFp4WinLo - 1));
      bound_range(max(lo2, cs + kFp4WinHi + 1), hi2);
    }
    // the block's magnitudes for the lanes that score its pairs
#pragma unroll
    for (int p = 0; p < B / 4; ++p)
      *reinterpret_cast<float4*>(&S.a[lane][4 * p]) =
          make_float4(a[2 * p].x, a[2 * p].y, a[2 * p + 1].x, a[2 * p + 1].y);
    int off = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, off, o);
      if (lane >= o) off += v;
    }
    const int total = __shfl_sync(kFull, off, 31);
    off -= cnt;
    S.off[lane] = off;
    __syncwarp();
    for (int wbase = 0; wbase < total; wbase += kFp4Queue) {
      const int wend = min(total, wbase + kFp4Queue);
      for (int g = wbase + lane; g < wend; g += 32) {
        int o = 0;                                      // the lane whose pairs include g
#pragma unroll
        for (int step = 16; step > 0; step >>= 1)
          if (S.off[o + step] <= g) o += step;
        const int cc = S.list[o * kFp4List + (g - S.off[o])];
        float2 ao[B / 2];
#pragma unroll
        for (int p = 0; p < B / 4; ++p) {
          const float4 v = *reinterpret_cast<const float4*>(&S.a[o][4 * p]);
          ao[2 * p] = make_float2(v.x, v.y);
          ao[2 * p + 1] = make_float2(v.z, v.w);
        }
        S.res[g - wbase] = fp4_eval<B, HOPT>(ao, c, tab[cc]);
      }
      __syncwarp();
      const int j1 = min(off + cnt, wend);
      for (int j = max(off, wbase); j < j1; ++j) track(S.res[j - wbase], my_list[j - off], m1, m2, i1);
      __syncwarp();
    }
    if (valid) {
      const float upper = fmaf(m1, hi_f, slack);
      const int64_t b = row * kb + jb;
      if (!(m2 * lo_f - slack > upper)) {
        // A second candidate may tie or beat the float32 winner: flag the block (bit 7 of
        // the scale byte) for the exact pass, k_fp4_fixup.
        P.scales[b] = (uint8_t)(0x80 | i1);
      } else {
        const float4 t = tab[i1];
        fp4_emit<B>(a, sgn, t, false, P.codes + row * (P.k / 2) + jb * (B / 2));
        P.scales[b] = (uint8_t)i1;
        if (want_err) {
          if constexpr (HOPT) {
            fp4_block_sums<B, true>(a, c, t, acc);
          } else if (err_h) {
            float2 ce[B / 2];
            load_h<B>(P.h_err + jb * B, ce);
            fp4_block_sums<B, true>(a, ce, t, acc);
          } else {
            fp4_block_sums<B, false>(a, c, t, acc);
          }
        }
      }
    }
    __syncwarp();                                       // S is refilled by the next tile
  }
  if (want_err) cta_sums(acc, P.err_partial, blockIdx.x);
}

// Exact pass over the blocks the search flagged. Each warp scans 32 scale bytes at a time;
// every flagged block is handled by the whole warp: lanes evaluate candidates lo + lane +
// 32 t in float32, the warp minimum bounds the band, candidates inside it are re-scored in
// double in the definition's order, and the warp arg-min (lowest code on equal doubles)
// is emitted. With P.err_partial set, the emitted blocks' error sums go into this CTA's
// partial (after the search CTAs' partials).
template <int B, bool BF16, bool HOPT>
__global__ void __launch_bounds__(kThreads)
k_fp4_fixup(Fp4Params P, Fp4Table T) {
  __shared__ float4 tab[128];
  for (int i = threadIdx.x; i < 128; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t kb = P.k / B, nblocks = P.n * kb;
  const int elsz = BF16 ? 2 : 4;
  const float gam = (float)(B + 8) * 5.9604645e-8f;
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
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
      const int c0 = e4m3_rn_code(__fdiv_rn(block_amax<B>(a), 6.0f));
      int lo = 1, hi = 126;
      if (P.window >= 0) {
        lo = max(1, c0 - P.window);
        hi = min(126, c0 + P.window);
        if (c0 == 0) { lo = 1; hi = max(1, P.window); }
      }
      float ef[4];
      float mloc = __int_as_float(0x7f800000);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int cc = lo + lane + 32 * t;
        ef[t] = cc <= hi ? fp4_eval<B, HOPT>(a, c, tab[cc]) : __int_as_float(0x7f800000);
        mloc = fminf(mloc, ef[t]);
      }
      const float m1 = warp_min(mloc);
      const float upper = fmaf(m1, hi_f, slack);
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bi = 0x7fffffff;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int cc = lo + lane + 32 * t;
        if (cc <= hi && !(ef[t] * lo_f - slack > upper)) {
          const double ed = fp4_exact<B, HOPT>(a, c, tab[cc]);
          if (ed < best || (ed == best && cc < bi)) { best = ed; bi = cc; }
        }
      }
      warp_argmin(best, bi);
      if (lane == 0) {
        fp4_emit<B>(a, sgn, tab[bi], false, P.codes + row * (P.k / 2) + jb * (B / 2));
        P.scales[b] = (uint8_t)bi;
        if (P.err_partial) {
          if constexpr (HOPT) {
            fp4_block_sums<B, true>(a, c, tab[bi], acc);
          } else if (P.h_err) {
            float2 ce[B / 2];
            load_h<B>(P.h_err + jb * B, ce);
            fp4_block_sums<B, true>(a, ce, tab[bi], acc);
          } else {
            fp4_block_sums<B, false>(a, c, tab[bi], acc);
          }
        }
      }
    }
  }
  if (P.err_partial) cta_sums(acc, P.err_partial, P.fix_slot0 + blockIdx.x);
}

// ---------------------------------------------------------------------------------------
// INT8 with E4M3 stored amax. G = B / 32 lanes per block, each lane owns 32 consecutive
// elements; a warp holds 32 / G blocks of one column block in consecutive rows, so every
// group reads the same 32 h values per lane.
//
// Ranking without a division. Per candidate the lanes form x = fl(|w| * r) with
// r = fl32(1/s) and q~ = RNE(min(x, 127)) (rounding by adding 2^23, which for
// 0 <= x < 2^23 leaves an integer, ties to even), then fl32(q~ s) as one fma
// (q~ + 2^23) s - 2^23 s, exact because 2^23 s is. x is within 2.0001 u |w|/s of
// the real quotient (u = 2^-24) and the definition's fl32(|w|/s) within u |w|/s, so q~
// can differ from the definition's q (by one) only when |w|/s lies within 2.0001 u |w|/s
// of a half-integer k + 1/2; the two dequantised values then sit on either side of |w|
// at distance ~s/2 and their squared errors differ by at most 10 u s |w| (4 u s |w| from
// the real identity, 6 u s |w| from the float32 rounding of q s). So every candidate's
// float32 error brackets the definition's double error within gamma (float32 rounding,
// at most 24 roundings deep) plus delta = 16 u s sum_j c_j |w_j|. A block whose winner
// is not separated from every other candidate by these brackets is flagged (scale byte
// bit 7) and re-scored exactly by k_int8_fixup.
// ---------------------------------------------------------------------------------------
struct Int8Params {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* h;
  int window;
  int8_t* codes;
  uint8_t* scales;
};

// Per candidate code: {s = fl32(E4M3 / 127), -fl32(1/s), -2^23 s, 0}; host-computed.
struct Int8Table {
  float4 c[128];
};

// Float32 error of one candidate over a lane's 32 elements, from the negated magnitudes
// na = -|w| (d = fl32(q s) - |w| has the magnitude of the definition's difference).
template <bool HOPT>
__device__ __forceinline__ float int8_eval(const float2 (&na)[16], const float2 (&c)[16],
                                           float4 t) {
  const float2 nr = make_float2(t.y, t.y), s2 = make_float2(t.x, t.x);
  const float2 nms = make_float2(t.z, t.z), mag = make_float2(8388608.f, 8388608.f);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const float2 x = __fmul2_rn(na[p], nr);
    const float2 xt = __fadd2_rn(make_float2(fminf(x.x, 127.f), fminf(x.y, 127.f)), mag);
    const float2 d = __fadd2_rn(__ffma2_rn(xt, s2, nms), na[p]);
    float2& acc = (p & 1) ? acc1 : acc0;
    if constexpr (HOPT) acc = __ffma2_rn(__fmul2_rn(c[p], d), d, acc);
    else acc = __ffma2_rn(d, d, acc);
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// The definition's code magnitude: min(RNE(fl32(|w| / s)), 127).
__device__ __forceinline__ int int8_code(float a, float s) {
  return (int)fminf(rintf(__fdiv_rn(a, s)), 127.0f);
}

__device__ __forceinline__ void int8_window(int c0, int window, int& lo, int& hi) {
  lo = 1;
  hi = 126;
  if (window >= 0) {
    lo = max(1, c0 - window);
    hi = min(126, c0 + window);
    if (c0 == 0) hi = max(1, window);
  }
}

template <int B, bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads, 2)
k_int8_search(Int8Params P, Int8Table T) {
  constexpr int G = B / 32, RPW = 32 / G;
  __shared__ float4 tab[128];
  for (int i = threadIdx.x; i < 128; i += kThreads) tab[i] = T.c[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, sub = lane % G, grp = lane / G;
  const int64_t kb = P.k / B, items = (P.n + RPW - 1) / RPW * kb;
  const int elsz = BF16 ? 2 : 4;
  const float gam = 40.0f * 5.9604645e-8f;
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;
  const float kdel = 16.0f * 5.9604645e-8f;
  const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
  for (int64_t it = gw; it < items; it += nw) {
    const int64_t rg = it / kb, jb = it - rg * kb;
    const int64_t row = rg * RPW + grp;
    const bool valid = row < P.n;
    const int64_t col = jb * B + sub * 32;
    float2 a[16], c[16];
    uint32_t sgn = 0;
    if (valid) {
      load_block<32, BF16>(P.W + row * P.ld_bytes + col * elsz, a, sgn);
    } else {
#pragma unroll
      for (int p = 0; p < 16; ++p) a[p] = make_float2(0.f, 0.f);
    }
    if constexpr (MODE == 2) load_h<32>(P.h + col, c);
    float amax = block_amax<32>(a);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const int c0 = e4m3_rn_code(amax);
    int best = c0;
    bool flag = false;
    if constexpr (MODE != 0) {
      int lo, hi;
      int8_window(c0, P.window, lo, hi);
      float Q = 0.f;
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        Q = (MODE == 2) ? fmaf(c[p].x, a[p].x, fmaf(c[p].y, a[p].y, Q)) : Q + (a[p].x + a[p].y);
        a[p] = make_float2(-a[p].x, -a[p].y);
      }
#pragma unroll
      for (int o = 1; o < G; o <<= 1) Q += __shfl_xor_sync(kFull, Q, o);
      const int span = P.window < 0 ? 126 : 2 * P.window + 1;
      const float inf = __int_as_float(0x7f800000);
      float m1 = inf, hi1 = inf, l1 = inf, l2 = inf;
      int i1 = lo, j1 = -1;
      auto visit = [&](int cc, float e, float s) {
        const float del = fmaf(kdel * s, Q, slack);
        const float elo = fmaf(e, lo_f, -del);
        if (e < m1) { m1 = e; i1 = cc; hi1 = fmaf(e, hi_f, del); }
        if (elo < l1) { l2 = l1; l1 = elo; j1 = cc; }
        else if (elo < l2) l2 = elo;
      };
      // Seed: the naive code (clipped to the range), evaluated first.
      const int cs = min(max(c0, lo), hi);
      {
        float e = int8_eval<MODE == 2>(a, c, tab[cs]);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) e += __shfl_xor_sync(kFull, e, o);
        visit(cs, e, tab[cs].x);
      }
      // Saturation cut: for s <= a_j / 127 every level is at most 127 s, so the definition's
      // error is at least c_j (a_j - 127 s)^2, which exceeds the seed's upper bound hi1 for
      // every s below (a_j - sqrt(hi1 / c_j)) / 127; such candidates can neither win nor tie.
      // The warp starts at the lowest cut among its blocks (candidate loop stays uniform).
      float s_cut = 0.f;
      {
        const float sqt = sqrtf(hi1) * 1.00001f;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float cx = MODE == 2 ? c[p].x : 1.f, cy = MODE == 2 ? c[p].y : 1.f;
          if (cx > 0.f) s_cut = fmaxf(s_cut, (-a[p].x - sqt * rsqrtf(cx)) * (1.0f / 127.0f) * 0.99999f);
          if (cy > 0.f) s_cut = fmaxf(s_cut, (-a[p].y - sqt * rsqrtf(cy)) * (1.0f / 127.0f) * 0.99999f);
        }
#pragma unroll
        for (int o = 1; o < G; o <<= 1) s_cut = fmaxf(s_cut, __shfl_xor_sync(kFull, s_cut, o));
      }
      int cl = lo;
      while (cl < hi && tab[cl].x < s_cut) ++cl;
      const int t0 = __reduce_min_sync(kFull, (unsigned)(cl - lo));
      for (int t = t0; t < span; ++t) {
        const int cc = lo + t;
        const float4 tb = tab[min(cc, 126)];
        float e = int8_eval<MODE == 2>(a, c, tb);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) e += __shfl_xor_sync(kFull, e, o);
        if (cc <= hi && cc != cs) visit(cc, e, tb.x);
      }
      flag = !((j1 == i1 ? l2 : l1) > hi1);
      best = i1;
#pragma unroll
      for (int p = 0; p < 16; ++p) a[p] = make_float2(-a[p].x, -a[p].y);
    }
    if (valid) {
      const float s = tab[best].x;
      uint32_t pk[8];
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        int q0 = best ? int8_code(a[p].x, s) : 0, q1 = best ? int8_code(a[p].y, s) : 0;
        if ((sgn >> (2 * p)) & 1u) q0 = -q0;
        if ((sgn >> (2 * p + 1)) & 1u) q1 = -q1;
        const uint32_t v = ((uint32_t)q0 & 0xffu) | (((uint32_t)q1 & 0xffu) << 8);
        if (p & 1) pk[p >> 1] |= v << 16;
        else pk[p >> 1] = v;
      }
      uint4* out = reinterpret_cast<uint4*>(P.codes + row * P.k + col);
      out[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      out[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      if (sub == 0) P.scales[row * kb + jb] = (uint8_t)(best | (flag ? 0x80 : 0));
    }
  }
}

// Exact pass over the INT8 blocks the search flagged. Each warp scans 32 scale bytes at a
// time; a flagged block is staged in the warp's shared memory, lane l scores candidates
// lo + l + 32 t in double in the definition's order (e += c_j * (d * d) over j), the warp
// arg-min (lowest code on equal doubles) wins, and the warp rewrites the block's codes.
template <int B, bool BF16, bool HOPT>
__global__ void __launch_bounds__(kThreads)
k_int8_fixup(Int8Params P, Int8Table T) {
  constexpr int NE = B / 32;
  __shared__ float tab[128];
  __shared__ float sa[kThreads / 32][B];
  __shared__ float sc[kThreads / 32][HOPT ? B : 1];
  for (int i = threadIdx.x; i < 128; i += kThreads) tab[i] = T.c[i].x;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t kb = P.k / B, nblocks = P.n * kb;
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
      const char* rp = P.W + row * P.ld_bytes + jb * B * (BF16 ? 2 : 4);
      uint32_t sgn = 0;
      float amax = 0.f;
#pragma unroll
      for (int t = 0; t < NE; ++t) {
        const int j = lane + 32 * t;
        uint32_t bits;
        if constexpr (BF16) bits = (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(rp) + j) << 16;
        else bits = __float_as_uint(__ldg(reinterpret_cast<const float*>(rp) + j));
        sgn |= (bits >> 31) << t;
        const float a = __uint_as_float(bits & 0x7fffffffu);
        sa[wid][j] = a;
        if constexpr (HOPT) sc[wid][j] = __ldg(P.h + jb * B + j);
        amax = fmaxf(amax, a);
      }
      __syncwarp();
      int lo, hi;
      int8_window(e4m3_rn_code(warp_max(amax)), P.window, lo, hi);
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bi = 0x7fffffff;
      for (int cc = lo + lane; cc <= hi; cc += 32) {
        const float s = tab[cc];
        double e = 0.0;
        for (int j = 0; j < B; ++j) {
          const float a = sa[wid][j];
          const float wq = __fmul_rn((float)int8_code(a, s), s);
          const double d = (double)a - (double)wq;
          const double cj = HOPT ? (double)sc[wid][j] : 1.0;
          e = __dadd_rn(e, __dmul_rn(cj, __dmul_rn(d, d)));
        }
        if (e < best) { best = e; bi = cc; }
      }
      warp_argmin(best, bi);
      if (bi > 126) bi = lo;  // every candidate NaN (non-finite input): keep the first
      const float s = tab[bi];
      int8_t* out = P.codes + row * P.k + jb * B;
#pragma unroll
      for (int t = 0; t < NE; ++t) {
        const int j = lane + 32 * t;
        const int q = int8_code(sa[wid][j], s);
        out[j] = (int8_t)(((sgn >> t) & 1u) ? -q : q);
      }
      if (lane == 0) P.scales[b] = (uint8_t)bi;
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------------------
// E4M3 elements, one float32 scale per 64 x 64 tile searched on a logarithmic grid.
// One CTA (256 threads) per tile; thread t owns row t/4, columns 16 (t%4) .. +16.
//
// Ranking without a division: per candidate s the threads form x = fl(|w| * fl32(1/s))
// and its E4M3 code, in float32 with packed f32x2 math. x lies within 2.0001 u |w|/s of
// the real quotient (u = 2^-24) and the definition's fl32(|w|/s) within u |w|/s, so the
// two codes can differ only when |w|/s is that close to a rounding midpoint m of E4M3;
// the neighbouring values v1 < m < v2 then give squared errors that differ by
// 2 s^2 (v2 - v1) |w/s - m| <= 8 u w^2 (spacing at most twice the value), plus at most
// 2 u w^2 from rounding s v in float32. So each candidate's float32 error brackets the
// definition's within gamma (float32 rounding) plus delta = 17 u sum_j c_j w_j^2. Every
// candidate whose bracket meets the winner's is re-scored in double as the definition
// writes it (d = |w| - fl32(s v) in double, e += c (d d)), in a fixed parallel order, and
// the smallest double error wins (lowest grid index on equal values).
// ---------------------------------------------------------------------------------------
struct TileParams {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* h;
  int points;
  uint8_t* codes;
  float* scales;
};
struct LogGrid {
  float g[256];
};

constexpr int kTile = 64;
constexpr int kTileChunk = 16;  // candidates per register pass

// E4M3 values of the codes of two non-negative floats (RNE, saturating), as float32.
__device__ __forceinline__ float2 e4m3x2_round_values(float x0, float x1) {
  float v0, v1;
  asm("{\n\t.reg .b16 q, h0, h1;\n\t.reg .b32 v;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 q, %3, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 v, q;\n\t"
      "mov.b32 {h0, h1}, v;\n\t"
      "cvt.f32.f16 %0, h0;\n\t"
      "cvt.f32.f16 %1, h1;\n\t}"
      : "=f"(v0), "=f"(v1)
      : "f"(x0), "f"(x1));
  return make_float2(v0, v1);
}

// Float32 error of one candidate over a thread's 16 elements; na = -|w|,
// t = {s, -fl32(1/s)}.
template <bool HOPT>
__device__ __forceinline__ float tile_eval(const float2 (&na)[8], const float2 (&c)[8],
                                           float2 t) {
  const float2 nr = make_float2(t.y, t.y), s2 = make_float2(t.x, t.x);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 x = __fmul2_rn(na[p], nr);
    const float2 v = e4m3x2_round_values(x.x, x.y);
    const float2 d = __fadd2_rn(__fmul2_rn(v, s2), na[p]);
    float2& acc = (p & 1) ? acc1 : acc0;
    if constexpr (HOPT) acc = __ffma2_rn(__fmul2_rn(c[p], d), d, acc);
    else acc = __ffma2_rn(d, d, acc);
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// The definition's dequantised magnitude fl32(s * E4M3(RNE(fl32(a / s)))).
__device__ __forceinline__ float e4m3_elem_wq(float a, float s) {
  const float2 v = e4m3x2_round_values(__fdiv_rn(a, s), 0.0f);
  return __fmul_rn(s, v.x);
}

template <bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads)
k_e4m3_tile(TileParams P, LogGrid G) {
  constexpr int kWarps = kThreads / 32;
  __shared__ float g[256];
  __shared__ float2 cand[256];
  __shared__ float errf[256];
  __shared__ unsigned char band[256];
  __shared__ float red[kWarps][kTileChunk];
  __shared__ double redd[kWarps];
  __shared__ float red_max[kWarps], red_a[kWarps];
  __shared__ int pick, nband;
  for (int i = threadIdx.x; i < P.points; i += kThreads) g[i] = G.g[i];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int r = threadIdx.x >> 2, c0 = (threadIdx.x & 3) * 16;
  const int64_t tn = P.n / kTile, tk = P.k / kTile, ntiles = tn * tk;
  const int elsz = BF16 ? 2 : 4;
  const float inf = __int_as_float(0x7f800000);
  const float gam = 40.0f * 5.9604645e-8f;
  const float lo_f = 1.0f - gam, hi_f = 1.0f + 2.0f * gam;
  const float slack = 7.3468396e-40f;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t ti = tile / tk, tj = tile - ti * tk;
    const int64_t row = ti * kTile + r, col = tj * kTile + c0;
    float2 na[8], c[8];
    uint32_t sgn;
    load_block<16, BF16>(P.W + row * P.ld_bytes + col * elsz, na, sgn);
    if constexpr (MODE == 2) load_h<16>(P.h + col, c);
    else {
#pragma unroll
      for (int p = 0; p < 8; ++p) c[p] = make_float2(1.f, 1.f);
    }
    float am = block_amax<16>(na), aw = 0.f;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      aw = fmaf(c[p].x * na[p].x, na[p].x, fmaf(c[p].y * na[p].y, na[p].y, aw));
      na[p] = make_float2(-na[p].x, -na[p].y);
    }
    am = warp_max(am);
    aw = warp_sum(aw);
    if (lane == 0) { red_max[wid] = am; red_a[wid] = aw; }
    __syncthreads();
    am = red_max[0];
    aw = red_a[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) { am = fmaxf(am, red_max[w]); aw += red_a[w]; }
    const float base = __fdiv_rn(am, 448.0f);
    float s = base;
    if (MODE != 0 && base > 0.0f) {
      // A candidate below 2^-100 would push 1/s, x or s v out of the normal float32
      // range the bracket assumes: it gets the bracket [0, inf) (always re-scored).
      for (int p = threadIdx.x; p < P.points; p += kThreads) {
        const float sp = __fmul_rn(base, g[p]);
        const bool fast = sp >= 0x1p-100f;
        cand[p] = make_float2(sp, fast ? -__frcp_rn(sp) : 0.0f);
        band[p] = sp > 0.0f && !fast;
      }
      __syncthreads();
      const float del = fmaf(17.0f * 5.9604645e-8f, aw, slack);
      for (int p0 = 0; p0 < P.points; p0 += kTileChunk) {
        float part[kTileChunk];
#pragma unroll
        for (int u = 0; u < kTileChunk; ++u) {
          const int p = p0 + u;
          part[u] = 0.f;
          if (p < P.points && cand[p].y != 0.0f) part[u] = tile_eval<MODE == 2>(na, c, cand[p]);
        }
#pragma unroll
        for (int u = 0; u < kTileChunk; ++u) {
          const float v = warp_sum(part[u]);
          if (lane == 0) red[wid][u] = v;
        }
        __syncthreads();
        if (threadIdx.x < kTileChunk && p0 + (int)threadIdx.x < P.points) {
          const int p = p0 + threadIdx.x;
          float e = red[0][threadIdx.x];
#pragma unroll
          for (int w = 1; w < kWarps; ++w) e += red[w][threadIdx.x];
          errf[p] = cand[p].y != 0.0f ? e : inf;
        }
        __syncthreads();
      }
      if (wid == 0) {
        float v = inf;
        int vi = 0x7fffffff;
        for (int p = lane; p < P.points; p += 32)
          if (errf[p] < v) { v = errf[p]; vi = p; }
        warp_argmin(v, vi);
        const float hi1 = fmaf(v, hi_f, del);
        int cnt = 0;
        for (int p = lane; p < P.points; p += 32) {
          const bool in = band[p] || (p != vi && errf[p] < inf &&
                                       !(fmaf(errf[p], lo_f, -del) > hi1));
          band[p] = in;
          cnt += in;
        }
        cnt = __reduce_add_sync(kFull, cnt);
        if (lane == 0) { pick = v < inf ? vi : -1; nband = cnt; }
      }
      __syncthreads();
      if (nband > 0) {
        // Re-score the winner and every candidate in its band in double.
        const int first = pick;
        double bestd = __longlong_as_double(0x7ff0000000000000ll);
        int bi = first;
        for (int p = 0; p < P.points; ++p) {
          if (p != first && !band[p]) continue;
          const float sp = cand[p].x;
          double e = 0.0;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const double d0 = (double)(-na[q].x) - (double)e4m3_elem_wq(-na[q].x, sp);
            const double d1 = (double)(-na[q].y) - (double)e4m3_elem_wq(-na[q].y, sp);
            e += (double)c[q].x * (d0 * d0);
            e += (double)c[q].y * (d1 * d1);
          }
          e = warp_sum(e);
          if (lane == 0) redd[wid] = e;
          __syncthreads();
          e = redd[0];
#pragma unroll
          for (int w = 1; w < kWarps; ++w) e += redd[w];
          if (e < bestd || (e == bestd && p < bi)) { bestd = e; bi = p; }
          __syncthreads();
        }
        if (threadIdx.x == 0) pick = bi;
        __syncthreads();
      }
      s = pick >= 0 ? cand[pick].x : 0.0f;
    }
    // emit 16 bytes per thread
    uint32_t wds[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float a0 = -na[j / 2].x, a1 = -na[j / 2].y;
      uint32_t pair = 0;
      if (s > 0.0f) pair = e4m3x2_rn(__fdiv_rn(a0, s), __fdiv_rn(a1, s)) & 0x7f7fu;
      pair |= ((sgn >> j) & 1u) << 7;
      pair |= ((sgn >> (j + 1)) & 1u) << 15;
      wds[j / 4] |= pair << (8 * (j % 4));
    }
    *reinterpret_cast<uint4*>(P.codes + row * P.k + col) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
    if (threadIdx.x == 0) P.scales[tile] = s;
    __syncthreads();
  }
}

// Element projection at one fixed scale (verification entry point): the magnitude code
// that the search kernels produce for |w| at that scale.
__global__ void k_project(const float* __restrict__ w, int64_t count, int fmt, float scale,
                          float rhi, float rlo, uint8_t* __restrict__ q) {
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * kThreads) {
    const float a = fabsf(w[i]);
    uint32_t code;
    if (fmt == 0 || fmt == 3) {
      // the split-reciprocal quotient of the search kernels (exact for every scale grid)
      const float2 x = fp4_quot(make_float2(a, 0.f), make_float2(rhi, rhi), make_float2(rlo, rlo));
      code = fmt == 0 ? (e2m1x2_rn(x.x, 0.f) & 7u) : (uint32_t)fminf(rintf(x.x), 7.0f);
    } else if (fmt == 1) {
      code = (uint32_t)int8_code(a, __fdiv_rn(scale, 127.0f));
    } else {
      code = e4m3x2_rn(__fdiv_rn(a, scale), 0.f) & 0x7fu;
    }
    q[i] = (uint8_t)code;
  }
}

Fp4Table make_fp4_table() {
  Fp4Table t;
  for (int c = 0; c < 128; ++c) {
    double v;
    if (c == 0 || c == 127) {
      t.c[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const int e = c >> 3, m = c & 7;
    v = e == 0 ? (double)m / 8.0 * (1.0 / 64.0) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    const double r = 1.0 / v;
    const float rhi = (float)r;
    const float rlo = (float)(r - (double)rhi);
    const __half sh = __double2half(v);  // exact: every E4M3 value is an fp16 value
    const uint32_t sbits = (uint32_t)__half_as_ushort(sh);
    float sfl;
    memcpy(&sfl, &sbits, sizeof sfl);
    t.c[c] = make_float4((float)v, rhi, rlo, sfl);
  }
  for (int m = 0; m < 8; ++m) {
    const double q = 8.0 / (8.0 + m);
    const float qh = (float)q;
    t.sig[m] = make_float2(qh, (float)(q - (double)qh));
  }
  return t;
}

int grid_for(int64_t work_threads) {
  const int64_t want = (work_threads + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sm_count() * 64;
  return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

// Grids of the NVFP4 search and its exact pass (fixed by the shape and the device's SM
// count, so the order of the fused error sums is too).
template <int B>
void fp4_grids(int64_t n, int64_t k, int ctas_per_sm, int& gs, int& gf) {
  const int64_t ntiles = (n + 31) / 32 * (k / B);
  const int fit = B == 16 ? 3 : 2;                 // resident CTAs per SM (registers)
  const int64_t cap = (int64_t)sm_count() * (ctas_per_sm > 0 && ctas_per_sm < fit ? ctas_per_sm : fit);
  const int64_t want = (ntiles + kThreads / 32 - 1) / (kThreads / 32);
  gs = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  const int64_t fwant = (n * (k / B) + 32 * 8 - 1) / (32 * 8);   // one 32-block tile per warp
  gf = (int)(fwant < 1 ? 1 : (fwant < (int64_t)sm_count() * 8 ? fwant : (int64_t)sm_count() * 8));
}

template <int B, bool BF16>
cudaError_t fp4_dispatch(const QuantArgs& a, cudaStream_t st) {
  static const Fp4Table T = make_fp4_table();
  Fp4Params P{(const char*)a.W, a.n, a.k, a.ld * (BF16 ? 2 : 4), a.h, a.window,
              (uint8_t*)a.codes, (uint8_t*)a.scales, a.err_partial, a.h_err, 0};
  const int64_t nblocks = a.n * (a.k / B);
  if (a.mode == 0) {
    k_fp4_naive<B, BF16><<<grid_for(nblocks), kThreads, 0, st>>>(P, T);
    return cudaGetLastError();
  }
  int gs, gf;
  fp4_grids<B>(a.n, a.k, a.ctas_per_sm, gs, gf);
  P.fix_slot0 = gs;
  const size_t smem = fp4_search_smem<B>();
  const void* kern = a.mode == 1 ? (const void*)k_fp4_search<B, BF16, false>
                                 : (const void*)k_fp4_search<B, BF16, true>;
  cudaError_t e = ensure_dynamic_smem(kern, (int)smem);
  if (e != cudaSuccess) return e;
  if (a.mode == 1) k_fp4_search<B, BF16, false><<<gs, kThreads, smem, st>>>(P, T);
  else k_fp4_search<B, BF16, true><<<gs, kThreads, smem, st>>>(P, T);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.mode == 1) k_fp4_fixup<B, BF16, false><<<gf, kThreads, 0, st>>>(P, T);
  else k_fp4_fixup<B, BF16, true><<<gf, kThreads, 0, st>>>(P, T);
  e = cudaGetLastError();
  if (e != cudaSuccess || !a.err_partial) return e;
  return launch_error_final(a.err_partial, gs + gf, a.err_sums, st);
}


Int8Table make_int8_table() {
  Int8Table t;
  for (int c = 0; c < 128; ++c) {
    if (c == 0 || c == 127) {
      t.c[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const int e = c >> 3, m = c & 7;
    const float v = (float)(e == 0 ? (double)m / 8.0 * (1.0 / 64.0)
                                   : (1.0 + m / 8.0) * ldexp(1.0, e - 7));  // exact
    volatile float s = v / 127.0f;  // IEEE float32 division, as on the device
    const float sf = s;
    volatile float r = 1.0f / sf;
    t.c[c] = make_float4(sf, -(float)r, -8388608.0f * sf, 0.f);
  }
  return t;
}

template <int B, bool BF16>
cudaError_t int8_dispatch(const QuantArgs& a, cudaStream_t st) {
  static const Int8Table T = make_int8_table();
  Int8Params P{(const char*)a.W, a.n, a.k, a.ld * (BF16 ? 2 : 4), a.h, a.window,
               (int8_t*)a.codes, (uint8_t*)a.scales};
  constexpr int RPW = 32 / (B / 32);
  const int64_t items = (a.n + RPW - 1) / RPW * (a.k / B);
  const int64_t want = (items * 32 + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sm_count() * 2;
  const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  if (a.mode == 0) {
    k_int8_search<B, BF16, 0><<<grid, kThreads, 0, st>>>(P, T);
    return cudaGetLastError();
  }
  if (a.mode == 1) k_int8_search<B, BF16, 1><<<grid, kThreads, 0, st>>>(P, T);
  else k_int8_search<B, BF16, 2><<<grid, kThreads, 0, st>>>(P, T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nblocks = a.n * (a.k / B);
  const int64_t fwant = (nblocks + 32 * 8 - 1) / (32 * 8);
  const int fgrid = (int)(fwant < (int64_t)sm_count() * 8 ? fwant : (int64_t)sm_count() * 8);
  if (a.mode == 1) k_int8_fixup<B, BF16, false><<<fgrid, kThreads, 0, st>>>(P, T);
  else k_int8_fixup<B, BF16, true><<<fgrid, kThreads, 0, st>>>(P, T);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t tile_dispatch(const QuantArgs& a, cudaStream_t st) {
  TileParams P{(const char*)a.W, a.n, a.k, a.ld * (BF16 ? 2 : 4), a.h, a.log_points,
               (uint8_t*)a.codes, (float*)a.scales};
  LogGrid G;
  for (int i = 0; i < 256; ++i) G.g[i] = i < a.log_points ? a.log_grid[i] : 0.f;
  const int64_t ntiles = (a.n / kTile) * (a.k / kTile);
  int64_t grid = ntiles;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (grid > cap) grid = cap;
  if (a.mode == 0) k_e4m3_tile<BF16, 0><<<(unsigned)grid, kThreads, 0, st>>>(P, G);
  else if (a.mode == 1) k_e4m3_tile<BF16, 1><<<(unsigned)grid, kThreads, 0, st>>>(P, G);
  else k_e4m3_tile<BF16, 2><<<(unsigned)grid, kThreads, 0, st>>>(P, G);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_project(const float* w, int64_t count, int fmt, float scale, uint8_t* q,
                           cudaStream_t st) {
  float rhi = 0.f, rlo = 0.f;
  if (fmt == 0 || fmt == 3) {
    const double r = 1.0 / (double)scale;
    rhi = (float)r;
    rlo = (float)(r - (double)rhi);
  }
  int64_t grid = (count + kThreads - 1) / kThreads;
  if (grid > 4096) grid = 4096;
  k_project<<<(unsigned)grid, kThreads, 0, st>>>(w, count, fmt, scale, rhi, rlo, q);
  return cudaGetLastError();
}

int fp4_error_parts(int64_t n, int64_t k, int B, int ctas_per_sm) {
  int gs, gf;
  if (B == 16) fp4_grids<16>(n, k, ctas_per_sm, gs, gf);
  else fp4_grids<32>(n, k, ctas_per_sm, gs, gf);
  return gs + gf;
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == 1;
  if (a.fmt == 3 || (a.fmt == 0 && a.scale_fmt != 0)) return launch_quantize_grid(a, st);
  if (a.fmt == 0) {
    if (a.block == 16) return bf ? fp4_dispatch<16, true>(a, st) : fp4_dispatch<16, false>(a, st);
    return bf ? fp4_dispatch<32, true>(a, st) : fp4_dispatch<32, false>(a, st);
  }
  if (a.fmt == 1) {
    switch (a.block) {
      case 32: return bf ? int8_dispatch<32, true>(a, st) : int8_dispatch<32, false>(a, st);
      case 64: return bf ? int8_dispatch<64, true>(a, st) : int8_dispatch<64, false>(a, st);
      case 128: return bf ? int8_dispatch<128, true>(a, st) : int8_dispatch<128, false>(a, st);
      default: return bf ? int8_dispatch<256, true>(a, st) : int8_dispatch<256, false>(a, st);
    }
  }
  return bf ? tile_dispatch<true>(a, st) : tile_dispatch<false>(a, st);
}

}  // namespace mxq
