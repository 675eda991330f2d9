// mxq_error.cu -- dequantisation and weight-error metrics.
//
// Dequantised value (the microscaling reconstruction x^ = s q, "Is Finer Better? The
// Limits of Microscaling Formats in LLMs", sec. 2.1):
//   NVFP4  E4M3(scale) * E2M1(code)                (exact in float32 and in fp16)
//   E2M1 on the UE4M4 / UE5M3 / UE8M0 grids: grid(scale) * E2M1(code)   (exact)
//   INT4   grid(scale) * code, code the signed nibble (exact)
//   INT8   fl32(q * fl32(E4M3(scale) / 127))
//   E4M3   fl32(tile scale * E4M3(code))
// Metrics (qwantize "Results": weight error ||Q(W) - W||_F / ||W||_F; the h-weighted
// error of "quantization_algorithms.txt", sec. 1): the four sums sum d^2, sum w^2,
// sum h d^2, sum h w^2. HBM-bound: each thread decodes 16 consecutive elements of a row
// with the hardware E2M1 / E4M3 conversions; float32 partials over those 16 (packed f32x2
// math), double from there on; the per-CTA partials are combined by a one-CTA kernel in a
// fixed order (deterministic).
#include "mxq_common.cuh"
#include "mxq_grids.h"
#include "mxq_internal.h"

#include <cuda_fp16.h>

namespace mxq {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxErrCtas = 148 * 8;

// Decoder variants: 0 E2M1 on E4M3 scales, 1 INT8, 2 E4M3 tiles, 3 INT4 on a scale table,
// 4 E2M1 on a scale table.
enum { kDecFp4 = 0, kDecInt8 = 1, kDecTile = 2, kDecInt4 = 3, kDecFp4Tab = 4 };

// Scale-code values of a grid (NaN for the codes it does not define); staged in shared
// memory by the kernels that decode through a table.
struct ScaleTab {
  float v[256];
};

ScaleTab make_scale_tab(int sfmt) {
  ScaleTab t;
  const GridInfo g = grid_info(sfmt);
  for (int c = 0; c < 256; ++c) t.v[c] = c < g.ncodes ? (float)grid_value(sfmt, c) : __builtin_nanf("");
  return t;
}

const ScaleTab& scale_tab(int sfmt) {
  static const ScaleTab tabs[4] = {make_scale_tab(0), make_scale_tab(1), make_scale_tab(2),
                                   make_scale_tab(3)};
  return tabs[sfmt];
}

int decoder_of(const DecodeArgs& d) {
  if (d.fmt == 3) return kDecInt4;
  if (d.fmt == 0 && d.scale_fmt != kScaleE4M3) return kDecFp4Tab;
  return d.fmt;
}

__device__ __forceinline__ float2 h2f2(uint32_t h2) {
  return make_float2(__half2float(__ushort_as_half(lo16(h2))),
                     __half2float(__ushort_as_half(hi16(h2))));
}

// Decoded (w^) values of the 16 elements starting at (row, col), as 8 float pairs.
// stab: the scale table in shared memory (decoders 3 and 4).
template <int FMT>
__device__ __forceinline__ void decode16(const DecodeArgs& d, int64_t row, int64_t col,
                                         float2 (&v)[8], const float* stab) {
  if constexpr (FMT == kDecFp4Tab || FMT == kDecInt4) {
    const uint8_t* cp = (const uint8_t*)d.codes + row * (d.k / 2) + col / 2;
    const uint2 cw = *reinterpret_cast<const uint2*>(cp);
    const float s = stab[((const uint8_t*)d.scales)[row * (d.k / d.block) + col / d.block]];
    const float2 s2 = make_float2(s, s);
    const uint32_t w2[2] = {cw.x, cw.y};
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t byte = (w2[p / 4] >> (8 * (p % 4))) & 0xffu;
      if constexpr (FMT == kDecFp4Tab) {
        v[p] = __fmul2_rn(h2f2(e2m1x2_to_f16x2(byte)), s2);   // exact products
      } else {
        const int q0 = (int)(byte << 28) >> 28, q1 = (int)(byte << 24) >> 28;  // sign-extend
        v[p] = __fmul2_rn(make_float2((float)q0, (float)q1), s2);
      }
    }
  } else if constexpr (FMT == 0) {
    const uint8_t* cp = (const uint8_t*)d.codes + row * (d.k / 2) + col / 2;
    const uint2 cw = *reinterpret_cast<const uint2*>(cp);
    const float s = e4m3_pos(((const uint8_t*)d.scales)[row * (d.k / d.block) + col / d.block]);
    const float2 s2 = make_float2(s, s);
    const uint32_t w2[2] = {cw.x, cw.y};
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t byte = (w2[p / 4] >> (8 * (p % 4))) & 0xffu;
      v[p] = __fmul2_rn(h2f2(e2m1x2_to_f16x2(byte)), s2);     // exact products
    }
  } else if constexpr (FMT == 1) {
    const int8_t* cp = (const int8_t*)d.codes + row * d.k + col;
    const uint4 cw = *reinterpret_cast<const uint4*>(cp);
    const int sc = ((const uint8_t*)d.scales)[row * (d.k / d.block) + col / d.block];
    const float s = __fdiv_rn(e4m3_pos(sc), 127.0f);
    const float2 s2 = make_float2(s, s);
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t wd = w4[p / 2] >> (16 * (p % 2));
      const float q0 = (float)(int8_t)(wd & 0xffu), q1 = (float)(int8_t)((wd >> 8) & 0xffu);
      v[p] = __fmul2_rn(make_float2(q0, q1), s2);
    }
  } else {
    const uint8_t* cp = (const uint8_t*)d.codes + row * d.k + col;
    const uint4 cw = *reinterpret_cast<const uint4*>(cp);
    const float s = ((const float*)d.scales)[(row / d.block) * (d.k / d.block) + col / d.block];
    const float2 s2 = make_float2(s, s);
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint16_t pair = (uint16_t)(w4[p / 2] >> (16 * (p % 2)));
      v[p] = __fmul2_rn(h2f2(e4m3x2_to_f16x2(pair)), s2);
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads)
k_dequant(DecodeArgs d, ScaleTab T, float* __restrict__ out) {
  __shared__ float stab[256];
  if constexpr (FMT == kDecFp4Tab || FMT == kDecInt4) {
    for (int i = threadIdx.x; i < 256; i += kThreads) stab[i] = T.v[i];
    __syncthreads();
  }
  const int64_t units = d.n * (d.k / 16);
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int64_t row = u / (d.k / 16), col = (u - row * (d.k / 16)) * 16;
    float2 v[8];
    decode16<FMT>(d, row, col, v, stab);
    float4* o = reinterpret_cast<float4*>(out + row * d.k + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = make_float4(v[2 * i].x, v[2 * i].y, v[2 * i + 1].x, v[2 * i + 1].y);
  }
}

template <int FMT, bool BF16, bool HAS_H>
__global__ void __launch_bounds__(kThreads)
k_error(DecodeArgs d, ScaleTab T, const char* __restrict__ W, int64_t ld_bytes,
        const float* __restrict__ h, double* __restrict__ partial) {
  __shared__ double red[kThreads / 32][4];
  __shared__ float stab[256];
  if constexpr (FMT == kDecFp4Tab || FMT == kDecInt4) {
    for (int i = threadIdx.x; i < 256; i += kThreads) stab[i] = T.v[i];
    __syncthreads();
  }
  const int64_t units = d.n * (d.k / 16);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int64_t row = u / (d.k / 16), col = (u - row * (d.k / 16)) * 16;
    float2 v[8], w[8];
    decode16<FMT>(d, row, col, v, stab);
    const char* wp = W + row * ld_bytes + col * (BF16 ? 2 : 4);
    if constexpr (BF16) {
      const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(wp));
      const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(wp) + 1);
      const uint32_t wd[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int p = 0; p < 8; ++p) w[p] = make_float2(bf16lo(wd[p]), bf16hi(wd[p]));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(wp) + i);
        w[2 * i] = make_float2(x.x, x.y);
        w[2 * i + 1] = make_float2(x.z, x.w);
      }
    }
    float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float2 dd = __fadd2_rn(w[p], make_float2(-v[p].x, -v[p].y));
      const float2 d2 = __fmul2_rn(dd, dd), w2 = __fmul2_rn(w[p], w[p]);
      s0 = __fadd2_rn(s0, d2);
      s1 = __fadd2_rn(s1, w2);
      if constexpr (HAS_H) {
        const float4 hv = __ldg(reinterpret_cast<const float4*>(h + col) + p / 2);
        const float2 hh = (p & 1) ? make_float2(hv.z, hv.w) : make_float2(hv.x, hv.y);
        s2 = __ffma2_rn(hh, d2, s2);
        s3 = __ffma2_rn(hh, w2, s3);
      }
    }
    acc[0] += (double)s0.x + (double)s0.y;
    acc[1] += (double)s1.x + (double)s1.y;
    if constexpr (HAS_H) {
      acc[2] += (double)s2.x + (double)s2.y;
      acc[3] += (double)s3.x + (double)s3.y;
    }
  }
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
    partial[(int64_t)blockIdx.x * 4 + threadIdx.x] = s;
  }
}

// One CTA: thread t sums partials t, t + 256, ... in order; then a fixed-shape tree.
__global__ void __launch_bounds__(kThreads)
k_error_final(const double* __restrict__ partial, int parts, double* sums) {
  __shared__ double red[4][kThreads];
  double s[4] = {0.0, 0.0, 0.0, 0.0};
  for (int p = threadIdx.x; p < parts; p += kThreads)
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] += partial[p * 4 + i];
#pragma unroll
  for (int i = 0; i < 4; ++i) red[i][threadIdx.x] = s[i];
  __syncthreads();
  for (int half = kThreads / 2; half > 0; half >>= 1) {
    if ((int)threadIdx.x < half)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[i][threadIdx.x] += red[i][threadIdx.x + half];
    __syncthreads();
  }
  if (threadIdx.x < 4) sums[threadIdx.x] = red[threadIdx.x][0];
}

template <int FMT>
cudaError_t dequant_fmt(const DecodeArgs& d, float* out, cudaStream_t st) {
  const int64_t units = d.n * (d.k / 16);
  int64_t grid = (units + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sm_count() * 16;
  if (grid > cap) grid = cap;
  k_dequant<FMT><<<(unsigned)grid, kThreads, 0, st>>>(d, scale_tab(d.scale_fmt), out);
  return cudaGetLastError();
}

template <int FMT>
cudaError_t error_fmt(const DecodeArgs& d, const void* W, int dtype, int64_t ld, const float* h,
                      double* partial, int parts, cudaStream_t st) {
  const char* Wc = (const char*)W;
  const ScaleTab& T = scale_tab(d.scale_fmt);
  if (dtype == 1) {
    if (h) k_error<FMT, true, true><<<parts, kThreads, 0, st>>>(d, T, Wc, ld * 2, h, partial);
    else k_error<FMT, true, false><<<parts, kThreads, 0, st>>>(d, T, Wc, ld * 2, h, partial);
  } else {
    if (h) k_error<FMT, false, true><<<parts, kThreads, 0, st>>>(d, T, Wc, ld * 4, h, partial);
    else k_error<FMT, false, false><<<parts, kThreads, 0, st>>>(d, T, Wc, ld * 4, h, partial);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_error_final(const double* partial, int parts, double* sums, cudaStream_t st) {
  k_error_final<<<1, kThreads, 0, st>>>(partial, parts, sums);
  return cudaGetLastError();
}

int error_partials(int64_t n, int64_t k) {
  const int64_t units = n * (k / 16);
  int64_t ctas = (units + kThreads - 1) / kThreads;
  if (ctas > kMaxErrCtas) ctas = kMaxErrCtas;
  return (int)(ctas < 1 ? 1 : ctas);
}

namespace {
// One output byte per thread: the 128 x 4 tile layout of sm_100 block-scaled MMA.
__global__ void k_swizzle_scales(const uint8_t* __restrict__ in, int64_t n, int64_t kb,
                                 uint8_t* __restrict__ out, int64_t total) {
  const int64_t ct = (kb + 3) / 4;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = o / 512, w = o % 512;
    const int64_t m = (tile / ct) * 128 + (w % 16) / 4 * 32 + w / 16;
    const int64_t c = (tile % ct) * 4 + (w % 4);
    out[o] = (m < n && c < kb) ? in[m * kb + c] : (uint8_t)0;
  }
}
}  // namespace

size_t swizzled_scales_bytes(int64_t n, int64_t kb) {
  return (size_t)((n + 127) / 128) * 128 * (size_t)((kb + 3) / 4) * 4;
}

cudaError_t launch_swizzle_scales(const uint8_t* in, int64_t n, int64_t kb, uint8_t* out,
                                  cudaStream_t st) {
  const int64_t total = (int64_t)swizzled_scales_bytes(n, kb);
  int64_t grid = (total + 255) / 256;
  if (grid > 4096) grid = 4096;
  k_swizzle_scales<<<(unsigned)grid, 256, 0, st>>>(in, n, kb, out, total);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const DecodeArgs& d, float* out, cudaStream_t st) {
  switch (decoder_of(d)) {
    case kDecFp4: return dequant_fmt<kDecFp4>(d, out, st);
    case kDecInt8: return dequant_fmt<kDecInt8>(d, out, st);
    case kDecInt4: return dequant_fmt<kDecInt4>(d, out, st);
    case kDecFp4Tab: return dequant_fmt<kDecFp4Tab>(d, out, st);
    default: return dequant_fmt<kDecTile>(d, out, st);
  }
}

cudaError_t launch_error(const DecodeArgs& d, const void* W, int dtype, int64_t ld,
                         const float* h, double* partial, int parts, double* sums,
                         cudaStream_t st) {
  cudaError_t e;
  switch (decoder_of(d)) {
    case kDecFp4: e = error_fmt<kDecFp4>(d, W, dtype, ld, h, partial, parts, st); break;
    case kDecInt8: e = error_fmt<kDecInt8>(d, W, dtype, ld, h, partial, parts, st); break;
    case kDecInt4: e = error_fmt<kDecInt4>(d, W, dtype, ld, h, partial, parts, st); break;
    case kDecFp4Tab: e = error_fmt<kDecFp4Tab>(d, W, dtype, ld, h, partial, parts, st); break;
    default: e = error_fmt<kDecTile>(d, W, dtype, ld, h, partial, parts, st); break;
  }
  if (e != cudaSuccess) return e;
  k_error_final<<<1, kThreads, 0, st>>>(partial, parts, sums);
  return cudaGetLastError();
}

}  // namespace mxq
