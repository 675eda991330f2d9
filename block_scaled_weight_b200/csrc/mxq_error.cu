// mxq_error.cu -- dequantisation and weight-error metrics.
//
// Dequantised value (the microscaling reconstruction x^ = s q, "Is Finer Better? The
// Limits of Microscaling Formats in LLMs", sec. 2.1):
//   NVFP4  E4M3(scale) * E2M1(code)                (exact in float32)
//   INT8   fl32(|q| * fl32(E4M3(scale) / 127)), signed
//   E4M3   fl32(tile scale * E4M3(code)), signed
// Metrics (qwantize "Results": weight error ||Q(W) - W||_F / ||W||_F; the h-weighted
// error of "quantization_algorithms.txt", sec. 1): the four sums sum d^2, sum w^2,
// sum h d^2, sum h w^2. HBM-bound: each thread decodes 16 consecutive elements of a row;
// float32 partials over those 16, double from there on; the per-CTA partials are summed
// in a fixed order by a second one-CTA kernel (deterministic).
#include "mxq_common.cuh"
#include "mxq_internal.h"

namespace mxq {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxErrCtas = 148 * 8;

__device__ __forceinline__ float e2m1_mag(uint32_t nib) {
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6 from the code bits: e = nib >> 1, m = nib & 1.
  const uint32_t e = (nib >> 1) & 3u, m = nib & 1u;
  return e == 0 ? 0.5f * (float)m : __uint_as_float(((126u + e) << 23) | (m << 22));
}

// Decode the 16 elements starting at (row, col) into v[16].
__device__ __forceinline__ void decode16(const DecodeArgs& d, int64_t row, int64_t col,
                                         float (&v)[16]) {
  if (d.fmt == 0) {
    const uint8_t* cp = (const uint8_t*)d.codes + row * (d.k / 2) + col / 2;
    const uint2 cw = *reinterpret_cast<const uint2*>(cp);
    const float s = e4m3_pos(((const uint8_t*)d.scales)[row * (d.k / d.block) + col / d.block]);
    const uint32_t w2[2] = {cw.x, cw.y};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t nib = (w2[j / 8] >> (4 * (j % 8))) & 15u;
      const float m = __fmul_rn(s, e2m1_mag(nib & 7u));
      v[j] = (nib & 8u) ? -m : m;
    }
  } else if (d.fmt == 1) {
    const int8_t* cp = (const int8_t*)d.codes + row * d.k + col;
    const uint4 cw = *reinterpret_cast<const uint4*>(cp);
    const int sc = ((const uint8_t*)d.scales)[row * (d.k / d.block) + col / d.block];
    const float s = __fdiv_rn(e4m3_pos(sc), 127.0f);
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int q = (int)(int8_t)((w4[j / 4] >> (8 * (j % 4))) & 0xffu);
      const float m = __fmul_rn((float)(q < 0 ? -q : q), s);
      v[j] = q < 0 ? -m : m;
    }
  } else {
    const uint8_t* cp = (const uint8_t*)d.codes + row * d.k + col;
    const uint4 cw = *reinterpret_cast<const uint4*>(cp);
    const float s = ((const float*)d.scales)[(row / d.block) * (d.k / d.block) + col / d.block];
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t c = (w4[j / 4] >> (8 * (j % 4))) & 0xffu;
      const float m = __fmul_rn(s, e4m3_pos((int)(c & 0x7fu)));
      v[j] = (c & 0x80u) ? -m : m;
    }
  }
}

__global__ void __launch_bounds__(kThreads)
k_dequant(DecodeArgs d, float* __restrict__ out) {
  const int64_t units = d.n * (d.k / 16);
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int64_t row = u / (d.k / 16), col = (u - row * (d.k / 16)) * 16;
    float v[16];
    decode16(d, row, col, v);
    float4* o = reinterpret_cast<float4*>(out + row * d.k + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
k_error(DecodeArgs d, const char* __restrict__ W, int64_t ld_bytes, const float* __restrict__ h,
        double* __restrict__ partial) {
  __shared__ double red[kThreads / 32][4];
  const int64_t units = d.n * (d.k / 16);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int64_t row = u / (d.k / 16), col = (u - row * (d.k / 16)) * 16;
    float v[16], w[16], hh[16];
    decode16(d, row, col, v);
    const char* wp = W + row * ld_bytes + col * (BF16 ? 2 : 4);
    if constexpr (BF16) {
      const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(wp));
      const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(wp) + 1);
      const uint32_t wd[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) { w[2 * i] = bf16lo(wd[i]); w[2 * i + 1] = bf16hi(wd[i]); }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(wp) + i);
        w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
      }
    }
    if (h) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(h + col) + i);
        hh[4 * i] = x.x; hh[4 * i + 1] = x.y; hh[4 * i + 2] = x.z; hh[4 * i + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) hh[j] = 0.0f;
    }
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float dj = __fsub_rn(w[j], v[j]);
      const float d2 = __fmul_rn(dj, dj), w2 = __fmul_rn(w[j], w[j]);
      s0 += d2;
      s1 += w2;
      s2 = fmaf(hh[j], d2, s2);
      s3 = fmaf(hh[j], w2, s3);
    }
    acc[0] += (double)s0; acc[1] += (double)s1; acc[2] += (double)s2; acc[3] += (double)s3;
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

__global__ void k_error_final(const double* __restrict__ partial, int parts, double* sums) {
  if (threadIdx.x < 4) {
    double s = 0.0;
    for (int p = 0; p < parts; ++p) s += partial[p * 4 + threadIdx.x];
    sums[threadIdx.x] = s;
  }
}

}  // namespace

int error_partials(int64_t n, int64_t k) {
  const int64_t units = n * (k / 16);
  int64_t ctas = (units + kThreads - 1) / kThreads;
  if (ctas > kMaxErrCtas) ctas = kMaxErrCtas;
  return (int)(ctas < 1 ? 1 : ctas);
}

cudaError_t launch_dequant(const DecodeArgs& d, float* out, cudaStream_t st) {
  const int64_t units = d.n * (d.k / 16);
  int64_t grid = (units + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sm_count() * 16;
  if (grid > cap) grid = cap;
  k_dequant<<<(unsigned)grid, kThreads, 0, st>>>(d, out);
  return cudaGetLastError();
}

cudaError_t launch_error(const DecodeArgs& d, const void* W, int dtype, int64_t ld,
                         const float* h, double* partial, int parts, double* sums,
                         cudaStream_t st) {
  if (dtype == 1)
    k_error<true><<<parts, kThreads, 0, st>>>(d, (const char*)W, ld * 2, h, partial);
  else
    k_error<false><<<parts, kThreads, 0, st>>>(d, (const char*)W, ld * 4, h, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_error_final<<<1, 32, 0, st>>>(partial, parts, sums);
  return cudaGetLastError();
}

}  // namespace mxq
