// mxq_common.cuh -- device helpers shared by the mxq kernels (sm_100a only).
//
// Number formats (OCP E4M3 "FN", E2M1) are decoded from bit fields or converted with the
// sm_100a hardware conversions `cvt.rn.satfinite.{e4m3x2,e2m1x2}.f32` (round to nearest,
// ties to even, saturating at the largest finite value) and their inverses
// `cvt.rn.f16x2.{e4m3x2,e2m1x2}`.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "mxq kernels target sm_100a (B200) only"
#endif

namespace mxq {

constexpr unsigned kFull = 0xffffffffu;

// Value of a non-negative E4M3 code 0..126: normals (1 + m/8) 2^(e-7) are the fp32 bit
// pattern (c << 20) + (120 << 23); subnormals are c * 2^-9.
__device__ __forceinline__ float e4m3_pos(int c) {
  return c >= 8 ? __int_as_float((c << 20) + (120 << 23)) : (float)c * 0.001953125f;
}

// Round-to-nearest-even E4M3 code of x >= 0, saturating at 448 (code 0x7E).
__device__ __forceinline__ int e4m3_rn_code(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0x7f;
}

// Two E4M3 bytes (lo from x0, hi from x1), RNE + saturation; keeps the sign.
__device__ __forceinline__ uint32_t e4m3x2_rn(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// Two E4M3 bytes -> two halves (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t b) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(b));
  return r;
}

// Two E2M1 codes in one byte (lo nibble from x0, hi from x1), RNE + saturation at 6.
__device__ __forceinline__ uint32_t e2m1x2_rn(float x0, float x1) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u16.u8 %0, t;\n\t}"
      : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// One byte of two E2M1 codes -> two halves (lo nibble -> low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r) : "r"(byte));
  return r;
}

// fl32(g * s - a) for a half g and a half s (the product of two halves is exact in fp32;
// one rounding of the sum) -- the mixed-precision fma of sm_100.
__device__ __forceinline__ float fma_h_h_f(uint16_t g, uint16_t s, float minus_a) {
  float r;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(r) : "h"(g), "h"(s), "f"(minus_a));
  return r;
}

__device__ __forceinline__ uint16_t lo16(uint32_t v) { return (uint16_t)(v & 0xffffu); }
__device__ __forceinline__ uint16_t hi16(uint32_t v) { return (uint16_t)(v >> 16); }

// bf16 pair in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Warp arg-min over (value, index): smallest value, then smallest index.
__device__ __forceinline__ void warp_argmin(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(kFull, v, o);
    int oi = __shfl_xor_sync(kFull, i, o);
    if (ov < v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

__device__ __forceinline__ void warp_argmin(double& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    double ov = __shfl_xor_sync(kFull, v, o);
    int oi = __shfl_xor_sync(kFull, i, o);
    if (ov < v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

}  // namespace mxq
