// mxq_gptq.cu -- FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1, the
// 64x64 tile scheme: a fixed tile scale, H = X^T X + lambda I over the tile's 64 input
// dimensions, columns quantised one after another to E4M3 with each residual propagated
// through H^-1 -- GPTQ's update in its Cholesky form).
//
// Two kernels:
//   k_gptq_prepare  one CTA per column block b: H = sym(G_b) + lambda I (lambda = damp times
//                   the mean of diag G_b, 1 when that mean is 0), U the upper Cholesky factor
//                   of H^-1 (H^-1 = U^T U), all in float64, rounded to float32 once. U is
//                   reached without forming H^-1: with J the order reversal, J H J = L L^T
//                   (lower Cholesky) gives H^-1 = (J L^-1 J)^T (J L^-1 J), so U = J L^-1 J;
//                   L and L^-1 come from one register-resident elimination (mxq_chol64.cuh).
//   k_gptq_tiles    one thread per (row, column block): the row's 64 weights live in
//                   registers and are swept column by column,
//                       q = E4M3(RNE(fl32(|w_c| / s))),  wq = +-fl32(s q),
//                       err = fl32(fl32(w_c - wq) / U_cc),  w_j = fl32(w_j - fl32(err U_cj)),
//                   every step a separately rounded float32 operation, as in the definition.
//                   Rows are independent; U (16 KB) is staged once per CTA in shared memory
//                   and read as warp-wide broadcasts.
#include "mxq_chol64.cuh"
#include "mxq_common.cuh"
#include "mxq_internal.h"

#include <cuda_bf16.h>

namespace mxq {
namespace {

constexpr int kT = 64;                 // tile edge
constexpr int kPrepThreads = kCholThreads;
constexpr int kSweepThreads = 128;     // rows per CTA pass

__global__ void __launch_bounds__(kPrepThreads)
k_gptq_prepare(const float* __restrict__ G, double damp, float* __restrict__ U) {
  __shared__ Chol64Smem s;
  __shared__ double lam_s;
  const float* Gb = G + (int64_t)blockIdx.x * kT * kT;
  float* Ub = U + (int64_t)blockIdx.x * kT * kT;
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;

  if (t < 32) {                   // lambda = damp * mean(diag G_b)
    double d = (double)Gb[t * (kT + 1)] + (double)Gb[(t + 32) * (kT + 1)];
    d = warp_sum(d);
    if (t == 0) {
      const double lam = damp * (d / kT);
      lam_s = lam > 0.0 ? lam : 1.0;
    }
  }
  __syncthreads();
  // A_il = H_{63-i, 63-l}, H = (G + G^T) / 2 + lambda I, this thread's 16 elements
  double a[4][4], bm[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ty + 16 * r, l = tx + 16 * c, p = kT - 1 - i, q = kT - 1 - l;
      double v = 0.5 * ((double)Gb[p * kT + q] + (double)Gb[q * kT + p]);
      if (i == l) v += lam_s;
      a[r][c] = v;
    }
  // L (A = L L^T) and L^-1 = D^-1/2 B
  chol64_regs(a, bm, s);
  // U_pq = (L^-1)_{63-p, 63-q} (upper), rounded to float32 once
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ty + 16 * r, l = tx + 16 * c;
      Ub[(kT - 1 - i) * kT + (kT - 1 - l)] = i >= l ? (float)(bm[r][c] * s.rdg[i]) : 0.0f;
    }
}

template <bool BF16>
__device__ __forceinline__ void load_row(const char* src, float (&w)[kT]) {
  if constexpr (BF16) {
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + v);
      const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        w[v * 8 + 2 * p] = bf16lo(x[p]);
        w[v * 8 + 2 * p + 1] = bf16hi(x[p]);
      }
    }
  } else {
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const float4 u = __ldg(reinterpret_cast<const float4*>(src) + v);
      w[4 * v] = u.x;
      w[4 * v + 1] = u.y;
      w[4 * v + 2] = u.z;
      w[4 * v + 3] = u.w;
    }
  }
}

struct SweepParams {
  const char* W;
  int64_t n, k, ld_bytes;
  const float* U;       // [k/64][64][64]
  const float* scales;  // [n/64][k/64]
  uint8_t* codes;       // [n][k]
};

template <bool BF16>
__global__ void __launch_bounds__(kSweepThreads)
k_gptq_tiles(SweepParams P) {
  __shared__ __align__(16) float Us[kT * kT];
  const int tj = blockIdx.x;
  const int64_t tk = P.k / kT;
  {
    const float4* src = reinterpret_cast<const float4*>(P.U + (int64_t)tj * kT * kT);
    for (int e = threadIdx.x; e < kT * kT / 4; e += kSweepThreads)
      reinterpret_cast<float4*>(Us)[e] = src[e];
  }
  __syncthreads();
  const int elsz = BF16 ? 2 : 4;
  for (int64_t row = (int64_t)blockIdx.y * kSweepThreads + threadIdx.x; row < P.n;
       row += (int64_t)gridDim.y * kSweepThreads) {
    float w[kT];
    load_row<BF16>(P.W + row * P.ld_bytes + (int64_t)tj * kT * elsz, w);
    const float s = __ldg(P.scales + (row / kT) * tk + tj);
    uint32_t cw[kT / 4];
#pragma unroll
    for (int i = 0; i < kT / 4; ++i) cw[i] = 0u;
#pragma unroll
    for (int c = 0; c < kT; ++c) {
      const float wv = w[c];
      const uint32_t sign = __float_as_uint(wv) >> 31;
      const uint32_t q = s > 0.0f ? (e4m3x2_rn(__fdiv_rn(fabsf(wv), s), 0.0f) & 0x7fu) : 0u;
      cw[c / 4] |= ((sign << 7) | q) << (8 * (c % 4));
      if (c == kT - 1) break;              // nothing left to propagate into
      const float wq = copysignf(__fmul_rn(s, e4m3_pos((int)q)), wv);
      const float err = __fdiv_rn(__fsub_rn(wv, wq), Us[c * kT + c]);
      const float4* Ur = reinterpret_cast<const float4*>(Us + c * kT);
#pragma unroll
      for (int jb = (c + 1) / 4; jb < kT / 4; ++jb) {
        const float4 u = Ur[jb];
        const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * jb + e;
          if (j > c) w[j] = __fsub_rn(w[j], __fmul_rn(err, uu[e]));
        }
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(P.codes + row * P.k + (int64_t)tj * kT);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      dst[v] = make_uint4(cw[4 * v], cw[4 * v + 1], cw[4 * v + 2], cw[4 * v + 3]);
  }
}

}  // namespace

cudaError_t launch_gptq_prepare(const float* G, int64_t nblocks, double damp, float* U,
                                cudaStream_t st) {
  if (nblocks <= 0) return cudaSuccess;
  k_gptq_prepare<<<(unsigned)nblocks, kPrepThreads, 0, st>>>(G, damp, U);
  return cudaGetLastError();
}

cudaError_t launch_gptq_tiles(const void* W, int dtype, int64_t n, int64_t k, int64_t ld,
                              const float* U, const float* scales, uint8_t* codes,
                              cudaStream_t st) {
  if (n == 0 || k == 0) return cudaSuccess;
  const bool bf = dtype == 1;
  SweepParams P{(const char*)W, n, k, ld * (bf ? 2 : 4), U, scales, codes};
  const int64_t tk = k / kT;
  const int64_t groups = (n + kSweepThreads - 1) / kSweepThreads;
  // about 4 resident CTAs per SM in total
  int64_t gy = ((int64_t)sm_count() * 4 + tk - 1) / tk;
  if (gy > groups) gy = groups;
  if (gy < 1) gy = 1;
  const dim3 grid((unsigned)tk, (unsigned)gy);
  if (bf) k_gptq_tiles<true><<<grid, kSweepThreads, 0, st>>>(P);
  else k_gptq_tiles<false><<<grid, kSweepThreads, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace mxq
