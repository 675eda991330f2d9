// mxq_chol64.cuh -- the Cholesky factor of a 64 x 64 symmetric positive definite float64
// matrix and the inverse of that factor, by one CTA of 256 threads, in registers (the
// factorisation behind GPTQ's update: Frantar et al. 2022, Algorithm 1, in its Cholesky form).
//
// Thread (ty, tx) = (t / 16, t % 16) keeps the 16 elements (ty + 16a, tx + 16b), a, b = 0..3,
// of the matrix T and of B (B = I at the start). Step j = 0 .. 63 publishes column j of T and
// row j of B through shared memory (double-buffered, one barrier per step); with
// f_i = T_ij / T_jj every thread then updates its elements,
//     T_il -= f_i T_lj   (l > j, i >= l: the unscaled elimination, T = L_unit D L_unit^T),
//     B_ic -= f_i B_jc   (i > j: the same row operations applied to I, so B -> L_unit^-1).
// With d = sqrt(diag D): L_il = T_il / d_l, L_ll = d_l, and L^-1 = D^-1/2 B, (L^-1)_ic = B_ic / d_i.
// Only the lower triangle of the input affects the result (the upper one may hold anything finite).
#pragma once

#include <cuda_runtime.h>

namespace mxq {

constexpr int kCholN = 64;
constexpr int kCholThreads = 256;

struct Chol64Smem {
  double colT[2][kCholN], rowB[2][kCholN], piv[kCholN];
  double dg[kCholN], rdg[kCholN];   // d and 1 / d, valid after chol64_regs returns
};

// 1 / x for the elimination's pivots, off the division unit: a float32 reciprocal as the seed,
// then two Newton-Raphson steps r <- r + r (1 - x r) (quadratic convergence: 2^-24 -> 2^-48
// -> below the float64 rounding); x outside float32's normal range takes the division.
__device__ __forceinline__ double chol_recip(double x) {
  const float xf = (float)x;
  if (!(fabsf(xf) >= 1.2e-38f && fabsf(xf) <= 3.0e38f)) return 1.0 / x;
  double r = (double)__frcp_rn(xf);
  r = fma(r, fma(-x, r, 1.0), r);
  r = fma(r, fma(-x, r, 1.0), r);
  return r;
}

// a: this thread's elements of the matrix (lower triangle significant); on return a holds the
// unscaled elimination (T above), bm the elements of L_unit^-1, and s.dg / s.rdg the column
// scales d and 1 / d (a barrier has passed since they were written).
__device__ __forceinline__ void chol64_regs(double (&a)[4][4], double (&bm)[4][4],
                                            Chol64Smem& s) {
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) bm[r][c] = ty + 16 * r == tx + 16 * c ? 1.0 : 0.0;
#pragma unroll
  for (int jb = 0; jb < 4; ++jb) {
#pragma unroll 1
    for (int jj = 0; jj < 16; ++jj) {
      const int j = 16 * jb + jj, buf = j & 1;
      // jb is a compile-time constant here, so the register blocks a step cannot touch
      // (T: block columns before jb or above the diagonal; B: block rows before jb, block
      // columns after jb, where row j of B is 0) drop out of the code
      if (tx == jj) {
#pragma unroll
        for (int r = jb; r < 4; ++r) s.colT[buf][ty + 16 * r] = a[r][jb];
      }
      if (ty == jj) {
#pragma unroll
        for (int c = 0; c <= jb; ++c) s.rowB[buf][tx + 16 * c] = bm[jb][c];
      }
      __syncthreads();
      const double pv = s.colT[buf][j];
      if (t == 0) s.piv[j] = pv;
      const double rr = chol_recip(pv);
      double f[4], tl[4], bj[4];
#pragma unroll
      for (int q = jb; q < 4; ++q) {
        f[q] = s.colT[buf][ty + 16 * q] * rr;
        tl[q] = s.colT[buf][tx + 16 * q];
      }
#pragma unroll
      for (int q = 0; q <= jb; ++q) bj[q] = s.rowB[buf][tx + 16 * q];
#pragma unroll
      for (int r = jb; r < 4; ++r)
#pragma unroll
        for (int c = 0; c <= r; ++c) {
          const int i = ty + 16 * r, l = tx + 16 * c;
          if (c >= jb && l > j && i >= l) a[r][c] -= f[r] * tl[c];
          if (c <= jb && i > j) bm[r][c] -= f[r] * bj[c];
        }
    }
  }
  __syncthreads();
  if (t < kCholN) {
    const double d = sqrt(s.piv[t]);
    s.dg[t] = d;
    s.rdg[t] = 1.0 / d;
  }
  __syncthreads();
}

}  // namespace mxq
