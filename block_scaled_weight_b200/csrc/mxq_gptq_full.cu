// mxq_gptq_full.cu -- GPTQ with the block quantizer as its inner step (qwantize "Results",
// "GPTQ Quantization": the GPTQ block is the quantization block; sequential and ordered
// variants; the algorithm is Frantar et al. 2022, Algorithm 1, in its Cholesky form).
//
// Three stages, each its own entry point:
//   factor  U = upper Cholesky factor of the damped H^-1, H's rows and columns in sweep
//           order (a block permutation for the ordered variant), in float64, rounded to
//           float32 once. With J the order reversal, J H J = L L^T gives H^-1 = U^T U with
//           U = J L^-1 J, so one blocked Cholesky and one blocked triangular inverse (64 x 64
//           tiles, float64 products on the tensor cores) replace GPTQ's
//           inverse-then-Cholesky; the inverse follows the Cholesky panel by panel.
//   order   (ordered variant) the Hessian-weighted loss of every column block under the
//           plain quantizer, and the blocks sorted by descending loss.
//   sweep   rows are independent. Positions are processed in panels of up to 64: one
//           half-warp per row searches each block's scale exactly on its current weights
//           (candidate errors in double, element order, lowest code on ties), quantises
//           the block's columns one after another with the in-block updates, and applies
//           each block's product to the panel's later blocks; a tiled kernel then applies
//           the panel's block products to every later position of every row (the next
//           panel's positions first, the rest overlapping the next panel).
// Every float32 step follows the definition's operation order: in-block updates
// w -= fl32(err U), past the block acc = fma(err_j, U_j, acc) over the block's columns in
// order, then one subtraction.
#include "mxq_chol64.cuh"
#include "mxq_common.cuh"
#include "mxq_gridk.cuh"
#include "mxq_internal.h"

#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

namespace mxq {
namespace {

// ======================================================================================
// factor
// ======================================================================================
constexpr int kNB = 64;                  // tile edge of the blocked factorisation
constexpr int kFThreads = 256;
static_assert(kFThreads == kCholThreads && kNB == kCholN, "the diagonal tile is one chol64 CTA");
constexpr int kPanelTiles = 4;           // tile columns per trailing update of the Cholesky

struct FactorArgs {
  const float* H;        // [k][k]
  int64_t k, kp;         // order, padded to a multiple of 64
  int B;                 // block of the permutation
  const int32_t* perm;   // [k / B] or null
  double* A;             // [kp][kp]: J H J + lambda I, then L (lower tiles)
  double* M;             // [kp][kp]: L^-1 (lower tiles)
  double* scal;          // [0] lambda
  float* U;              // [k][k]
};

// Column of sweep position pos; a block index outside 0 .. k/B - 1 is clamped into range
// (an invalid permutation gives a meaningless result, never an out-of-bounds access).
__device__ __forceinline__ int64_t perm_col(const FactorArgs& a, int64_t pos) {
  if (!a.perm) return pos;
  const int64_t b = min(max((int64_t)a.perm[pos / a.B], (int64_t)0), a.k / a.B - 1);
  return b * a.B + pos % a.B;
}

// lambda = damp * mean(diag H), 1 when that is not positive; fixed-order reduction.
__global__ void __launch_bounds__(kFThreads)
k_factor_lambda(const float* __restrict__ H, int64_t k, double damp, double* scal) {
  __shared__ double part[kFThreads];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < k; i += kFThreads) s += (double)H[i * k + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = kFThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double lam = damp * (part[0] / (double)k);
    scal[0] = lam > 0.0 ? lam : 1.0;
  }
}

// A_ij = H~_{k-1-i, k-1-j} (+ lambda on the diagonal), H~ = sym(H) in sweep order; the
// padding beyond k is the identity.
__global__ void k_factor_load(FactorArgs a) {
  const double lam = a.scal[0];
  const int64_t total = a.kp * a.kp;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / a.kp, j = e % a.kp;
    double v;
    if (i >= a.k || j >= a.k) {
      v = i == j ? 1.0 : 0.0;
    } else {
      const int64_t p = perm_col(a, a.k - 1 - i), q = perm_col(a, a.k - 1 - j);
      v = 0.5 * ((double)a.H[p * a.k + q] + (double)a.H[q * a.k + p]);
      if (i == j) v += lam;
    }
    a.A[e] = v;
  }
}

// Diagonal tile p: its Cholesky factor L_pp (lower, the upper part 0) into A and its
// inverse M_pp into M (the register-resident elimination of mxq_chol64.cuh).
__global__ void __launch_bounds__(kFThreads) k_potrf_inv(double* A, double* M, int64_t kp, int p) {
  __shared__ Chol64Smem s;
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
  double* g = A + (int64_t)p * kNB * kp + (int64_t)p * kNB;
  double* gm = M + (int64_t)p * kNB * kp + (int64_t)p * kNB;
  double a[4][4], bm[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) a[r][c] = g[(int64_t)(ty + 16 * r) * kp + tx + 16 * c];
  chol64_regs(a, bm, s);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ty + 16 * r, l = tx + 16 * c;
      g[(int64_t)i * kp + l] = i > l ? a[r][c] * s.rdg[l] : (i == l ? s.dg[i] : 0.0);
      gm[(int64_t)i * kp + l] = i >= l ? bm[r][c] * s.rdg[i] : 0.0;
    }
}

// ---- 64 x 64 x 64 float64 tile products (FP64 tensor cores) -----------------------------
// 128 threads = 4 warps; warp w computes the 32 x 32 quadrant (rows 32 (w / 2), columns
// 32 (w % 2)) as 4 x 4 fragments of mma.sync m8n8k4 f64 (A row-major 8 x 4, B 4 x 8, C 8 x 8
// in two doubles per lane). Operand tiles sit row-major in shared memory with rows of kPLd
// doubles (68: every fragment load -- 8 rows x 4 columns of A, or of B either way round --
// touches each bank pair exactly twice), fetched with 16-byte cp.async.
constexpr int kPThreads = 128;
constexpr int kPLd = kNB + 4;
constexpr size_t kProdSmem1 = 2 * kNB * kPLd * sizeof(double);
using Frag = double[4][4][2];            // [m tile][n tile][c0, c1]

__device__ __forceinline__ void cp_async16d(double* s, const double* g) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(s);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(a), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ void stage_async(double* s, const double* g, int64_t ld) {
  for (int e = threadIdx.x * 2; e < kNB * kNB; e += kPThreads * 2)
    cp_async16d(s + (e / kNB) * kPLd + e % kNB, g + (int64_t)(e / kNB) * ld + e % kNB);
}

__device__ __forceinline__ void dmma(double a, double b, double (&c)[2]) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

// c += S1 S2^T (NT = true: S2 holds B^T, [n][k]) or S1 S2 (NT = false: S2 is [k][n]).
template <bool NT>
__device__ __forceinline__ void tile_mul(const double* S1, const double* S2, Frag& c) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int mb = 32 * (w >> 1), nb = 32 * (w & 1);
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll 2
  for (int k0 = 0; k0 < kNB; k0 += 4) {
    double a[4], b[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) a[m] = S1[(mb + 8 * m + g) * kPLd + k0 + t4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
      b[n] = NT ? S2[(nb + 8 * n + g) * kPLd + k0 + t4] : S2[(k0 + t4) * kPLd + nb + 8 * n + g];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < 4; ++n) dmma(a[m], b[n], c[m][n]);
  }
}

// c = sum over n steps of tile(G1(q)) x tile(G2(q)) (x: NT or NN), q = 0 .. n-1, in k-chunks
// of 32: each chunk's operand halves are fetched into one of two stages while the other
// stage is multiplied (A half [64][32] and B^T half [64][32] in rows of kHLd doubles, or B
// half [32][64] in rows of kPLd; both keep every fragment load at two wavefronts).
constexpr int kHLd = kNB / 2 + 4;
constexpr int kStageD = kNB * kHLd + (kNB * kHLd > (kNB / 2) * kPLd ? kNB * kHLd : (kNB / 2) * kPLd);
constexpr size_t kProdSmem = 2 * kStageD * sizeof(double);
static_assert(kProdSmem >= kProdSmem1, "the last product of k_minv_row reuses the stages");

template <bool NT>
__device__ __forceinline__ void half_mul(const double* S1, const double* S2, Frag& c) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int mb = 32 * (w >> 1), nb = 32 * (w & 1);
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll 2
  for (int k0 = 0; k0 < kNB / 2; k0 += 4) {
    double a[4], b[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) a[m] = S1[(mb + 8 * m + g) * kHLd + k0 + t4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
      b[n] = NT ? S2[(nb + 8 * n + g) * kHLd + k0 + t4] : S2[(k0 + t4) * kPLd + nb + 8 * n + g];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int n = 0; n < 4; ++n) dmma(a[m], b[n], c[m][n]);
  }
}

template <bool NT, class F1, class F2>
__device__ __forceinline__ void tile_sum(double* sm, int n, F1 g1, F2 g2, int64_t ld, Frag& c) {
  if (n <= 0) return;
  auto stage = [&](int buf, int ch) {
    const int q = ch >> 1, h = ch & 1;
    double* sa = sm + buf * kStageD;
    double* sb = sa + kNB * kHLd;
    const double* ga = g1(q) + 32 * h;
    for (int e = threadIdx.x; e < kNB * 16; e += kPThreads) {
      const int r = e >> 4, c2 = 2 * (e & 15);
      cp_async16d(sa + r * kHLd + c2, ga + (int64_t)r * ld + c2);
    }
    if (NT) {
      const double* gb = g2(q) + 32 * h;
      for (int e = threadIdx.x; e < kNB * 16; e += kPThreads) {
        const int r = e >> 4, c2 = 2 * (e & 15);
        cp_async16d(sb + r * kHLd + c2, gb + (int64_t)r * ld + c2);
      }
    } else {
      const double* gb = g2(q) + (int64_t)(32 * h) * ld;
      for (int e = threadIdx.x; e < (kNB / 2) * 32; e += kPThreads) {
        const int r = e >> 5, c2 = 2 * (e & 31);
        cp_async16d(sb + r * kPLd + c2, gb + (int64_t)r * ld + c2);
      }
    }
  };
  const int chunks = 2 * n;
  stage(0, 0);
  cp_async_commit();
  for (int ch = 0; ch < chunks; ++ch) {
    if (ch + 1 < chunks) stage((ch + 1) & 1, ch + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const double* sa = sm + (ch & 1) * kStageD;
    half_mul<NT>(sa, sa + kNB * kHLd, c);
    __syncthreads();
  }
}

// g = c (MODE 0), -c (1), g - c (2) or g + c (3); row-major tile, leading dimension ld.
template <int MODE>
__device__ __forceinline__ void put_tile(double* g, int64_t ld, const Frag& c) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int mb = 32 * (w >> 1), nb = 32 * (w & 1);
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      double2* q = reinterpret_cast<double2*>(
          g + (int64_t)(mb + 8 * m + (lane >> 2)) * ld + nb + 8 * n + 2 * (lane & 3));
      const double2 o = MODE >= 2 ? *q : make_double2(0.0, 0.0);
      if (MODE == 0) *q = make_double2(c[m][n][0], c[m][n][1]);
      else if (MODE == 1) *q = make_double2(-c[m][n][0], -c[m][n][1]);
      else if (MODE == 2) *q = make_double2(o.x - c[m][n][0], o.y - c[m][n][1]);
      else *q = make_double2(o.x + c[m][n][0], o.y + c[m][n][1]);
    }
}

// Tiles below the diagonal tile p: L_ip = A_ip L_pp^-T = A_ip M_pp^T.
__global__ void __launch_bounds__(kPThreads) k_trsm(double* A, const double* M, int64_t kp, int p) {
  extern __shared__ double sm[];
  const int64_t i = p + 1 + blockIdx.x;
  double* g = A + i * kNB * kp + (int64_t)p * kNB;
  const double* mpp = M + (int64_t)p * kNB * kp + (int64_t)p * kNB;
  Frag c = {};
  tile_sum<true>(sm, 1, [&](int) { return (const double*)g; }, [&](int) { return mpp; }, kp, c);
  put_tile<0>(g, kp, c);
}

// Inside a panel of tile columns [p0, pe): before column p is factored, its tiles i >= p
// receive the panel's earlier columns: A_ip -= sum_{t=p0}^{p-1} L_it L_pt^T.
__global__ void __launch_bounds__(kPThreads)
k_panel_update(double* A, int64_t kp, int p0, int p) {
  extern __shared__ double sm[];
  const int64_t i = p + blockIdx.x;
  Frag c = {};
  const double* rowi = A + i * kNB * kp + (int64_t)p0 * kNB;
  const double* rowp = A + (int64_t)p * kNB * kp + (int64_t)p0 * kNB;
  tile_sum<true>(sm, p - p0, [&](int q) { return rowi + (int64_t)q * kNB; },
                 [&](int q) { return rowp + (int64_t)q * kNB; }, kp, c);
  put_tile<2>(A + i * kNB * kp + (int64_t)p * kNB, kp, c);
}

// Trailing update after the panel [p0, pe): A_ij -= sum_{t=p0}^{pe-1} L_it L_jt^T for the
// lower tiles j <= i < nt with j0 <= j < j1, one read-modify-write per tile. tri: the grid
// enumerates the triangle j0 <= j <= i < nt itself ((nt - j0)(nt - j0 + 1) / 2 CTAs; j1 = nt);
// otherwise rows [j0, nt) by columns [j0, j1) ((nt - j0)(j1 - j0) CTAs, those above the
// diagonal return).
__global__ void __launch_bounds__(kPThreads)
k_syrk(double* A, int64_t kp, int p0, int pe, int j0, int j1, bool tri) {
  extern __shared__ double sm[];
  int64_t i, j;
  if (tri) {                               // blockIdx.x -> (ii, jj), jj <= ii
    const int64_t idx = blockIdx.x;
    int64_t ii = (int64_t)((sqrt(8.0 * (double)idx + 1.0) - 1.0) / 2.0);
    while (ii * (ii + 1) / 2 > idx) --ii;
    while ((ii + 1) * (ii + 2) / 2 <= idx) ++ii;
    i = j0 + ii;
    j = j0 + (idx - ii * (ii + 1) / 2);
  } else {                                 // band of columns: rows x columns
    const int w = j1 - j0;
    i = j0 + blockIdx.x / w;
    j = j0 + blockIdx.x % w;
    if (j > i) return;
  }
  Frag c = {};
  const double* rowi = A + i * kNB * kp + (int64_t)p0 * kNB;
  const double* rowj = A + j * kNB * kp + (int64_t)p0 * kNB;
  tile_sum<true>(sm, pe - p0, [&](int q) { return rowi + (int64_t)q * kNB; },
                 [&](int q) { return rowj + (int64_t)q * kNB; }, kp, c);
  put_tile<2>(A + i * kNB * kp + j * kNB, kp, c);
}

// Off-diagonal tiles of M = L^-1, one row panel [p0, pe) at a time, right after the
// Cholesky has finished that panel. Row i of L M = I gives, for j < i,
//   M_ij = -M_ii sum_{t=j}^{i-1} L_it M_tj.
// The terms with t below the panel arrive early: when panel P is final, k_minv_update adds
// sum_{t in P} L_it M_tj into M_ij for every later row i >= pe and column j < pe (M's lower
// tiles hold these partial sums S_ij until their row is finished); k_minv_row then finishes
// row i of panel P from S_ij and the panel's own earlier rows. The work of the update is
// largest when the Cholesky's trailing update has become small, so the two share the GPU.

// Row i of the panel that starts at p0: M_ij for every j < i (one CTA per j).
__global__ void __launch_bounds__(kPThreads)
k_minv_row(const double* A, double* M, int64_t kp, int p0, int i) {
  extern __shared__ double sm[];
  const int64_t j = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int mb = 32 * (w >> 1), nb = 32 * (w & 1);
  Frag c;
  double* g = M + (int64_t)i * kNB * kp + j * kNB;
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      double2 v = make_double2(0.0, 0.0);    // S_ij from the earlier panels (none for j >= p0)
      if (j < p0)
        v = *reinterpret_cast<const double2*>(
            g + (int64_t)(mb + 8 * m + (lane >> 2)) * kp + nb + 8 * n + 2 * (lane & 3));
      c[m][n][0] = v.x;
      c[m][n][1] = v.y;
    }
  const int64_t t0 = j > p0 ? j : p0;      // this panel's rows t in [max(j, p0), i)
  tile_sum<false>(sm, (int)(i - t0),
                  [&](int q) { return A + (int64_t)i * kNB * kp + (t0 + q) * kNB; },
                  [&](int q) { return (const double*)(M + (t0 + q) * kNB * kp + j * kNB); }, kp,
                  c);
  // M_ij = -M_ii X, X = c: X through shared memory, M_ii staged beside it
  double* xs = sm + kNB * kPLd;
#pragma unroll
  for (int m = 0; m < 4; ++m)
#pragma unroll
    for (int n = 0; n < 4; ++n)
      *reinterpret_cast<double2*>(xs + (mb + 8 * m + (lane >> 2)) * kPLd + nb + 8 * n +
                                  2 * (lane & 3)) = make_double2(c[m][n][0], c[m][n][1]);
  stage_async(sm, M + (int64_t)i * kNB * kp + (int64_t)i * kNB, kp);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  Frag d = {};
  tile_mul<false>(sm, xs, d);
  put_tile<1>(g, kp, d);
}

// After the rows of panel [p0, pe) are final: S_ij += sum_{t = max(j, p0)}^{pe-1} L_it M_tj
// for rows pe <= i < nt and columns j < pe (the first contribution to a tile, j >= p0,
// writes it).
__global__ void __launch_bounds__(kPThreads)
k_minv_update(const double* A, double* M, int64_t kp, int p0, int pe) {
  extern __shared__ double sm[];
  const int64_t i = pe + blockIdx.x / pe, j = blockIdx.x % pe;
  const int64_t t0 = j > p0 ? j : p0;
  Frag c = {};
  tile_sum<false>(sm, (int)(pe - t0),
                  [&](int q) { return A + i * kNB * kp + (t0 + q) * kNB; },
                  [&](int q) { return (const double*)(M + (t0 + q) * kNB * kp + j * kNB); }, kp,
                  c);
  double* g = M + i * kNB * kp + j * kNB;
  if (j >= p0) put_tile<0>(g, kp, c);
  else put_tile<3>(g, kp, c);
}

// U_pq = fl32(M_{k-1-p, k-1-q}) for q >= p, else 0.
__global__ void k_factor_store(FactorArgs a) {
  const int64_t total = a.k * a.k;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = e / a.k, q = e % a.k;
    a.U[e] = q >= p ? (float)a.M[(a.k - 1 - p) * a.kp + (a.k - 1 - q)] : 0.0f;
  }
}

}  // namespace

namespace {
// Three streams and events for the factor's and the sweep's look-ahead, one set per device,
// created on first use; calls on one device enqueue under its mutex. chain (the highest
// priority) carries the panel factorisations, side the bulk trailing updates, inv (the
// lowest) the factor's row panels of L^-1, so the block scheduler serves the serial chain
// first, then the updates the chain waits for, and fills the rest with the inverse.
constexpr int kEvRing = 1024;
struct FactorStreams {
  std::mutex mu;
  cudaStream_t chain = nullptr, side = nullptr, inv = nullptr;
  cudaEvent_t ring[kEvRing] = {};
  int next = 0;
  // a fresh event for each record, so that no event is recorded again while an earlier wait
  // on it may still be queued
  cudaEvent_t take() {
    cudaEvent_t e = ring[next];
    next = (next + 1) % kEvRing;
    return e;
  }
};
// The current device's three streams and seven events, created on first use; *err is set (and
// nothing kept, so that a later call tries again) when any of them cannot be created.
FactorStreams& factor_streams(cudaError_t* err) {
  static FactorStreams fs[64];
  static std::mutex init_mu;
  int dev = 0;
  cudaGetDevice(&dev);
  FactorStreams& f = fs[dev < 0 || dev >= 64 ? 0 : dev];
  std::lock_guard<std::mutex> lk(init_mu);
  *err = cudaSuccess;
  if (!f.side) {
    int least = 0, greatest = 0;
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    // greatest is the numerically smallest; side sits between the two when the range allows
    const int mid = least - greatest >= 2 ? (least + greatest) / 2 : least;
    cudaStream_t chain = nullptr, side = nullptr, inv = nullptr;
    cudaEvent_t ev[kEvRing] = {};
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&chain, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&side, cudaStreamNonBlocking, mid);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&inv, cudaStreamNonBlocking, least);
    for (int i = 0; i < kEvRing && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (cudaEvent_t x : ev)
        if (x) cudaEventDestroy(x);
      if (inv) cudaStreamDestroy(inv);
      if (side) cudaStreamDestroy(side);
      if (chain) cudaStreamDestroy(chain);
      *err = e;
      return f;
    }
    f.chain = chain;
    f.inv = inv;
    for (int i = 0; i < kEvRing; ++i) f.ring[i] = ev[i];
    f.side = side;                          // last: marks the set complete
  }
  return f;
}
}  // namespace

size_t gptq_factor_workspace(int64_t k) {
  const int64_t kp = (k + kNB - 1) / kNB * kNB;
  return 256 + 2 * (size_t)kp * (size_t)kp * sizeof(double);
}

cudaError_t launch_gptq_factor(const float* H, int64_t k, int B, const int32_t* perm,
                               double damp, float* U, void* ws, cudaStream_t st) {
  for (const void* f : {(const void*)k_trsm, (const void*)k_syrk, (const void*)k_panel_update,
                        (const void*)k_minv_row, (const void*)k_minv_update}) {
    const cudaError_t ae = ensure_dynamic_smem(f, (int)kProdSmem);
    if (ae != cudaSuccess) return ae;
  }
  const int64_t kp = (k + kNB - 1) / kNB * kNB, nt = kp / kNB;
  char* w = (char*)ws;
  FactorArgs a{H, k, kp, B, perm, (double*)(w + 256), (double*)(w + 256) + kp * kp,
               (double*)w, U};
  const int gs = sm_count() * 8;
  // Right-looking over panels of kPanelTiles tile columns, left-looking inside a panel, with
  // a look-ahead of one panel: after panel P is factored (stream chain), its update of the
  // next panel's columns runs on chain, its update of everything beyond on side while chain
  // factors panel P + 1; panel P + 1's column update waits for the previous panel's update
  // of everything beyond (both write those tiles). Panel P's rows of L^-1 and their
  // contributions to the later rows run on inv as soon as chain has factored it (they read
  // only final tiles of L and write only M). The three streams fork from and join the
  // caller's stream.
  cudaError_t serr = cudaSuccess;
  FactorStreams& fs = factor_streams(&serr);
  if (serr != cudaSuccess) return serr;
  std::lock_guard<std::mutex> lk(fs.mu);
  cudaStream_t cs = fs.chain;
  cudaEvent_t e0 = fs.take();
  cudaEventRecord(e0, st);
  cudaStreamWaitEvent(cs, e0, 0);
  cudaStreamWaitEvent(fs.side, e0, 0);
  cudaStreamWaitEvent(fs.inv, e0, 0);
  cudaEvent_t ev_rest = nullptr;
  k_factor_lambda<<<1, kFThreads, 0, cs>>>(H, k, damp, a.scal);
  k_factor_load<<<gs, 256, 0, cs>>>(a);
  bool rest_pending = false;
  for (int p0 = 0; p0 < nt; p0 += kPanelTiles) {
    const int pe = (int)(p0 + kPanelTiles < nt ? p0 + kPanelTiles : nt);
    for (int p = p0; p < pe; ++p) {
      if (p > p0) k_panel_update<<<(unsigned)(nt - p), kPThreads, kProdSmem, cs>>>(a.A, kp, p0, p);
      k_potrf_inv<<<1, kFThreads, 0, cs>>>(a.A, a.M, kp, p);
      if (nt - 1 - p > 0)
        k_trsm<<<(unsigned)(nt - 1 - p), kPThreads, kProdSmem, cs>>>(a.A, a.M, kp, p);
    }
    {
      cudaEvent_t ec = fs.take();
      cudaEventRecord(ec, cs);
      cudaStreamWaitEvent(fs.inv, ec, 0);
    }
    for (int i = (p0 > 1 ? p0 : 1); i < pe; ++i)
      k_minv_row<<<(unsigned)i, kPThreads, kProdSmem, fs.inv>>>(a.A, a.M, kp, p0, i);
    if (pe < nt)
      k_minv_update<<<(unsigned)((nt - pe) * pe), kPThreads, kProdSmem, fs.inv>>>(a.A, a.M, kp,
                                                                                 p0, pe);
    if (pe >= nt) break;
    const int pn = (int)(pe + kPanelTiles < nt ? pe + kPanelTiles : nt);   // next panel's end
    if (rest_pending) cudaStreamWaitEvent(cs, ev_rest, 0);
    k_syrk<<<(unsigned)((nt - pe) * (pn - pe)), kPThreads, kProdSmem, cs>>>(a.A, kp, p0, pe, pe,
                                                                            pn, false);
    rest_pending = false;
    if (pn < nt) {
      cudaEvent_t ep = fs.take();
      cudaEventRecord(ep, cs);
      cudaStreamWaitEvent(fs.side, ep, 0);
      const int64_t m = nt - pn;
      k_syrk<<<(unsigned)(m * (m + 1) / 2), kPThreads, kProdSmem, fs.side>>>(a.A, kp, p0, pe, pn,
                                                                              (int)nt, true);
      ev_rest = fs.take();
      cudaEventRecord(ev_rest, fs.side);
      rest_pending = true;
    }
  }
  cudaEvent_t e_end = fs.take(), e_inv = fs.take();
  cudaEventRecord(e_end, fs.side);
  cudaEventRecord(e_inv, fs.inv);
  cudaStreamWaitEvent(cs, e_end, 0);
  cudaStreamWaitEvent(cs, e_inv, 0);
  k_factor_store<<<gs, 256, 0, cs>>>(a);
  cudaEvent_t e_done = fs.take();
  cudaEventRecord(e_done, cs);
  cudaStreamWaitEvent(st, e_done, 0);
  return cudaGetLastError();
}

// ======================================================================================
// sweep
// ======================================================================================
namespace {

constexpr int kPanel = 64;               // positions per panel
constexpr int kTrRows = 8;               // rows per thread of the trailing update
constexpr int kTrailThreads = 16 * (64 / kTrRows);   // 64 rows x 64 positions per CTA

struct SweepArgs {
  const char* W;
  int64_t n, k, ld_bytes;
  int bf16;
  const float* h;
  const float* U;        // [k][k], sweep order
  const int32_t* perm;   // [k / B] or null
  int window;
  float* Wc;             // [n][k] working weights, sweep order
  float* Err;            // 2 x [n][kPanel]: the residuals of alternate panels
  uint8_t* codes;        // [n][k / 2]
  uint8_t* scales;       // [n][k / B]
};

template <int B>
__device__ __forceinline__ int64_t pos_col(const SweepArgs& a, int64_t pos) {
  if (!a.perm) return pos;
  const int64_t b = min(max((int64_t)a.perm[pos / B], (int64_t)0), a.k / B - 1);
  return b * B + pos % B;
}

template <int B>
__global__ void k_sweep_init(SweepArgs a) {
  const int64_t total = a.n * a.k;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / a.k, pos = e % a.k;
    const int64_t c = pos_col<B>(a, pos);
    const char* row = a.W + r * a.ld_bytes;
    a.Wc[e] = a.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(row)[c])
                     : reinterpret_cast<const float*>(row)[c];
  }
}

// Element step of the definition at scale t = {s, r_hi, r_lo}: the magnitude code q and
// fl32(s g(q)) for a = |w| (q = 0 for a zero scale).
template <int ELEM>
__device__ __forceinline__ int elem_project(float a, float4 t, float& wq_abs) {
  if (t.x == 0.0f) {
    wq_abs = 0.0f;
    return 0;
  }
  const float2 z = quot2(make_float2(a, 0.0f), t);
  const float g = elem_values<ELEM>(z).x;
  wq_abs = __fmul_rn(t.x, g);
  if constexpr (ELEM == kElemE2M1) return (int)(e2m1x2_rn(z.x, 0.0f) & 7u);
  else return (int)g;
}

// fl32(s g(q)) of two magnitudes at scale t = {s, r_hi, r_lo} (0 for a zero scale): the
// element step of the definition for a pair of elements at once.
template <int ELEM>
__device__ __forceinline__ float2 pair_project(float2 a, float4 t) {
  const float2 g = elem_values<ELEM>(quot2(a, t));
  const float2 wq = __fmul2_rn(make_float2(t.x, t.x), g);
  return t.x == 0.0f ? make_float2(0.0f, 0.0f) : wq;
}

// The definition's candidate error sum_j c_j (w_j - wq_j)^2 of one block (magnitudes in wb,
// h weights in cw): double, element order, each operation rounded once. |w| - wq is the
// negation of w - copysign(wq, w) for a negative w, so its square is the same double.
template <int B, int ELEM, bool HOPT>
__device__ __forceinline__ double exact_error1(const float* wb, const float* cw, float4 t) {
  double e = 0.0;
#pragma unroll 4
  for (int j = 0; j < B; j += 2) {
    const float2 av = make_float2(fabsf(wb[j]), fabsf(wb[j + 1]));
    const float2 wq = pair_project<ELEM>(av, t);
    const double d0 = __dsub_rn((double)av.x, (double)wq.x);
    const double d1 = __dsub_rn((double)av.y, (double)wq.y);
    const double s0 = __dmul_rn(d0, d0), s1 = __dmul_rn(d1, d1);
    e = __dadd_rn(e, HOPT ? __dmul_rn((double)cw[j], s0) : s0);
    e = __dadd_rn(e, HOPT ? __dmul_rn((double)cw[j + 1], s1) : s1);
  }
  return e;
}

constexpr int kPanWinBelow = 8;          // the full-scored window starts this far below naive

// Two rows per warp, one per half-warp: lane l of half f (l = lane & 15) holds panel
// positions 4l .. 4l + 3 of row 2 w + f, so that the per-column chain (projection, division,
// broadcast), which leaves all but one lane of a row waiting, serves two rows per
// instruction. Each block's scale search is exact (float64, element order, the split-
// reciprocal quotient that equals the IEEE one; the lowest code on ties) but scores in full
// only a window of 32 codes from 8 below the naive code (two per lane); every other code gets
// a lower bound from the block's two elements with the largest c a^2 -- the same double terms
// its full sum would add, so the bound less 2^-45 relative lies below that sum -- and only
// codes whose bound does not exceed the best error so far are listed and scored in full.
constexpr int kPanelWarpsH = 2;          // warps per CTA (four rows)

// Smallest error within each half-warp, the lowest code among equal errors.
__device__ __forceinline__ void half_argmin(double& be, int& bc) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    const double oe = __shfl_xor_sync(kFull, be, o);
    const int oc = __shfl_xor_sync(kFull, bc, o);
    if (oe < be || (oe == be && oc < bc)) { be = oe; bc = oc; }
  }
}

template <int B, int ELEM, int MODE>
__global__ void __launch_bounds__(kPanelWarpsH * 32)
k_gptq_panel(SweepArgs a, GridTable T, int64_t p0, int S, float* __restrict__ Err) {
  __shared__ float4 tab[256];
  __shared__ float Us[kPanel][kPanel + 1];
  __shared__ float hs[kPanel];
  __shared__ float wb[kPanelWarpsH][2][32];
  __shared__ float errs[kPanelWarpsH][2][32];
  __shared__ uint8_t surv[kPanelWarpsH][2][256];   // codes left after the bounds, ascending
  for (int c = threadIdx.x; c < T.ncodes; c += blockDim.x) tab[c] = T.c[c];
  for (int e = threadIdx.x; e < kPanel * kPanel; e += blockDim.x) {
    const int i = e / kPanel, j = e % kPanel;
    Us[i][j] = (i < S && j < S) ? a.U[(p0 + i) * a.k + p0 + j] : 0.0f;
  }
  for (int i = threadIdx.x; i < kPanel; i += blockDim.x)
    hs[i] = (MODE == 2 && i < S) ? a.h[pos_col<B>(a, p0 + i)] : 1.0f;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int hf = lane >> 4, sl = lane & 15;
  const int64_t r = (int64_t)blockIdx.x * (2 * kPanelWarpsH) + 2 * wid + hf;
  const bool row_ok = r < a.n;
  if (__ballot_sync(kFull, row_ok) == 0) return;   // both of the warp's rows past the end
  const int64_t kb = a.k / B;
  const bool live = row_ok && 4 * sl < S;
  float w[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    const float4 v = *reinterpret_cast<const float4*>(a.Wc + r * a.k + p0 + 4 * sl);
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
  }
  float errv[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t nib = 0;                       // the lane's four nibbles
  float* wbh = wb[wid][hf];
  float* erh = errs[wid][hf];
  uint8_t* svh = surv[wid][hf];
  for (int bb = 0; bb * B < S; ++bb) {
    const int q0 = bb * B;                // the block's first panel position
    const bool mine = 4 * sl >= q0 && 4 * sl < q0 + B;
    if (mine) {
#pragma unroll
      for (int c = 0; c < 4; ++c) wbh[4 * sl - q0 + c] = w[c];
    }
    __syncwarp();
    float amax = 0.0f;
#pragma unroll 4
    for (int j = 0; j < B; ++j) amax = fmaxf(amax, fabsf(wbh[j]));
    const int c0 = naive_code<ELEM>(amax, tab, T.ncodes, T.sfmt);
    int cbest = c0;
    if (MODE != 0) {
      int lo, hi;
      grid_window(tab, T.ncodes, T.first, c0, a.window, lo, hi);
      // (1) a window of 32 codes from just below the naive code, two per lane, in full
      const int ws = max(lo, min(c0 - kPanWinBelow, hi - 31)), we = min(hi, ws + 31);
      double be = __longlong_as_double(0x7ff0000000000000LL);   // +inf
      int bc = 0x7fffffff;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int c = ws + sl + 16 * t;
        if (c <= we) {
          const double e = exact_error1<B, ELEM, MODE == 2>(wbh, hs + q0, tab[c]);
          if (e < be) { be = e; bc = c; }
        }
      }
      half_argmin(be, bc);
      // (2) the codes outside the window, by the two-element bounds; the loop runs over the
      // union of both halves' ranges so that every lane takes part in the ballots
      const bool need = lo < ws || we < hi;
      if (__any_sync(kFull, need)) {
        float2 top = make_float2(0.f, 0.f), ctop = make_float2(0.f, 0.f);
        {
          float v1 = -1.f, v2 = -1.f;
          for (int j = 0; j < B; ++j) {
            const float aj = fabsf(wbh[j]), cj = MODE == 2 ? hs[q0 + j] : 1.f;
            const float v = cj * aj * aj;
            if (v > v1) { v2 = v1; top.y = top.x; ctop.y = ctop.x; v1 = v; top.x = aj; ctop.x = cj; }
            else if (v > v2) { v2 = v; top.y = aj; ctop.y = cj; }
          }
        }
        const double bound_cut = be;
        const int lo_u = min(lo, __shfl_xor_sync(kFull, lo, 16));
        const int hi_u = max(hi, __shfl_xor_sync(kFull, hi, 16));
        int total = 0;
        for (int cb = lo_u; cb <= hi_u; cb += 16) {
          const int c = cb + sl;
          const bool in = need && c >= lo && c <= hi && (c < ws || c > we);
          bool keep = false;
          if (in) {
            const float2 wq = pair_project<ELEM>(top, tab[c]);
            const double d0 = __dsub_rn((double)top.x, (double)wq.x);
            const double d1 = __dsub_rn((double)top.y, (double)wq.y);
            const double s0 = __dmul_rn(d0, d0), s1 = __dmul_rn(d1, d1);
            const double lb = __dadd_rn(MODE == 2 ? __dmul_rn((double)ctop.x, s0) : s0,
                                        MODE == 2 ? __dmul_rn((double)ctop.y, s1) : s1);
            keep = !(lb * (1.0 - 0x1p-45) > bound_cut);
          }
          const unsigned m = (__ballot_sync(kFull, keep) >> (16 * hf)) & 0xffffu;
          if (keep) svh[total + __popc(m & ((1u << sl) - 1u))] = (uint8_t)c;
          total += __popc(m);
        }
        __syncwarp();
        // (3) the survivors in full, 16 at a time per row
        for (int i = sl; i < total; i += 16) {
          const int c = svh[i];
          const double e = exact_error1<B, ELEM, MODE == 2>(wbh, hs + q0, tab[c]);
          if (e < be || (e == be && c < bc)) { be = e; bc = c; }
        }
        half_argmin(be, bc);
        __syncwarp();
      }
      cbest = bc == 0x7fffffff ? lo : bc;
    }
    const float4 t = tab[cbest];
    const int64_t blk = pos_col<B>(a, p0 + q0) / B;   // the block's index in W
    if (row_ok && sl == 0) a.scales[r * kb + blk] = (uint8_t)cbest;
    // the block's columns, one after another (the owner lane of each row divides, the
    // residual is broadcast within the half)
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int q = q0 + j;
      const int owner = q >> 2;
      const int comp = j & 3;             // q0 is a multiple of 4: q & 3 == j & 3
      float err = 0.0f;
      if (sl == owner) {
        const float wv = w[comp];
        float wq_abs;
        const int code = elem_project<ELEM>(fabsf(wv), t, wq_abs);
        const uint32_t neg = __float_as_uint(wv) >> 31;
        const uint32_t nb = ELEM == kElemE2M1 ? ((neg << 3) | (uint32_t)code)
                                              : ((uint32_t)(neg ? -code : code) & 15u);
        nib |= nb << (4 * comp);
        err = __fdiv_rn(__fsub_rn(wv, copysignf(wq_abs, wv)), Us[q][q]);
        errv[comp] = err;
        erh[j] = err;
      }
      err = __shfl_sync(kFull, err, (lane & 16) | owner);
      // in-block updates of the later columns: w -= fl32(err U)
      if (mine) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (4 * sl + c > q) w[c] = __fsub_rn(w[c], __fmul_rn(err, Us[q][4 * sl + c]));
      }
    }
    __syncwarp();
    // the block's product into the panel's later blocks: acc = sum_j fma, one subtraction
    if (live && 4 * sl >= q0 + B) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int j = 0; j < B; ++j) {
        const float e = erh[j];
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[c] = __fmaf_rn(e, Us[q0 + j][4 * sl + c], acc[c]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) w[c] = __fsub_rn(w[c], acc[c]);
    }
    __syncwarp();
  }
  if (live) {
    const int64_t c = pos_col<B>(a, p0 + 4 * sl);     // four positions of one block
    *reinterpret_cast<uint16_t*>(a.codes + r * (a.k / 2) + c / 2) = (uint16_t)nib;
    *reinterpret_cast<float4*>(Err + r * kPanel + 4 * sl) =
        make_float4(errv[0], errv[1], errv[2], errv[3]);
  }
}

// Later positions p in [cbeg, cend) (after the panel [p0, p0 + S)): for each block of the
// panel (in order) acc = sum_j fma(err_j, U[j][p], acc) over the block's columns, then
// w -= acc. CTA: 64 positions x rg groups of 64 rows; thread: kTrRows rows (ty, ty + 64 /
// kTrRows, ...: the rows a warp reads at once sit in different banks) x 4 consecutive
// positions, as paired float32 FMAs (fma.rn.f32x2: two FMAs per instruction, each rounded
// on its own). The CTA's rows of U are staged once; the residuals of the next row group are
// fetched with cp.async while the current group is updated, and read four columns at a
// time (one 16-byte load per row feeds 8 FMAs per position pair).
constexpr int kEsLd = kPanel + 4;        // padded residual row (16-byte aligned)
constexpr size_t kTrailSmem = (2 * 64 * kEsLd + kPanel * 64) * sizeof(float);

__device__ __forceinline__ void cp_async16f(float* s, const float* g) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(s);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(a), "l"(g) : "memory");
}

template <int B>
__global__ void __launch_bounds__(kTrailThreads)
k_gptq_trailing(SweepArgs a, const float* __restrict__ Err, int64_t p0, int S, int64_t cbeg,
                int64_t cend, int rg) {
  extern __shared__ __align__(16) float tsm[];
  float (*Es)[64 * kEsLd] = reinterpret_cast<float (*)[64 * kEsLd]>(tsm);
  float (*Ut)[64] = reinterpret_cast<float (*)[64]>(tsm + 2 * 64 * kEsLd);
  constexpr int kRs = 64 / kTrRows;      // row stride of a thread's rows
  const int64_t c0 = cbeg + (int64_t)blockIdx.x * 64;
  const int64_t groups = (a.n + 63) / 64;
  const int64_t g0 = (int64_t)blockIdx.y * rg;
  const int ng = (int)(groups - g0 < rg ? groups - g0 : rg);
  auto stage_es = [&](int buf, int64_t r0) {
    for (int e = threadIdx.x; e < 64 * (kPanel / 4); e += kTrailThreads) {
      const int i = e / (kPanel / 4), q = e % (kPanel / 4);
      if (r0 + i < a.n) cp_async16f(&Es[buf][i * kEsLd + 4 * q], Err + (r0 + i) * kPanel + 4 * q);
    }
  };
  stage_es(0, g0 * 64);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  for (int e = threadIdx.x; e < kPanel * 16; e += kTrailThreads) {
    const int j = e / 16, g = e % 16;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < S && c0 + 4 * g < cend)
      u = *reinterpret_cast<const float4*>(a.U + (p0 + j) * a.k + c0 + 4 * g);
    *reinterpret_cast<float4*>(&Ut[j][4 * g]) = u;
  }
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t col = c0 + 4 * tx;
  const bool on = col < cend;
  for (int g = 0; g < ng; ++g) {
    const int64_t r0 = (g0 + g) * 64;
    if (g + 1 < ng) stage_es((g + 1) & 1, r0 + 64);
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    float2 w[kTrRows][2];
#pragma unroll
    for (int i = 0; i < kTrRows; ++i) {
      const int64_t r = r0 + ty + kRs * i;
      const float4 v = (on && r < a.n) ? *reinterpret_cast<const float4*>(a.Wc + r * a.k + col)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      w[i][0] = make_float2(v.x, v.y);
      w[i][1] = make_float2(v.z, v.w);
    }
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    __syncthreads();
    const float* E = Es[g & 1] + ty * kEsLd;
    for (int q0 = 0; q0 < S; q0 += B) {
      float2 acc[kTrRows][2];
#pragma unroll
      for (int i = 0; i < kTrRows; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j4 = 0; j4 < B; j4 += 4) {
        float4 e[kTrRows];
#pragma unroll
        for (int i = 0; i < kTrRows; ++i)
          e[i] = *reinterpret_cast<const float4*>(E + kRs * i * kEsLd + q0 + j4);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float4 u = *reinterpret_cast<const float4*>(&Ut[q0 + j4 + jj][4 * tx]);
          const float2 ua = make_float2(u.x, u.y), ub = make_float2(u.z, u.w);
#pragma unroll
          for (int i = 0; i < kTrRows; ++i) {
            const float ev = jj == 0 ? e[i].x : jj == 1 ? e[i].y : jj == 2 ? e[i].z : e[i].w;
            const float2 e2 = make_float2(ev, ev);
            acc[i][0] = __ffma2_rn(e2, ua, acc[i][0]);
            acc[i][1] = __ffma2_rn(e2, ub, acc[i][1]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kTrRows; ++i) {   // w - acc, as w + (-acc): the same rounding
        w[i][0] = __fadd2_rn(w[i][0], make_float2(-acc[i][0].x, -acc[i][0].y));
        w[i][1] = __fadd2_rn(w[i][1], make_float2(-acc[i][1].x, -acc[i][1].y));
      }
    }
#pragma unroll
    for (int i = 0; i < kTrRows; ++i) {
      const int64_t r = r0 + ty + kRs * i;
      if (on && r < a.n)
        *reinterpret_cast<float4*>(a.Wc + r * a.k + col) =
            make_float4(w[i][0].x, w[i][0].y, w[i][1].x, w[i][1].y);
    }
    __syncthreads();                      // Es[g & 1] is refilled two groups later
  }
}

template <int B>
void launch_trailing(const SweepArgs& a, const float* Err, int64_t p0, int S, int64_t cbeg,
                     int64_t cend, cudaStream_t st) {
  // row groups per CTA: as many as keep at least ~4 CTAs per SM
  const int64_t ctiles = (cend - cbeg + 63) / 64, groups = (a.n + 63) / 64;
  int64_t rg = ctiles * groups / ((int64_t)sm_count() * 4);
  rg = rg < 1 ? 1 : (rg > 8 ? 8 : rg);
  const dim3 grid((unsigned)ctiles, (unsigned)((groups + rg - 1) / rg));
  k_gptq_trailing<B><<<grid, kTrailThreads, kTrailSmem, st>>>(a, Err, p0, S, cbeg, cend, (int)rg);
}

// Panels of 64 positions with a look-ahead of one panel, as the factor: panel t's update of
// the next 64 positions runs on the chain stream (the next panel needs only those), its
// update of everything beyond on the side stream while the chain runs panel t + 1; the
// residuals alternate between two buffers, and the next-64 update of panel t + 1 waits for
// panel t's update beyond (both write those positions).
template <int B, int ELEM>
cudaError_t sweep_dispatch(const SweepArgs& a, const GridTable& T, int mode, cudaStream_t st) {
  const cudaError_t ae = ensure_dynamic_smem((const void*)k_gptq_trailing<B>, (int)kTrailSmem);
  if (ae != cudaSuccess) return ae;
  cudaError_t serr = cudaSuccess;
  FactorStreams& fs = factor_streams(&serr);
  if (serr != cudaSuccess) return serr;
  std::lock_guard<std::mutex> lk(fs.mu);
  cudaStream_t cs = fs.chain;
  cudaEvent_t e0 = fs.take();
  cudaEventRecord(e0, st);
  cudaStreamWaitEvent(cs, e0, 0);
  cudaStreamWaitEvent(fs.side, e0, 0);
  cudaEvent_t ev_rest = nullptr;
  k_sweep_init<B><<<sm_count() * 8, 256, 0, cs>>>(a);
  const unsigned prow = (unsigned)((a.n + 2 * kPanelWarpsH - 1) / (2 * kPanelWarpsH));
  bool rest_pending = false;
  int t = 0;
  for (int64_t p0 = 0; p0 < a.k; p0 += kPanel, ++t) {
    const int S = (int)(a.k - p0 < kPanel ? a.k - p0 : kPanel);
    float* err = a.Err + (t & 1) * a.n * kPanel;
    if (mode == 0) k_gptq_panel<B, ELEM, 0><<<prow, kPanelWarpsH * 32, 0, cs>>>(a, T, p0, S, err);
    else if (mode == 1) k_gptq_panel<B, ELEM, 1><<<prow, kPanelWarpsH * 32, 0, cs>>>(a, T, p0, S, err);
    else k_gptq_panel<B, ELEM, 2><<<prow, kPanelWarpsH * 32, 0, cs>>>(a, T, p0, S, err);
    const int64_t c1 = p0 + S, c2 = c1 + kPanel < a.k ? c1 + kPanel : a.k;
    if (c1 >= a.k) break;
    if (rest_pending) cudaStreamWaitEvent(cs, ev_rest, 0);
    launch_trailing<B>(a, err, p0, S, c1, c2, cs);
    rest_pending = false;
    if (c2 < a.k) {
      cudaEvent_t ep = fs.take();
      cudaEventRecord(ep, cs);
      cudaStreamWaitEvent(fs.side, ep, 0);
      launch_trailing<B>(a, err, p0, S, c2, a.k, fs.side);
      ev_rest = fs.take();
      cudaEventRecord(ev_rest, fs.side);
      rest_pending = true;
    }
  }
  cudaEvent_t e_end = fs.take(), e_done = fs.take();
  cudaEventRecord(e_end, fs.side);
  cudaStreamWaitEvent(cs, e_end, 0);
  cudaEventRecord(e_done, cs);
  cudaStreamWaitEvent(st, e_done, 0);
  return cudaGetLastError();
}

}  // namespace

size_t gptq_sweep_workspace(int64_t n, int64_t k) {
  return (size_t)n * (size_t)k * sizeof(float) + 2 * (size_t)n * kPanel * sizeof(float) + 256;
}

cudaError_t launch_gptq_sweep(const GptqArgs& g, cudaStream_t st) {
  static const GridTable tables[4] = {make_grid_table(0), make_grid_table(1),
                                      make_grid_table(2), make_grid_table(3)};
  char* ws = (char*)g.workspace;
  SweepArgs a{(const char*)g.W, g.n, g.k, g.ld * (g.dtype == 1 ? 2 : 4), g.dtype == 1, g.h,
              g.U, g.perm, g.window, (float*)ws, (float*)(ws + (size_t)g.n * g.k * sizeof(float)),
              (uint8_t*)g.codes, (uint8_t*)g.scales};
  const GridTable& T = tables[g.scale_fmt];
  if (g.fmt == 0) {
    return g.block == 16 ? sweep_dispatch<16, kElemE2M1>(a, T, g.mode, st)
                         : sweep_dispatch<32, kElemE2M1>(a, T, g.mode, st);
  }
  return g.block == 16 ? sweep_dispatch<16, kElemInt4>(a, T, g.mode, st)
                       : sweep_dispatch<32, kElemInt4>(a, T, g.mode, st);
}

// ======================================================================================
// order (ordered variant)
// ======================================================================================
namespace {

constexpr int kLossThreads = 256;
constexpr int kSortMax = 2048;           // blocks a single-CTA sort handles

struct LossArgs {
  const char* W;
  int64_t n, k, ld_bytes;
  int bf16, fmt, block;
  const float* h;
  const uint8_t* codes;
  const uint8_t* scales;
  GridTable T;
  double* loss;          // [k / B]
};

// loss_b = sum over rows and the block's columns of h_j (w_ij - w^_ij)^2 (double), one CTA
// per block: each thread sums its rows' blocks (columns in order), then a fixed tree.
__global__ void __launch_bounds__(kLossThreads) k_block_loss(LossArgs a) {
  __shared__ double part[kLossThreads];
  const int64_t b = blockIdx.x, kb = a.k / a.block;
  double acc = 0.0;
  for (int64_t r = threadIdx.x; r < a.n; r += kLossThreads) {
    const float s = a.T.c[a.scales[r * kb + b]].x;
    const char* row = a.W + r * a.ld_bytes;
    double e = 0.0;
    for (int j = 0; j < a.block; ++j) {
      const int64_t c = b * a.block + j;
      const float w = a.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(row)[c])
                             : reinterpret_cast<const float*>(row)[c];
      const uint32_t nib = (a.codes[r * (a.k / 2) + c / 2] >> (4 * (c & 1))) & 15u;
      float g;
      if (a.fmt == 0) {
        g = __half2float(__ushort_as_half((uint16_t)(e2m1x2_to_f16x2(nib & 7u) & 0xffffu)));
        if (nib & 8u) g = -g;
      } else {
        g = (float)((nib & 8u) ? (int)nib - 16 : (int)nib);
      }
      const double d = __dsub_rn((double)w, (double)__fmul_rn(s, g));
      e = __dadd_rn(e, __dmul_rn(__dmul_rn(d, d), (double)a.h[c]));
    }
    acc = __dadd_rn(acc, e);
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kLossThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) a.loss[b] = part[0];
}

// perm = blocks by descending loss, the lower block first on equal loss (bitonic sort).
__global__ void __launch_bounds__(1024) k_block_sort(const double* loss, int kb, int32_t* perm) {
  __shared__ double key[kSortMax];
  __shared__ int32_t idx[kSortMax];
  int m = 1;
  while (m < kb) m <<= 1;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    key[i] = i < kb ? loss[i] : -__longlong_as_double(0x7ff0000000000000LL);
    idx[i] = i < kb ? i : 0x7fffffff;
  }
  __syncthreads();
  // "before(x, y)": x sorts first (larger loss, then smaller index)
  for (int size = 2; size <= m; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < m; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const bool before_j = key[j] > key[i] || (key[j] == key[i] && idx[j] < idx[i]);
          if (before_j == up) {
            const double tk = key[i]; key[i] = key[j]; key[j] = tk;
            const int32_t ti = idx[i]; idx[i] = idx[j]; idx[j] = ti;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < kb; i += blockDim.x) perm[i] = idx[i];
}

}  // namespace

cudaError_t launch_gptq_order(const GptqArgs& g, const uint8_t* codes, const uint8_t* scales,
                              double* loss, int32_t* perm, cudaStream_t st) {
  static const GridTable tables[4] = {make_grid_table(0), make_grid_table(1),
                                      make_grid_table(2), make_grid_table(3)};
  const int64_t kb = g.k / g.block;
  LossArgs a{(const char*)g.W, g.n, g.k, g.ld * (g.dtype == 1 ? 2 : 4), g.dtype == 1, g.fmt,
             g.block, g.h, codes, scales, tables[g.scale_fmt], loss};
  k_block_loss<<<(unsigned)kb, kLossThreads, 0, st>>>(a);
  k_block_sort<<<1, 1024, 0, st>>>(loss, (int)kb, perm);
  return cudaGetLastError();
}

int gptq_sort_max() { return kSortMax; }

}  // namespace mxq
