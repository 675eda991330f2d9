// mxq_hpass.cu -- h_j = E_r[x_rj^2]: a streaming column reduction over the calibration
// activations ("quantization_algorithms.txt", sec. 1: the diagonal weights h_j = E[x_j^2]).
//
// HBM-bound: every byte of X is read once. Each warp owns a strip of 32 x 16-byte
// columns (256 bf16 or 128 f32 columns) and one of 8 interleaved row phases of a row
// chunk; each lane keeps its 8 (or 4) columns' running sums. Loads are 128-bit,
// non-caching in L1, eight rows in flight per lane; the grid is one wave of resident
// CTAs (strips x row chunks <= 148 SMs x 3). Squares accumulate in float32 (packed
// f32x2 FMA) for at most 32 rows, then fold into double, so the column sum carries at
// most ~32 float roundings (relative error <= 2e-6); the 8 row phases and the row chunks
// are combined in double in a fixed order, which makes the result deterministic.
#include "mxq_common.cuh"
#include "mxq_internal.h"

namespace mxq {

namespace {

constexpr int kWarps = kHpassThreads / 32;
constexpr int kRowsPerStep = 8;
constexpr int kCtasPerSm = kHpassCtasPerSm;    // resident CTAs per SM (launch bounds)
constexpr int kTargetCtas = kHpassTargetCtas;   // one wave on a 148-SM B200

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Accumulate the squares of one 16-byte vector into acc (VEC/2 packed pairs).
template <bool BF16>
__device__ __forceinline__ void acc_sq(const uint4& v, float2* acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if constexpr (BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p = make_float2(bf16lo(w[i]), bf16hi(w[i]));
      acc[i] = __ffma2_rn(p, p, acc[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float2 p = make_float2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
      acc[i] = __ffma2_rn(p, p, acc[i]);
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kHpassThreads, kCtasPerSm)
k_hpass_partial(const char* __restrict__ X, int64_t rows, int64_t cols, int64_t ld_bytes,
                int64_t rows_per_chunk, double* __restrict__ partial) {
  constexpr int VEC = BF16 ? 8 : 4;       // elements per 16-byte load
  constexpr int NP = VEC / 2;             // packed pairs per load
  constexpr int STRIP = 32 * VEC;
  constexpr int EL = BF16 ? 2 : 4;
  __shared__ double red[kWarps][STRIP];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col = (int64_t)blockIdx.x * STRIP + (int64_t)lane * VEC;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_chunk;
  const int64_t r1 = min(rows, r0 + rows_per_chunk);

  double tot[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) tot[i] = 0.0;

  if (col < cols) {
    const char* base = X + col * EL;
    float2 acc[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) acc[i] = make_float2(0.f, 0.f);
    auto flush = [&]() {
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        tot[2 * i] += (double)acc[i].x;
        tot[2 * i + 1] += (double)acc[i].y;
        acc[i] = make_float2(0.f, 0.f);
      }
    };
    int64_t r = r0 + warp;
    int it = 0;
    // Eight rows per step (r, r+8, ..., r+56): eight 16-byte loads in flight per lane.
    for (; r + 7 * kWarps < r1; r += kRowsPerStep * kWarps) {
      uint4 v[kRowsPerStep];
#pragma unroll
      for (int u = 0; u < kRowsPerStep; ++u) v[u] = ld_stream(base + (r + u * kWarps) * ld_bytes);
#pragma unroll
      for (int u = 0; u < kRowsPerStep; ++u) acc_sq<BF16>(v[u], acc);
      if (++it == 32 / kRowsPerStep) {  // at most 32 rows per float accumulator
        flush();
        it = 0;
      }
    }
    for (; r < r1; r += kWarps) acc_sq<BF16>(ld_stream(base + r * ld_bytes), acc);
    flush();
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[warp][lane * VEC + i] = tot[i];
  __syncthreads();
  for (int c = threadIdx.x; c < STRIP; c += kHpassThreads) {
    const int64_t gc = (int64_t)blockIdx.x * STRIP + c;
    if (gc < cols) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[w][c];
      partial[(int64_t)blockIdx.y * cols + gc] = s;
    }
  }
}

__global__ void k_hpass_finalize(const double* __restrict__ partial, int64_t parts,
                                 int64_t cols, int64_t total_rows,
                                 double* __restrict__ colsum, float* __restrict__ h) {
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < cols;
       c += (int64_t)gridDim.x * blockDim.x) {
    double s = 0.0;
    for (int64_t p = 0; p < parts; ++p) s += partial[p * cols + c];
    if (colsum) colsum[c] = s;
    if (h) h[c] = total_rows > 0 ? (float)(s / (double)total_rows) : 0.0f;
  }
}

int strip_cols(int dtype) { return dtype == 1 ? 256 : 128; }

}  // namespace

int hpass_chunks(int64_t rows, int64_t cols, int dtype) {
  if (rows <= 0 || cols <= 0) return 1;
  const int64_t strips = (cols + strip_cols(dtype) - 1) / strip_cols(dtype);
  int64_t chunks = kTargetCtas / strips;   // strips x chunks <= one wave
  const int64_t by_rows = (rows + 255) / 256;  // at least ~256 rows per chunk
  if (chunks > by_rows) chunks = by_rows;
  if (chunks < 1) chunks = 1;
  if (chunks > 65535) chunks = 65535;
  return (int)chunks;
}

cudaError_t launch_hpass_partial(const void* X, int dtype, int64_t rows, int64_t cols,
                                 int64_t ld, int chunks, double* partial, cudaStream_t st) {
  const int64_t strips = (cols + strip_cols(dtype) - 1) / strip_cols(dtype);
  const int64_t rpc = (rows + chunks - 1) / chunks;
  dim3 grid((unsigned)strips, (unsigned)chunks);
  if (dtype == 1)
    k_hpass_partial<true><<<grid, kHpassThreads, 0, st>>>((const char*)X, rows, cols, ld * 2,
                                                          rpc, partial);
  else
    k_hpass_partial<false><<<grid, kHpassThreads, 0, st>>>((const char*)X, rows, cols, ld * 4,
                                                           rpc, partial);
  return cudaGetLastError();
}

cudaError_t launch_hpass_finalize(const double* partial, int64_t parts, int64_t cols,
                                  int64_t total_rows, double* colsum, float* h,
                                  cudaStream_t st) {
  const int threads = 256;
  int64_t blocks = (cols + threads - 1) / threads;
  if (blocks > 4096) blocks = 4096;
  k_hpass_finalize<<<(unsigned)blocks, threads, 0, st>>>(partial, parts, cols, total_rows,
                                                        colsum, h);
  return cudaGetLastError();
}

}  // namespace mxq
