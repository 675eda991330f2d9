// mxq_gram_full.cu -- the full Gram matrix H = X^T X / R of the calibration activations on
// the 5th-generation tensor cores: GPTQ's Hessian up to a factor (qwantize "Results", "GPTQ
// Quantization": each block's error is compensated through the inverse Hessian).
//
// H is symmetric, so only the tiles that reach the upper triangle are multiplied out; a
// transpose then copies the upper triangle onto the lower one (H comes out exactly
// symmetric). The contraction runs over the R rows of X [R, K] (bf16, row-major), so both
// operands are MN-major: a tile of 64 rows x 64 columns of X is 64 K-steps of 64 M (or N)
// values, which a 2-D TMA box with 128-byte swizzle lands in the layout the MMA reads.
//
// Work split. A pair of CTAs on neighbouring SMs (a cluster of two) computes one 256 x 512
// tile of H with tcgen05.mma.cta_group::2 (M = 256: rows i0 .. i0 + 255 of H, 128 in each
// CTA; N = 256 per instruction, two accumulators = 512 columns j0 .. j0 + 511, all 512
// tensor-memory columns of each SM). Per 64-row stage each CTA loads its 128 columns of A
// and its 2 x 128 columns of B (48 KB, six 8 KB boxes; four stages in flight); the copies of
// both CTAs complete on the even CTA's stage barrier, one thread there issues the 8 MMAs of
// the stage, and its commits free the stage in both CTAs. The K loop runs over all R rows, so
// a tile's accumulator holds float32 sums of R bf16 products (each product exact). The
// pairs are persistent: tile t goes to pair t mod P. The tiles of the last, partial wave are
// cut along R into equal chunks so that every pair gets one: those chunks write float32
// partial tiles into the workspace and k_gf_reduce adds each tile's chunks in a fixed order,
// so the result does not depend on timing.
//
// Warp roles (192 threads per CTA): warps 0-3 drain the accumulators (tensor-memory lanes
// 32 w .. 32 w + 31 = H rows) and store H; warp 4 issues the TMA copies; warp 5 issues the
// MMAs (even CTA) and owns the tensor-memory allocation (both CTAs). Each CTA loads only
// its own tiles, into its own shared memory, from this GPU's memory. Every wait is bounded: on
// timeout a CTA sets the error word and its peer's abort flag, and the final transpose then
// writes NaN over all of H.
#include "mxq_common.cuh"
#include "mxq_internal.h"
#include "mxq_tc.cuh"

#include <cstring>

namespace mxq {
namespace {

constexpr int kGfM = 256;                   // pair tile rows
constexpr int kGfN = 512;                   // pair tile columns (two N = 256 accumulators)
constexpr int kGfRows = 64;                 // X rows per stage (the MMA's K: 4 x 16)
constexpr int kGfStages = 4;
constexpr int kGfBox = 64 * 64 * 2;         // one 64-row x 64-column bf16 box: 8 KB
constexpr int kGfA = 2 * kGfBox;            // this CTA's 128 columns of A
constexpr int kGfB = 2 * kGfBox;            // this CTA's 128 columns of one accumulator's B
constexpr int kGfStage = kGfA + 2 * kGfB;   // 48 KB
constexpr int kGfThreads = 192;
constexpr int kGfBarOff = kGfStages * kGfStage;
constexpr int kGfSmem = kGfBarOff + 256 + 1024;
constexpr uint32_t kGfIdesc = tc::idesc_bf16_mn(256, 256);
constexpr int kGfTileElems = kGfM * kGfN;

static_assert(kGfSmem <= 227 * 1024, "shared memory per CTA");

// The work list: `tiles` upper-triangle tiles in row-major order of (I, J), J >= I / 2;
// tiles [0, full) are processed whole, each later tile as `split` chunks of split_rows rows.
struct GfSchedule {
  int64_t rows, cols;
  int ni, nj;            // 256-row strips and 512-column strips of H
  int tiles, full, split;
  int64_t split_rows;    // a multiple of kGfRows
  int units;             // full + (tiles - full) * split
  int pairs;
};

struct GfParams {
  GfSchedule S;
  float* H;
  float* partial;        // [(tiles - full) * split][256][512]
  int* err;
  uint32_t polls;
  double inv_rows;
};

__host__ __device__ inline int gf_tiles_in_row(int I, int nj) { return nj - I / 2; }

// Tile t -> (I, J) in the row-major order of the upper-triangle tiles.
__host__ __device__ inline void gf_tile(int t, int ni, int nj, int& I, int& J) {
  int I_ = 0;
  while (I_ < ni - 1 && t >= gf_tiles_in_row(I_, nj)) {
    t -= gf_tiles_in_row(I_, nj);
    ++I_;
  }
  I = I_;
  J = I_ / 2 + t;
}

struct GfUnit {
  int I, J;
  int64_t r0;
  int nst;          // stages (64-row steps)
  int slot;         // partial slot, or -1 for a whole tile
};

__device__ inline GfUnit gf_unit(const GfSchedule& S, int u) {
  GfUnit w;
  int t;
  if (u < S.full) {
    t = u;
    w.r0 = 0;
    w.nst = (int)((S.rows + kGfRows - 1) / kGfRows);
    w.slot = -1;
  } else {
    const int v = u - S.full;
    t = S.full + v / S.split;
    w.r0 = (int64_t)(v % S.split) * S.split_rows;
    int64_t r1 = w.r0 + S.split_rows;
    if (r1 > S.rows) r1 = S.rows;
    w.nst = (int)((r1 - w.r0 + kGfRows - 1) / kGfRows);
    w.slot = v;
  }
  gf_tile(t, S.ni, S.nj, w.I, w.J);
  return w;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGfThreads, 1)
k_gram_full(const __grid_constant__ CUtensorMap tmap, GfParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + kGfBarOff);     // [stages]  (even CTA)
  uint64_t* empty = full + kGfStages;                 // [stages]  (both)
  uint64_t* accfull = empty + kGfStages;              // (both)
  uint64_t* accempty = accfull + 1;                   // (even CTA; 4 warps x 2 CTAs)
  uint64_t* done = accempty + 1;                      // (even CTA)
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const bool even = rank == 0;
  const int pair = blockIdx.x >> 1;
  const GfSchedule& S = P.S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGfStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(accfull, 1);
    tc::mbar_init(accempty, 8);
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::mbar_init_fence();
  }
  if (warp == 5) {
    tc::tmem_alloc_pair(tmem_slot, 512);
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::cluster_sync();       // both CTAs' barriers initialised before any remote signal
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // on failure: this CTA's roles and the peer's stop, and the result is marked bad
  auto fail = [&]() {
    *abort_flag = 1;
    tc::st_cluster_u32(tc::mapa(tc::smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
    atomicExch(P.err, 1);
  };
  bool aborted = false;

  if (warp == 4) {
    // ---- TMA producer (both CTAs) ------------------------------------------------------
    if (lane == 0) {
      uint32_t it = 0;
      for (int u = pair; u < S.units && !aborted; u += S.pairs) {
        const GfUnit w = gf_unit(S, u);
        const int xa = w.I * kGfM + 128 * (int)rank;
        const int xb0 = w.J * kGfN + 128 * (int)rank;
        const int xb1 = xb0 + 256;
        for (int st = 0; st < w.nst; ++st, ++it) {
          const int s = (int)(it % kGfStages);
          const uint32_t ph = (it / kGfStages) & 1u;
          if (!tc::mbar_wait(&empty[s], ph ^ 1u, abort_flag, P.polls)) {
            fail();
            aborted = true;
            break;
          }
          if (even) tc::mbar_expect_tx(&full[s], 2 * kGfStage);
          const uint32_t bar = tc::mapa(tc::smem_u32(&full[s]), 0);
          const int y = (int)(w.r0 + (int64_t)st * kGfRows);
          uint8_t* dst = smem + s * kGfStage;
          tc::tma_load_2d_pair(dst, &tmap, xa, y, bar);
          tc::tma_load_2d_pair(dst + kGfBox, &tmap, xa + 64, y, bar);
          tc::tma_load_2d_pair(dst + kGfA, &tmap, xb0, y, bar);
          tc::tma_load_2d_pair(dst + kGfA + kGfBox, &tmap, xb0 + 64, y, bar);
          tc::tma_load_2d_pair(dst + kGfA + kGfB, &tmap, xb1, y, bar);
          tc::tma_load_2d_pair(dst + kGfA + kGfB + kGfBox, &tmap, xb1 + 64, y, bar);
        }
      }
    }
  } else if (warp == 5) {
    // ---- MMA issuer (even CTA) ---------------------------------------------------------
    if (lane == 0 && even) {
      const uint32_t peer_empty0 = tc::mapa(tc::smem_u32(&empty[0]), 1);
      const uint32_t peer_accfull = tc::mapa(tc::smem_u32(accfull), 1);
      uint32_t it = 0, k = 0;
      for (int u = pair; u < S.units && !aborted; u += S.pairs, ++k) {
        const GfUnit w = gf_unit(S, u);
        if (!tc::mbar_wait(accempty, (k & 1u) ^ 1u, abort_flag, P.polls)) {
          fail();
          aborted = true;
          break;
        }
        tc::fence_after_sync();
        for (int st = 0; st < w.nst; ++st, ++it) {
          const int s = (int)(it % kGfStages);
          if (!tc::mbar_wait(&full[s], (it / kGfStages) & 1u, abort_flag, P.polls)) {
            fail();
            aborted = true;
            break;
          }
          tc::fence_after_sync();
          const uint32_t base = tc::smem_u32(smem + s * kGfStage);
#pragma unroll
          for (int kk = 0; kk < kGfRows / 16; ++kk) {
            const uint32_t off = (uint32_t)kk * 2048u;   // 16 rows of a 128-byte-row box
            const uint64_t a = tc::desc_mn_sw128(base + off, kGfBox);
            const uint64_t b0 = tc::desc_mn_sw128(base + kGfA + off, kGfBox);
            const uint64_t b1 = tc::desc_mn_sw128(base + kGfA + kGfB + off, kGfBox);
            const uint32_t acc = (st | kk) != 0 ? 1u : 0u;
            tc::mma_pair_f16(tmem, a, b0, kGfIdesc, acc);
            tc::mma_pair_f16(tmem + 256, a, b1, kGfIdesc, acc);
          }
          tc::commit_pair(tc::smem_u32(&empty[s]));
          tc::commit_pair(peer_empty0 + (uint32_t)s * 8u);
        }
        if (aborted) break;
        tc::commit_pair(tc::smem_u32(accfull));
        tc::commit_pair(peer_accfull);
      }
      // every MMA issued here has completed before the tensor memory can be freed
      tc::commit_pair(tc::smem_u32(done));
      for (uint32_t i = 0; i < tc::kDefaultPolls && !tc::mbar_try_wait(done, 0); ++i) {
      }
    }
  } else {
    // ---- epilogue: warps 0-3 of both CTAs ----------------------------------------------
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    const int m = 128 * (int)rank + warp * 32 + lane;     // row of the pair tile
    const uint32_t lead_accempty = tc::mapa(tc::smem_u32(accempty), 0);
    uint32_t k = 0;
    for (int u = pair; u < S.units; u += S.pairs, ++k) {
      const GfUnit w = gf_unit(S, u);
      const bool ok = tc::mbar_wait(accfull, k & 1u, abort_flag, P.polls);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0 && !*abort_flag) fail();
        break;
      }
      tc::fence_after_sync();
      const int64_t row = (int64_t)w.I * kGfM + m;
#pragma unroll 1
      for (int c = 0; c < kGfN / 32; ++c) {
        float v[32];
        tc::tmem_ld32(tmem + lanes + (uint32_t)(c * 32), v);
        if (w.slot >= 0) {
          float4* dst = (float4*)(P.partial + ((int64_t)w.slot * kGfM + m) * kGfN + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else if (row < S.cols) {
          const int64_t col = (int64_t)w.J * kGfN + c * 32;
          float* dst = P.H + row * S.cols + col;
          if (col + 32 <= S.cols && (S.cols & 3) == 0) {        // 16-byte aligned rows
#pragma unroll
            for (int q = 0; q < 8; ++q)
              ((float4*)dst)[q] = make_float4((float)((double)v[4 * q] * P.inv_rows),
                                              (float)((double)v[4 * q + 1] * P.inv_rows),
                                              (float)((double)v[4 * q + 2] * P.inv_rows),
                                              (float)((double)v[4 * q + 3] * P.inv_rows));
          } else {
            for (int q = 0; q < 32 && col + q < S.cols; ++q)
              dst[q] = (float)((double)v[q] * P.inv_rows);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster(lead_accempty);
    }
  }
  __syncthreads();
  // Copies complete on the even CTA's barriers, which the odd CTA cannot watch. On the normal
  // path every copy was consumed by an MMA that the accumulator hand-off waited for; after
  // an abort (either CTA sets both flags), give copies still in flight time to land before
  // shared memory can be released: a copy takes microseconds, this waits about a
  // millisecond, and the cluster barrier keeps the other CTA until then too.
  if (*abort_flag) {
    if (threadIdx.x == 0)
      for (int i = 0; i < 1000; ++i) __nanosleep(1000);
    __syncthreads();
  }
  tc::cluster_sync();       // neither CTA leaves while the other may still signal it
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, 512);
  }
}

// H tiles of the last wave: the sum of each tile's chunks in ascending order (double), / R.
__global__ void __launch_bounds__(256)
k_gf_reduce(const float* __restrict__ partial, GfSchedule S, double inv_rows, float* H) {
  const int v = blockIdx.y;                       // tail tile
  int I, J;
  gf_tile(S.full + v, S.ni, S.nj, I, J);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < kGfTileElems;
       e += gridDim.x * blockDim.x) {
    const int64_t row = (int64_t)I * kGfM + e / kGfN, col = (int64_t)J * kGfN + e % kGfN;
    if (row >= S.cols || col >= S.cols) continue;
    double s = 0.0;
    for (int c = 0; c < S.split; ++c)
      s += (double)partial[((int64_t)v * S.split + c) * kGfTileElems + e];
    H[row * S.cols + col] = (float)(s * inv_rows);
  }
}

constexpr int kMirror = 32;

// H[p][q] = H[q][p] for q < p; one 32 x 32 tile of the lower triangle per CTA (32 x 8
// threads). After a timed-out product (*err set) every entry becomes NaN instead.
__global__ void __launch_bounds__(256) k_mirror_lower(float* H, int64_t k, const int* err) {
  __shared__ float tile[kMirror][kMirror + 1];
  const int tq = blockIdx.x, tp = blockIdx.y;
  if (tq > tp) return;
  const int tx = threadIdx.x % kMirror, ty = threadIdx.x / kMirror;
  if (*err) {
    const float nan = __int_as_float(0x7fc00000);
#pragma unroll
    for (int r = 0; r < kMirror; r += 8) {
      const int64_t a = (int64_t)tq * kMirror + ty + r, b = (int64_t)tp * kMirror + tx;
      if (a < k && b < k) {
        H[a * k + b] = nan;
        H[b * k + a] = nan;
      }
    }
    return;
  }
#pragma unroll
  for (int r = 0; r < kMirror; r += 8) {
    const int64_t q = (int64_t)tq * kMirror + ty + r, pc = (int64_t)tp * kMirror + tx;
    if (q < k && pc < k) tile[ty + r][tx] = H[q * k + pc];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMirror; r += 8) {
    const int64_t pr = (int64_t)tp * kMirror + ty + r, q = (int64_t)tq * kMirror + tx;
    if (pr < k && q < pr) H[pr * k + q] = tile[tx][ty + r];
  }
}

GfSchedule gf_schedule(int64_t rows, int64_t cols) {
  GfSchedule S{};
  S.rows = rows;
  S.cols = cols;
  S.ni = (int)((cols + kGfM - 1) / kGfM);
  S.nj = (int)((cols + kGfN - 1) / kGfN);
  int64_t tiles = 0;
  for (int I = 0; I < S.ni; ++I) tiles += gf_tiles_in_row(I, S.nj);
  S.tiles = (int)tiles;
  const int pairs = sm_count() / 2 > 0 ? sm_count() / 2 : 1;
  const int64_t stages = (rows + kGfRows - 1) / kGfRows;
  S.full = (S.tiles / pairs) * pairs;
  const int tail = S.tiles - S.full;
  S.split = 1;
  S.split_rows = stages * kGfRows;
  if (tail > 0) {
    int64_t want = pairs / tail;
    if (want < 1) want = 1;
    if (want > stages) want = stages;
    const int64_t per = (stages + want - 1) / want;        // stages per chunk
    S.split = (int)((stages + per - 1) / per);             // every chunk non-empty
    S.split_rows = per * kGfRows;
  }
  S.units = S.full + tail * S.split;
  S.pairs = S.units < pairs ? S.units : pairs;
  return S;
}

}  // namespace

size_t gram_full_workspace(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 256;
  const GfSchedule S = gf_schedule(rows, cols);
  return 256 + (size_t)(S.tiles - S.full) * S.split * kGfTileElems * sizeof(float);
}

cudaError_t launch_gram_full(const void* X, int64_t rows, int64_t cols, int64_t ld, float* H,
                             void* workspace, cudaStream_t st, const char** why) {
  const int64_t mt = (cols + kMirror - 1) / kMirror;
  if (mt > 65535) {                     // the transpose's grid; H would hold over 4e12 entries
    *why = "cols beyond 65535 * 32";
    return cudaErrorUnknown;
  }
  const GfSchedule S = gf_schedule(rows, cols);
  CUtensorMap map;
  if (!encode_bf16_2d(&map, X, rows, cols, ld, 64, kGfRows)) {
    *why = "tensor map of X rejected";
    return cudaErrorUnknown;
  }
  int* err = (int*)workspace;
  float* partial = (float*)((char*)workspace + 256);
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem((const void*)k_gram_full, kGfSmem);
  if (e != cudaSuccess) return e;
  GfParams p{S, H, partial, err, wait_polls(), 1.0 / (double)rows};
  k_gram_full<<<2 * S.pairs, kGfThreads, kGfSmem, st>>>(map, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (S.tiles > S.full) {
    k_gf_reduce<<<dim3(64, (unsigned)(S.tiles - S.full)), 256, 0, st>>>(partial, S, 1.0 / (double)rows,
                                                                       H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  k_mirror_lower<<<dim3((unsigned)mt, (unsigned)mt), 256, 0, st>>>(H, cols, err);
  return cudaGetLastError();
}

}  // namespace mxq
