// mxq_gram.cu -- Gram blocks G_b = X_b^T X_b / R of the calibration activations on the
// 5th-generation tensor cores ("quantization_algorithms.txt", section 1: the block
// objective || X_b (W_b - s Q(W_b / s))^T ||_F^2 = R d^T G_b d per row of a block).
//
// One CTA owns a strip of 128 columns of X [R, K] (bf16) and a range of rows. Per stage a
// 64-row x 128-column tile arrives by TMA (two 64 x 64 boxes, 128-byte swizzle); the same
// shared-memory tile is both MMA operands -- A = tile^T (M-major, M = the 128 columns) and
// B = tile (N-major) -- so D[128 x 128] += tile^T tile, accumulated in tensor memory in
// float32 (bf16 products are exact). Every 8 stages (512 rows) the accumulator is drained:
// the epilogue warps read their rows' diagonal blocks (tcgen05.ld) and add them into double
// registers, while the MMA warp fills the second accumulator. The CTA writes its double
// partials; k_gram_finalize sums the row ranges in a fixed order and writes
// G = fl32(sum / R) and h = diag(G). Only the B x B diagonal blocks of each 128 x 128 tile
// are kept: the kernel is bound by reading X, the discarded products are free.
//
// Blocks of B = 16, 32 or 64 columns (64: the E4M3 tile width).
// Warp roles (192 threads): warps 0-3 epilogue (tensor-memory lanes 32 (w % 4) ..), warp 4
// TMA producer, warp 5 MMA issuer. Every wait is bounded: on timeout the CTA sets
// `*err`, stops issuing, lets its copies and MMAs finish (bounded) and frees its tensor
// memory before returning.
#include "mxq_common.cuh"
#include "mxq_internal.h"
#include "mxq_tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

namespace mxq {

namespace {

constexpr int kGramCols = 128;               // columns per CTA (the MMA's M and N)
constexpr int kGramRows = 64;                // rows per stage (the MMA's K, 4 x 16)
constexpr int kStages = 6;
constexpr int kPeriod = 8;                   // stages accumulated in float32 per drain
constexpr int kStageBytes = kGramRows * kGramCols * 2;   // 16 KB: two 8 KB boxes
constexpr int kGramThreads = 192;
constexpr uint32_t kSpinLimit = 1u << 26;    // a wait that long means something is wrong

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity (at most `polls` polls); false on
// timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag, uint32_t polls) {
  for (uint32_t it = 0; it < polls; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 1023u && *abort_flag) return false;
  }
  return false;
}

// 128-byte-swizzled, MN-major shared-memory operand descriptor (tcgen05): start address,
// leading byte offset = stride between 64-element column groups (8 KB: the second box),
// stride byte offset = stride between 8-row groups (1 KB), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((8192u >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((1024u >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: D float32, A and B bf16, both MN-major,
// N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                            ((uint32_t)(kGramCols >> 3) << 17) | ((uint32_t)(kGramCols >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 32 consecutive float32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace
}  // namespace mxq

namespace mxq {
namespace {

struct GramParams {
  int64_t rows, cols;
  int64_t rows_per_chunk;  // a multiple of kGramRows: chunk boundaries fall on stage edges
  double* partial;         // [chunks][cols][B]: column c's row of its diagonal block
  int* err;
  uint32_t polls;          // bound of every pipeline wait (the drains keep kSpinLimit)
};

// Shared-memory layout (dynamic, 1024-byte aligned for the swizzle atoms).
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kGramSmem = kBarOffset + 256 + 1024;

template <int B>
__global__ void __launch_bounds__(kGramThreads, 1)
k_gram_tc(const __grid_constant__ CUtensorMap tmap, GramParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  if ((size_t)(smem - smem_raw) + kBarOffset + 256 > (size_t)kGramSmem) {  // never
    if (threadIdx.x == 0) atomicExch(P.err, 1);
    return;
  }
  uint64_t* full = (uint64_t*)(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* accfull = empty + kStages;   // [2]
  uint64_t* accempty = accfull + 2;      // [2]
  uint64_t* done = accempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col0 = (int64_t)blockIdx.x * kGramCols;
  const int64_t row_begin = (int64_t)blockIdx.y * P.rows_per_chunk;
  int64_t row_end = row_begin + P.rows_per_chunk;
  if (row_end > P.rows) row_end = P.rows;
  const int nst = row_end > row_begin ? (int)((row_end - row_begin + kGramRows - 1) / kGramRows) : 0;
  const int nper = (nst + kPeriod - 1) / kPeriod;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
        smem_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicExch(P.err, 1);
  };

  if (warp == 4) {
    // ---- TMA producer ----------------------------------------------------------------
    if (lane == 0) {
      int issued[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) issued[s] = 0;
      for (int it = 0; it < nst; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, P.polls)) { fail(); break; }
        mbar_expect_tx(&full[s], kStageBytes);
        const int y = (int)(row_begin + (int64_t)it * kGramRows);
        uint8_t* dst = smem + s * kStageBytes;
        tma_load_2d(dst, &tmap, (int)col0, y, &full[s]);
        tma_load_2d(dst + kStageBytes / 2, &tmap, (int)col0 + 64, y, &full[s]);
        ++issued[s];
      }
      // every copy this thread started has landed before the CTA can exit
#pragma unroll
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0 && !mbar_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u, abort_flag, P.polls)) {
          for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(&full[s], (uint32_t)(issued[s] - 1) & 1u); ++it) {
          }
        }
    }
  } else if (warp == 5) {
    // ---- MMA issuer ------------------------------------------------------------------
    if (lane == 0) {
      int it = 0;
      for (int per = 0; per < nper; ++per) {
        const int buf = per & 1;
        if (!mbar_wait(&accempty[buf], ((uint32_t)(per >> 1) & 1u) ^ 1u, abort_flag, P.polls)) {
          fail();
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d = tmem + (uint32_t)(buf * kGramCols);
        const int end = min(nst, (per + 1) * kPeriod);
        bool ok = true;
        for (; it < end; ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u, abort_flag, P.polls)) { ok = false; break; }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t base = smem_u32(smem + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kGramRows / 16; ++kk) {
            const uint64_t desc = smem_desc(base + (uint32_t)kk * 2048u);  // 16 rows = 2 KB
            mma_bf16(d, desc, desc, (it != per * kPeriod || kk != 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) { fail(); break; }
        mma_commit(&accfull[buf]);
      }
      // all MMAs issued by this thread are complete before the tensor memory is freed
      mma_commit(done);
      for (uint32_t i = 0; i < kSpinLimit && !mbar_try_wait(done, 0); ++i) {
      }
    }
  } else {
    // ---- epilogue: warps 0-3, tensor-memory lanes 32 w .. 32 w + 31 --------------------
    const int m = warp * 32 + lane;  // column of the strip = accumulator row
    double acc[B];
#pragma unroll
    for (int j = 0; j < B; ++j) acc[j] = 0.0;
    const bool upper = B == 16 && lane >= 16;  // B = 16: lanes 16-31 own the second block
    for (int per = 0; per < nper; ++per) {
      const int buf = per & 1;
      const bool ok = mbar_wait(&accfull[buf], (uint32_t)(per >> 1) & 1u, abort_flag, P.polls);
      if (!__all_sync(kFull, ok)) {
        if (lane == 0) fail();
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t lanes = (uint32_t)(warp * 32) << 16;
      if constexpr (B == 64) {
        // lanes 32 w .. 32 w + 31 all lie in diagonal block w / 2: its 64 columns
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          float v[32];
          tmem_ld32(tmem + lanes + (uint32_t)(buf * kGramCols + (warp / 2) * 64 + hlf * 32), v);
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[hlf * 32 + j] += (double)v[j];
        }
      } else {
        float v[32];
        tmem_ld32(tmem + lanes + (uint32_t)(buf * kGramCols + warp * 32), v);
#pragma unroll
        for (int j = 0; j < B; ++j) acc[j] += (double)(B == 16 ? (upper ? v[16 + j] : v[j]) : v[j]);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      mbar_arrive(&accempty[buf]);
    }
    if (col0 + m < P.cols) {
      double* out = P.partial + ((int64_t)blockIdx.y * P.cols + col0 + m) * B;
#pragma unroll
      for (int j = 0; j < B; ++j) out[j] = acc[j];
    }
  }
  __syncthreads();
  if (warp == 5) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem));
  }
}

// G[b][i][j] = fl32(sum over chunks (ascending) of partial[chunk][b B + i][j] / rows);
// h[c] = G[c / B][c % B][c % B]. A timed-out Gram launch (err set) leaves NaN.
__global__ void k_gram_finalize(const double* __restrict__ partial, int chunks, int64_t cols,
                                int B, int64_t rows, const int* __restrict__ err,
                                float* __restrict__ G, float* __restrict__ h) {
  const int64_t total = cols * B;
  const bool bad = *err != 0;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    double s = 0.0;
    for (int c = 0; c < chunks; ++c) s += partial[(int64_t)c * total + t];
    const float g = bad ? __int_as_float(0x7fc00000) : (float)(s / (double)rows);
    const int64_t c = t / B;
    const int j = (int)(t - c * B);
    G[(c / B) * B * B + (c % B) * B + j] = g;
    if (h && j == c % B) h[c] = g;
  }
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_bf16_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                    uint32_t box_cols, uint32_t box_rows) {
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, ld, box_cols,
                   box_rows);
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, int elsize, const void* base,
               int64_t rows, int64_t cols, int64_t ld, uint32_t box_cols, uint32_t box_rows) {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return (EncodeTiledFn)p;
  }();
  if (!fn) return false;
  std::memset(map, 0, sizeof *map);
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * (cuuint64_t)elsize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, type, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gram_chunks(int64_t rows, int64_t cols, int B) {
  const int64_t strips = (cols + kGramCols - 1) / kGramCols;
  const int64_t stages = (rows + kGramRows - 1) / kGramRows;
  int64_t want = (8 * 2 * (int64_t)sm_count() + strips - 1) / strips;  // ~8 waves of 2 CTAs/SM
  // the partial sums (chunks x cols x B doubles, written and read back) stay within a quarter
  // of X's bytes: chunks <= rows / (16 B)
  const int64_t cap = rows / (16 * (int64_t)B);
  if (want > cap) want = cap;
  if (want > stages) want = stages;
  return (int)(want < 1 ? 1 : want);
}

size_t gram_workspace(int64_t rows, int64_t cols, int B) {
  return 256 + (size_t)gram_chunks(rows, cols, B) * (size_t)cols * (size_t)B * sizeof(double);
}

cudaError_t launch_gram(const void* X, int64_t rows, int64_t cols, int64_t ld, int B, float* G,
                        float* h, void* workspace, cudaStream_t st) {
  CUtensorMap map;
  if (!encode_bf16_2d(&map, X, rows, cols, ld, 64, kGramRows)) return cudaErrorInvalidValue;
  const int chunks = gram_chunks(rows, cols, B);
  const int64_t stages = (rows + kGramRows - 1) / kGramRows;
  const int64_t per_chunk = (stages + chunks - 1) / chunks * kGramRows;
  int* err = (int*)workspace;
  double* partial = (double*)((char*)workspace + 256);
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  GramParams P{rows, cols, per_chunk, partial, err, wait_polls()};
  const dim3 grid((unsigned)((cols + kGramCols - 1) / kGramCols), (unsigned)chunks);
  if (B == 16) {
    e = ensure_dynamic_smem((const void*)k_gram_tc<16>, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    k_gram_tc<16><<<grid, kGramThreads, kGramSmem, st>>>(map, P);
  } else if (B == 64) {
    e = ensure_dynamic_smem((const void*)k_gram_tc<64>, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    k_gram_tc<64><<<grid, kGramThreads, kGramSmem, st>>>(map, P);
  } else {
    e = ensure_dynamic_smem((const void*)k_gram_tc<32>, (int)kGramSmem);
    if (e != cudaSuccess) return e;
    k_gram_tc<32><<<grid, kGramThreads, kGramSmem, st>>>(map, P);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = cols * B;
  int64_t fg = (total + 255) / 256;
  if (fg > 4096) fg = 4096;
  k_gram_finalize<<<(unsigned)fg, 256, 0, st>>>(partial, chunks, cols, B, rows, err, G, h);
  return cudaGetLastError();
}

}  // namespace mxq
